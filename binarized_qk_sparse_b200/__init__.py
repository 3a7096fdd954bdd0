"""Python binding of the binarized-QK top-N attention library (include/had.h).

Thin ctypes marshalling over ``libhad_b200.so``: every step of the method runs
in the library's sm_100a kernels.  PyTorch supplies device memory and the
current CUDA stream.  There is no fallback: if the shared library or a CUDA
device is missing, calls raise.

Method ("Hamming Attention Distillation" top-N over binarized keys and
queries; "BinaryAttention" §2.2-§2.4 scaled binarization, bias, uint8 A x
int8 V): see include/had.h for the exact formulas and layouts.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhad_b200.so")

HAD_OK, HAD_ERR_INVALID, HAD_ERR_UNSUPPORTED, HAD_ERR_CUDA, HAD_ERR_DEVICE, HAD_ERR_TIMEOUT = range(6)
HAD_F32, HAD_BF16 = 0, 1
HAD_MODE_FLOAT, HAD_MODE_U8I8, HAD_MODE_U8I4 = 0, 1, 2
_MODES = {"float": HAD_MODE_FLOAT, "u8i8": HAD_MODE_U8I8, "u8i4": HAD_MODE_U8I4, HAD_MODE_FLOAT: HAD_MODE_FLOAT,
          HAD_MODE_U8I8: HAD_MODE_U8I8, HAD_MODE_U8I4: HAD_MODE_U8I4}


class HadError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = lib().had_status_string(status).decode()
        if status == HAD_ERR_CUDA:
            msg += f" ({lib().had_last_cuda_error().decode()})"
        super().__init__(f"{what}: {msg}")


class had_shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("n", ctypes.c_int), ("d", ctypes.c_int),
                ("in_dtype", ctypes.c_int), ("seqlens", ctypes.c_void_p)]


class had_relpos_bias(ctypes.Structure):
    _fields_ = [("table", ctypes.c_void_p), ("gh", ctypes.c_int), ("gw", ctypes.c_int), ("prefix", ctypes.c_int),
                ("dense", ctypes.c_int)]


@dataclass
class RelPosBias:
    """Per-head relative-position table [H, 2gh-1, 2gw-1] (fp32, on the device)."""
    table: torch.Tensor
    gh: int
    gw: int
    prefix: int = 0


@dataclass
class DenseBias:
    """Per-head dense bias matrix [H, n, n] (fp32): b_ij = table[h, i, j]."""
    table: torch.Tensor


def _bias_c(bias):
    if isinstance(bias, DenseBias):
        return had_relpos_bias(bias.table.data_ptr(), 0, 0, 0, 1)
    return had_relpos_bias(bias.table.data_ptr(), bias.gh, bias.gw, bias.prefix, 0)


_lib = None


def lib():
    """Load the in-tree CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing (run binarized_qk_sparse_b200._build)")
        L = ctypes.CDLL(LIB_PATH)
        P, I, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        SP, BP = ctypes.POINTER(had_shape), ctypes.POINTER(had_relpos_bias)
        L.had_binarize_pack_workspace_size.argtypes = [SP]
        L.had_binarize_pack_workspace_size.restype = SZ
        L.had_binarize_pack.argtypes = [P, SP, P, P, P, P, SZ, P]
        L.had_binarize_pack_noalloc.argtypes = [P, SP, P, P, P]
        L.had_attention_workspace_size.argtypes = [SP, I, I, BP]
        L.had_attention_workspace_size.restype = SZ
        L.had_attention.argtypes = [P, P, P, SP, BP, P, P, I, I, P, I, P, SZ, P]
        L.had_attention_host_workspace_size.argtypes = [SP, I, I, BP, I]
        L.had_attention_host_workspace_size.restype = SZ
        L.had_attention_host.argtypes = [P, P, P, SP, BP, P, P, I, I, P, I, I, P, SZ, P]
        L.had_dense_reference_workspace_size.argtypes = [SP, BP]
        L.had_dense_reference_workspace_size.restype = SZ
        L.had_dense_reference_mode.argtypes = [P, P, P, SP, BP, I, P, I, P, SZ, P]
        L.had_scores_int.argtypes = [P, P, SP, P, P]
        L.had_topn_indices.argtypes = [P, P, SP, BP, P, P, I, P, P, SZ, P]
        L.had_attention_codes_u8.argtypes = [P, P, P, SP, BP, P, P, I, I, I, P, P, SZ, P]
        L.had_quantize_v.argtypes = [P, SP, P, P, P, SZ, P]
        L.had_quantize_v4.argtypes = [P, SP, P, P, P, SZ, P]
        L.had_attention_prepare.argtypes = [P, P, P, SP, BP, I, I, P, SZ, P]
        L.had_attention_prepared.argtypes = [P, SP, BP, P, P, I, I, P, I, P, SZ, P]
        L.had_qkv_workspace_size.argtypes = [SP, I, I, I, BP]
        L.had_qkv_workspace_size.restype = SZ
        L.had_qkv_prepare.argtypes = [P, P, SP, I, BP, I, I, P, P, SZ, P]
        for f in ("had_binarize_pack", "had_binarize_pack_noalloc", "had_attention", "had_attention_host",
                  "had_dense_reference_mode", "had_scores_int",
                  "had_topn_indices", "had_attention_codes_u8", "had_quantize_v", "had_quantize_v4",
                  "had_attention_prepare", "had_attention_prepared", "had_qkv_prepare",
                  "had_get_device_status"):
            getattr(L, f).restype = I
        L.had_attention_scores.argtypes = [P, P, SP, P, P, SZ, P]
        L.had_attention_scores.restype = I
        L.had_debug_bounded_wait.argtypes = [ctypes.c_longlong, I]
        L.had_debug_bounded_wait.restype = I
        L.had_probe_mma_rate.argtypes = [I, I, P, P]
        L.had_probe_mma_rate.restype = I
        L.had_get_device_status.argtypes = []
        L.had_status_string.argtypes = [I]
        L.had_status_string.restype = ctypes.c_char_p
        L.had_last_cuda_error.argtypes = []
        L.had_last_cuda_error.restype = ctypes.c_char_p
        L.had_version.restype = I
        _lib = L
    return _lib


# ----------------------------------------------------------------------------- marshalling helpers

def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return HAD_BF16
    if t.dtype == torch.float32:
        return HAD_F32
    raise TypeError(f"unsupported dtype {t.dtype}; Q/K/V must be bfloat16 or float32")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check_dev(*ts):
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("tensors must live on a CUDA device")
            if not t.is_contiguous():
                raise ValueError("tensors must be contiguous")


def make_shape(X: torch.Tensor, seqlens: torch.Tensor | None = None) -> had_shape:
    B, H, n, d = X.shape
    if seqlens is not None and seqlens.dtype != torch.int32:
        raise TypeError("seqlens must be int32")
    return had_shape(B, H, n, d, _dtype_code(X), None if seqlens is None else seqlens.data_ptr())


def _bias_struct(bias: RelPosBias | None):
    if bias is None:
        return None
    if bias.table.dtype != torch.float32:
        raise TypeError("bias table must be float32")
    _check_dev(bias.table)
    return ctypes.byref(_bias_c(bias))


def _alpha(a, H):
    if a is None:
        return None, None
    arr = (ctypes.c_float * H)(*[float(x) for x in a])
    return arr, ctypes.cast(arr, ctypes.c_void_p)


def _raise(st, what):
    if st != HAD_OK:
        raise HadError(st, what)


def _workspace(nbytes: int, device, workspace, stream=None):
    if workspace is not None:
        if workspace.numel() * workspace.element_size() < nbytes:
            raise ValueError("workspace too small")
        return workspace
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)
    if stream is not None:
        # the allocation belongs to the current stream; the kernels run on `stream`,
        # so the caching allocator must not hand the block out again before they finish
        ws.record_stream(stream)
    return ws


# ----------------------------------------------------------------------------- entry points

def had_binarize_pack(X, seqlens=None, mu_in=None, want_mu=True, workspace=None, stream=None):
    """Sign bits of X - mu packed to uint32 [B,H,n,d/32] (bit 1 = negative), and mu [B,H,d] fp32."""
    _check_dev(X, seqlens, mu_in)
    B, H, n, d = X.shape
    shp = make_shape(X, seqlens)
    bits = torch.empty((B, H, n, d // 32), dtype=torch.int32, device=X.device)
    mu = torch.empty((B, H, d), dtype=torch.float32, device=X.device) if want_mu else None
    ws = None
    if mu_in is None:
        ws = _workspace(lib().had_binarize_pack_workspace_size(ctypes.byref(shp)), X.device, workspace, stream)
    st = lib().had_binarize_pack(_ptr(X), ctypes.byref(shp), _ptr(mu_in), _ptr(mu), _ptr(bits), _ptr(ws),
                                 0 if ws is None else ws.numel(), _stream(stream))
    _raise(st, "had_binarize_pack")
    return bits, (mu if mu_in is None else mu_in)


def had_binarize_pack_noalloc(X, seqlens=None, bits=None, mu=None, stream=None):
    """had_binarize_pack with the library's own fixed device scratch instead of a workspace.

    For callers that cannot allocate device memory when they call (the library
    allocates nothing either).  Shapes with B*H*ceil(n/64) > 8192 are rejected;
    concurrent calls on one device share the scratch and must be serialized.
    Returns (bits [B,H,n,d/32] int32 view of the uint32 words, mu [B,H,d] fp32).
    """
    _check_dev(X, seqlens, bits, mu)
    B, H, n, d = X.shape
    shp = make_shape(X, seqlens)
    if bits is None:
        bits = torch.empty((B, H, n, d // 32), dtype=torch.int32, device=X.device)
    elif bits.shape != (B, H, n, d // 32) or bits.dtype not in (torch.int32, torch.uint32) or bits.device != X.device:
        raise ValueError(f"bits must be int32 [{B}, {H}, {n}, {d // 32}] on {X.device}")
    if mu is None:
        mu = torch.empty((B, H, d), dtype=torch.float32, device=X.device)
    elif mu.shape != (B, H, d) or mu.dtype != torch.float32 or mu.device != X.device:
        raise ValueError(f"mu must be float32 [{B}, {H}, {d}] on {X.device}")
    st = lib().had_binarize_pack_noalloc(_ptr(X), ctypes.byref(shp), _ptr(mu), _ptr(bits), _stream(stream))
    _raise(st, "had_binarize_pack_noalloc")
    return bits, mu


def had_attention_workspace_size(X, N=0, mode="float", seqlens=None, bias=None) -> int:
    shp = make_shape(X, seqlens)
    return int(lib().had_attention_workspace_size(ctypes.byref(shp), int(N), _MODES[mode], _bias_struct(bias)))


def had_attention(Q, K, V, N=0, mode="float", seqlens=None, bias=None, alpha_q=None, alpha_k=None, out=None,
                  out_dtype=None, workspace=None, stream=None):
    """Binarized-QK top-N attention; returns O [B,H,n,d] (dtype of V unless out/out_dtype say otherwise)."""
    _check_dev(Q, K, V, seqlens, out, workspace)
    B, H, n, d = Q.shape
    shp = make_shape(Q, seqlens)
    m = _MODES[mode]
    if out is None:
        out = torch.empty((B, H, n, d), dtype=out_dtype or V.dtype, device=Q.device)
    bs = _bias_struct(bias)
    ws = _workspace(lib().had_attention_workspace_size(ctypes.byref(shp), int(N), m, bs), Q.device, workspace,
                    stream)
    aq_keep, aq = _alpha(alpha_q, H)
    ak_keep, ak = _alpha(alpha_k, H)
    st = lib().had_attention(_ptr(Q), _ptr(K), _ptr(V), ctypes.byref(shp), bs, aq, ak, int(N), m, _ptr(out),
                             _dtype_code(out), _ptr(ws), ws.numel(), _stream(stream))
    _raise(st, "had_attention")
    return out


def _check_host(*ts):
    for t in ts:
        if t is not None:
            if t.device.type != "cpu":
                raise ValueError("had_attention_host takes host (CPU) tensors")
            if not t.is_contiguous():
                raise ValueError("tensors must be contiguous")


def _host_bias_struct(bias: RelPosBias | None):
    if bias is None:
        return None
    if bias.table.dtype != torch.float32:
        raise TypeError("bias table must be float32")
    _check_host(bias.table)
    return ctypes.byref(_bias_c(bias))


def had_attention_host_workspace_size(X, N=0, mode="float", seqlens=None, bias=None, chunk_b=0) -> int:
    shp = make_shape(X, seqlens)
    return int(lib().had_attention_host_workspace_size(ctypes.byref(shp), int(N), _MODES[mode],
                                                       _host_bias_struct(bias), int(chunk_b)))


def had_attention_host(Q, K, V, N=0, mode="float", seqlens=None, bias=None, alpha_q=None, alpha_k=None, out=None,
                       out_dtype=None, chunk_b=0, workspace=None, stream=None, synchronize=True):
    """had_attention on host tensors: the library copies chunks of the batch in,
    computes them and copies O out, overlapping the three (from pinned memory).

    Q, K, V, seqlens, the bias table and `out` are CPU tensors; `workspace` is a
    device uint8 tensor (allocated on the current device if None).  With
    synchronize=False the call returns once everything is enqueued on `stream`,
    and `out` is valid after that stream has been synchronized.
    """
    _check_host(Q, K, V, seqlens, out)
    B, H, n, d = Q.shape
    shp = make_shape(Q, seqlens)
    m = _MODES[mode]
    if out is None:
        out = torch.empty((B, H, n, d), dtype=out_dtype or V.dtype, pin_memory=Q.is_pinned())
    bs = _host_bias_struct(bias)
    need = lib().had_attention_host_workspace_size(ctypes.byref(shp), int(N), m, bs, int(chunk_b))
    if need == 0:
        _raise(HAD_ERR_INVALID, "had_attention_host_workspace_size")
    if workspace is not None:
        _check_dev(workspace)
    ws = _workspace(need, torch.device("cuda", torch.cuda.current_device()), workspace, stream)
    aq_keep, aq = _alpha(alpha_q, H)
    ak_keep, ak = _alpha(alpha_k, H)
    st = lib().had_attention_host(_ptr(Q), _ptr(K), _ptr(V), ctypes.byref(shp), bs, aq, ak, int(N), m, _ptr(out),
                                  _dtype_code(out), int(chunk_b), _ptr(ws), ws.numel(), _stream(stream))
    _raise(st, "had_attention_host")
    if synchronize:
        (stream or torch.cuda.current_stream()).synchronize()
    return out


def had_dense_reference_workspace_size(X, seqlens=None, bias=None) -> int:
    shp = make_shape(X, seqlens)
    return int(lib().had_dense_reference_workspace_size(ctypes.byref(shp), _bias_struct(bias)))


def had_dense_reference_mode(Q, K, V, N=0, seqlens=None, bias=None, out=None, out_dtype=None, workspace=None,
                             stream=None):
    """Standard dense attention on the unbinarized bf16 inputs (the library's comparison mode)."""
    _check_dev(Q, K, V, seqlens, out, workspace)
    B, H, n, d = Q.shape
    shp = make_shape(Q, seqlens)
    if out is None:
        out = torch.empty((B, H, n, d), dtype=out_dtype or V.dtype, device=Q.device)
    bs = _bias_struct(bias)
    need = int(lib().had_dense_reference_workspace_size(ctypes.byref(shp), bs))
    ws = _workspace(need, Q.device, workspace, stream) if need > 0 else None
    st = lib().had_dense_reference_mode(_ptr(Q), _ptr(K), _ptr(V), ctypes.byref(shp), bs, int(N),
                                        _ptr(out), _dtype_code(out), _ptr(ws), 0 if ws is None else ws.numel(),
                                        _stream(stream))
    _raise(st, "had_dense_reference_mode")
    return out


def had_scores_int(qbits, kbits, seqlens=None, d=64, stream=None):
    """Integer scores d - 2*popcount(q XOR k) [B,H,n,n] int32 through the library's tensor-core fragments."""
    _check_dev(qbits, kbits, seqlens)
    B, H, n, _ = qbits.shape
    shp = had_shape(B, H, n, d, HAD_BF16, None if seqlens is None else seqlens.data_ptr())
    S = torch.empty((B, H, n, n), dtype=torch.int32, device=qbits.device)
    st = lib().had_scores_int(_ptr(qbits), _ptr(kbits), ctypes.byref(shp), _ptr(S), _stream(stream))
    _raise(st, "had_scores_int")
    return S


def had_attention_scores(Q, K, seqlens=None, workspace=None, stream=None):
    """Integer scores [B,H,n,n] int32 as the fused kernel forms them in tensor memory."""
    _check_dev(Q, K, seqlens)
    B, H, n, d = Q.shape
    shp = make_shape(Q, seqlens)
    ws = _workspace(lib().had_attention_workspace_size(ctypes.byref(shp), 0, HAD_MODE_FLOAT, None), Q.device,
                    workspace, stream)
    S = torch.empty((B, H, n, n), dtype=torch.int32, device=Q.device)
    st = lib().had_attention_scores(_ptr(Q), _ptr(K), ctypes.byref(shp), _ptr(S), _ptr(ws), ws.numel(),
                                    _stream(stream))
    _raise(st, "had_attention_scores")
    return S


def had_debug_bounded_wait(max_cycles=0, force_expiry=False):
    """Test hook of the fused kernel's timeout path (see include/had.h)."""
    _raise(lib().had_debug_bounded_wait(int(max_cycles), 1 if force_expiry else 0), "had_debug_bounded_wait")


def had_topn_indices(Q, K, N, seqlens=None, bias=None, alpha_q=None, alpha_k=None, workspace=None, stream=None):
    """Kept key indices per query, ascending, -1 padded: [B,H,n,N] int32."""
    _check_dev(Q, K, seqlens)
    B, H, n, d = Q.shape
    shp = make_shape(Q, seqlens)
    bs = _bias_struct(bias)
    ws = _workspace(lib().had_attention_workspace_size(ctypes.byref(shp), int(N), HAD_MODE_FLOAT, bs), Q.device,
                    workspace, stream)
    idx = torch.empty((B, H, n, N), dtype=torch.int32, device=Q.device)
    aq_keep, aq = _alpha(alpha_q, H)
    ak_keep, ak = _alpha(alpha_k, H)
    st = lib().had_topn_indices(_ptr(Q), _ptr(K), ctypes.byref(shp), bs, aq, ak, int(N), _ptr(idx), _ptr(ws),
                                ws.numel(), _stream(stream))
    _raise(st, "had_topn_indices")
    return idx


def had_attention_codes_u8(Q, K, V, row_begin, row_end, N=0, seqlens=None, bias=None, alpha_q=None, alpha_k=None,
                           workspace=None, stream=None):
    """uint8 attention codes floor(255 p + 0.5) of rows [row_begin, row_end): [B,H,rows,n] uint8."""
    _check_dev(Q, K, V, seqlens)
    B, H, n, d = Q.shape
    shp = make_shape(Q, seqlens)
    bs = _bias_struct(bias)
    ws = _workspace(lib().had_attention_workspace_size(ctypes.byref(shp), int(N), HAD_MODE_U8I8, bs), Q.device,
                    workspace, stream)
    A = torch.empty((B, H, row_end - row_begin, n), dtype=torch.uint8, device=Q.device)
    aq_keep, aq = _alpha(alpha_q, H)
    ak_keep, ak = _alpha(alpha_k, H)
    st = lib().had_attention_codes_u8(_ptr(Q), _ptr(K), _ptr(V), ctypes.byref(shp), bs, aq, ak, int(N),
                                      int(row_begin), int(row_end), _ptr(A), _ptr(ws), ws.numel(), _stream(stream))
    _raise(st, "had_attention_codes_u8")
    return A


def _quantize(fn, mode, V, seqlens, workspace, stream):
    _check_dev(V, seqlens)
    B, H, n, d = V.shape
    shp = make_shape(V, seqlens)
    ws = _workspace(lib().had_attention_workspace_size(ctypes.byref(shp), 0, mode, None), V.device,
                    workspace, stream)
    Vq = torch.empty((B, H, n, d), dtype=torch.int8, device=V.device)
    sc = torch.empty((B, H, d), dtype=torch.float32, device=V.device)
    st = getattr(lib(), fn)(_ptr(V), ctypes.byref(shp), _ptr(Vq), _ptr(sc), _ptr(ws), ws.numel(), _stream(stream))
    _raise(st, fn)
    return Vq, sc


def had_quantize_v(V, seqlens=None, workspace=None, stream=None):
    """Per-channel int8 V [B,H,n,d] and its fp32 scales [B,H,d]."""
    return _quantize("had_quantize_v", HAD_MODE_U8I8, V, seqlens, workspace, stream)


def had_quantize_v4(V, seqlens=None, workspace=None, stream=None):
    """Per-channel 4-bit V (codes in [-7, 7], one per int8) [B,H,n,d] and its fp32 scales [B,H,d]."""
    return _quantize("had_quantize_v4", HAD_MODE_U8I4, V, seqlens, workspace, stream)


def had_qkv_attention(X, W, H, N=0, mode="float", seqlens=None, bias=None, alpha_q=None, alpha_k=None, out=None,
                      out_dtype=None, workspace=None, stream=None, return_v=False):
    """The projection before the path (Q|K|V = X W^T, W in a linear layer's [3*H*64, Dm]
    layout), with Q and K binarized in its epilogue, then the fused attention.

    X: bf16 [B, n, Dm]; W: bf16 [3*H*64, Dm].  Returns O [B, H, 64-channel heads] as
    [B, H, n, 64] (and V, the bf16 projection the attention read, with return_v)."""
    _check_dev(X, W, seqlens, out, workspace)
    if X.dtype != torch.bfloat16 or W.dtype != torch.bfloat16:
        raise TypeError("X and W must be bfloat16")
    B, n, Dm = X.shape
    d = 64
    if seqlens is not None and seqlens.dtype != torch.int32:
        raise TypeError("seqlens must be int32")
    shp = had_shape(B, H, n, d, HAD_BF16, None if seqlens is None else seqlens.data_ptr())
    m = _MODES[mode]
    bs = _bias_struct(bias)
    V = torch.empty((B, H, n, d), dtype=torch.bfloat16, device=X.device)
    if out is None:
        out = torch.empty((B, H, n, d), dtype=out_dtype or torch.bfloat16, device=X.device)
    need = lib().had_qkv_workspace_size(ctypes.byref(shp), int(Dm), int(N), m, bs)
    if need == 0:
        _raise(HAD_ERR_UNSUPPORTED, "had_qkv_workspace_size")
    ws = _workspace(need, X.device, workspace, stream)
    st = lib().had_qkv_prepare(_ptr(X), _ptr(W), ctypes.byref(shp), int(Dm), bs, int(N), m, _ptr(V), _ptr(ws),
                               ws.numel(), _stream(stream))
    _raise(st, "had_qkv_prepare")
    aq_keep, aq = _alpha(alpha_q, H)
    ak_keep, ak = _alpha(alpha_k, H)
    st = lib().had_attention_prepared(_ptr(V), ctypes.byref(shp), bs, aq, ak, int(N), m, _ptr(out), _dtype_code(out),
                                      _ptr(ws), ws.numel(), _stream(stream))
    _raise(st, "had_attention_prepared")
    return (out, V) if return_v else out


def had_qkv_workspace(X, H, N=0, mode="float", seqlens=None, bias=None):
    """A workspace of the size had_qkv_attention needs (uint8 tensor on X's device).  It
    starts with the attention workspace: Q's sign bits as [B, H, n, 2] uint32 words at
    offset 0, then K's +-1 rows [B, H, n_pad, 64] at the next 256-byte boundary."""
    B, n, Dm = X.shape
    shp = had_shape(B, H, n, 64, HAD_BF16, None if seqlens is None else seqlens.data_ptr())
    need = lib().had_qkv_workspace_size(ctypes.byref(shp), int(Dm), int(N), _MODES[mode], _bias_struct(bias))
    if need == 0:
        _raise(HAD_ERR_UNSUPPORTED, "had_qkv_workspace_size")
    return torch.empty(need, dtype=torch.uint8, device=X.device)


def had_get_device_status() -> int:
    """Synchronize, read and clear the device status word (HAD_OK, HAD_ERR_DEVICE or HAD_ERR_TIMEOUT)."""
    return int(lib().had_get_device_status())


def had_probe_mma_rate(kind="i8", iters=200000):
    """Tensor-pipe rate of tcgen05.mma on this GPU: (10^12 ops/s, elapsed ms).

    kind "i8": kind::i8 (the +-1 score contraction); "bf16": kind::f16 with bf16
    operands.  Synchronizes the device."""
    k = {"i8": 0, "bf16": 1}[kind]
    tops, ms = ctypes.c_double(0.0), ctypes.c_double(0.0)
    _raise(lib().had_probe_mma_rate(k, int(iters), ctypes.byref(tops), ctypes.byref(ms)), "had_probe_mma_rate")
    return tops.value, ms.value


def had_version() -> int:
    return int(lib().had_version())

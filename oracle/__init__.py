"""CPU oracle for binarized-QK top-N attention (test infrastructure only).

The oracle is a plain C implementation (``had_oracle.c``) of what the method
computes, in fp64, written from the definitions in "Hamming Attention
Distillation" (HAD; top-N sparsification, binarized keys and queries) and
"BinaryAttention: One-Bit QK-Attention" (§2.1-§2.4: centering, sign, XNOR +
popcount, scaling 1/sqrt(d) + bias, uint8 A x int8 V).  This module only loads
it and marshals numpy arrays through ctypes.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  It shares no code with the CUDA library.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "had_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "libhad_oracle.so")

MODE_FLOAT = 0
MODE_U8I8 = 1
MODE_U8I4 = 2


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FP contraction, OpenMP)."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    cmd = ["gcc", "-std=c99", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-o", _LIB + ".tmp", _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        path = build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I = ctypes.c_int
        I64 = ctypes.c_int64
        L.hado_num_threads.restype = I
        L.hado_set_num_threads.argtypes = [I]
        L.hado_channel_mean.argtypes = [P, I, I, I, I, P, P]
        L.hado_sign_pack.argtypes = [P, P, I, I, I, I, P, P]
        L.hado_binary_scores.argtypes = [P, P, I, I, I, I, P, P]
        L.hado_v_quant.argtypes = [P, I, I, I, I, P, P, P]
        L.hado_v_quant4.argtypes = [P, I, I, I, I, P, P, P]
        L.hado_qkv_project.argtypes = [P, P, I, I, I, I, I, P, P, P, P, P, P, P, P]
        L.hado_logits.argtypes = [P, P, I, I, I, I, P, P, I, I, I, P, P, P]
        L.hado_attention.argtypes = [P, P, P, I, I, I, I, P, P, I, I, I, P, P, I, I, P, I64, P, P, P, P, P, P,
                                     P, P, P, P]
        L.hado_dense_attention.argtypes = [P, P, P, I, I, I, I, P, P, I, I, I, I, P, I64, P]
        for f in (L.hado_channel_mean, L.hado_sign_pack, L.hado_binary_scores, L.hado_v_quant, L.hado_v_quant4,
                  L.hado_logits, L.hado_qkv_project,
                  L.hado_attention, L.hado_dense_attention):
            f.restype = I
        _lib = L
    return _lib


def _p(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _seq(seqlens):
    return None if seqlens is None else np.ascontiguousarray(seqlens, dtype=np.int32)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} failed with code {rc}")


def num_threads() -> int:
    return lib().hado_num_threads()


def set_num_threads(t: int) -> None:
    lib().hado_set_num_threads(int(t))


def channel_mean(X, seqlens=None):
    """mu[b,h,c]: fp64 token-order sum over valid tokens, / L, rounded to fp32."""
    X = _f32(X)
    B, H, n, d = X.shape
    s = _seq(seqlens)
    mu = np.zeros((B, H, d), np.float32)
    _check(lib().hado_channel_mean(_p(X), B, H, n, d, _p(s), _p(mu)), "channel_mean")
    return mu


def sign_pack(X, mu, seqlens=None):
    """Packed sign bits [B,H,n,d/32] uint32: bit j of word w <=> X[..., 32w+j] < mu."""
    X = _f32(X)
    mu = _f32(mu)
    B, H, n, d = X.shape
    s = _seq(seqlens)
    bits = np.zeros((B, H, n, d // 32), np.uint32)
    _check(lib().hado_sign_pack(_p(X), _p(mu), B, H, n, d, _p(s), _p(bits)), "sign_pack")
    return bits


def binary_scores(qbits, kbits, d, seqlens=None):
    """Integer scores s = d - 2*popcount(q XOR k), [B,H,n,n] int32 (0 off the valid square)."""
    qbits = np.ascontiguousarray(qbits, np.uint32)
    kbits = np.ascontiguousarray(kbits, np.uint32)
    B, H, n, _ = qbits.shape
    s = _seq(seqlens)
    S = np.zeros((B, H, n, n), np.int32)
    _check(lib().hado_binary_scores(_p(qbits), _p(kbits), B, H, n, d, _p(s), _p(S)), "binary_scores")
    return S


def v_quant(V, seqlens=None, bits=8):
    """Per-channel symmetric int8 V (bits=8: [-127, 127], scale absmax/127) or 4-bit
    V (bits=4: [-7, 7], scale absmax/7): (Vq [B,H,n,d] int8, scale [B,H,d] fp32)."""
    V = _f32(V)
    B, H, n, d = V.shape
    s = _seq(seqlens)
    Vq = np.zeros((B, H, n, d), np.int8)
    sc = np.zeros((B, H, d), np.float32)
    fn = lib().hado_v_quant if bits == 8 else lib().hado_v_quant4
    if bits not in (4, 8):
        raise ValueError("bits must be 8 or 4")
    _check(fn(_p(V), B, H, n, d, _p(s), _p(Vq), _p(sc)), "v_quant")
    return Vq, sc


def qkv_project(X, W, H, d, seqlens=None):
    """The projection that precedes the path and its binarization: X [B, n, Dm],
    W [3*H*d, Dm] -> (Q, K, V) fp64 [B, H, n, d], mu_q, mu_k fp32 [B, H, d],
    qbits, kbits uint32 [B, H, n, d/32]."""
    X, W = _f32(X), _f32(W)
    B, n, Dm = X.shape
    if W.shape != (3 * H * d, Dm):
        raise ValueError("W must be [3*H*d, Dm]")
    s = _seq(seqlens)
    Q, K, V = (np.zeros((B, H, n, d), np.float64) for _ in range(3))
    mq, mk = np.zeros((B, H, d), np.float32), np.zeros((B, H, d), np.float32)
    qb, kb = np.zeros((B, H, n, d // 32), np.uint32), np.zeros((B, H, n, d // 32), np.uint32)
    _check(lib().hado_qkv_project(_p(X), _p(W), B, n, Dm, H, d, _p(s), _p(Q), _p(K), _p(V), _p(mq), _p(mk),
                                  _p(qb), _p(kb)), "qkv_project")
    return Q, K, V, mq, mk, qb, kb


@dataclass
class RelPosBias:
    """Per-head relative-position table [H, 2gh-1, 2gw-1] over a gh x gw patch grid after `prefix` tokens."""
    table: np.ndarray
    gh: int
    gw: int
    prefix: int


@dataclass
class DenseBias:
    """Per-head dense bias matrix [H, n, n]: b_ij = table[h, i, j] (one learnable value per query-key pair)."""
    table: np.ndarray


def _bias_args(bias):
    if bias is None:
        return None, 0, 0, 0
    if isinstance(bias, DenseBias):
        return _f32(bias.table), 0, 0, 0  # gh == gw == 0 selects the dense matrix
    return _f32(bias.table), int(bias.gh), int(bias.gw), int(bias.prefix)


def logits(qbits, kbits, d, seqlens=None, bias=None, alpha_q=None, alpha_k=None):
    """Logit matrix l = fmaf(s, c, b) [B,H,n,n] fp32, NaN off the valid square."""
    qbits = np.ascontiguousarray(qbits, np.uint32)
    kbits = np.ascontiguousarray(kbits, np.uint32)
    B, H, n, _ = qbits.shape
    s = _seq(seqlens)
    t, gh, gw, pf = _bias_args(bias)
    aq = None if alpha_q is None else _f32(alpha_q)
    ak = None if alpha_k is None else _f32(alpha_k)
    out = np.zeros((B, H, n, n), np.float32)
    _check(lib().hado_logits(_p(qbits), _p(kbits), B, H, n, d, _p(s), _p(t), gh, gw, pf, _p(aq), _p(ak), _p(out)),
           "logits")
    return out


@dataclass
class OracleResult:
    O: np.ndarray                 # [rows, d] fp64 (or [B,H,n,d] when rows is None)
    idx: np.ndarray | None        # [rows, N] int32 kept indices ascending, -1 padded
    Aq: np.ndarray | None         # [rows, n] uint8 codes
    P: np.ndarray | None          # [rows, n] fp64 probabilities
    mu_q: np.ndarray
    mu_k: np.ndarray
    qbits: np.ndarray
    kbits: np.ndarray
    Vq: np.ndarray
    vscale: np.ndarray


def attention(Q, K, V, N=0, mode=MODE_FLOAT, seqlens=None, bias=None, alpha_q=None, alpha_k=None, rows=None,
              want_idx=False, want_codes=False, want_probs=False):
    """Full forward pass.  rows: optional flat row ids ((b*H + h)*n + i)."""
    Q, K, V = _f32(Q), _f32(K), _f32(V)
    B, H, n, d = Q.shape
    s = _seq(seqlens)
    t, gh, gw, pf = _bias_args(bias)
    aq = None if alpha_q is None else _f32(alpha_q)
    ak = None if alpha_k is None else _f32(alpha_k)
    r = None if rows is None else np.ascontiguousarray(rows, np.int64)
    nr = B * H * n if r is None else int(r.shape[0])
    O = np.zeros((nr, d), np.float64)
    idx = np.zeros((nr, N), np.int32) if (want_idx and N > 0) else None
    Aq = np.zeros((nr, n), np.uint8) if want_codes else None
    P = np.zeros((nr, n), np.float64) if want_probs else None
    mu_q = np.zeros((B, H, d), np.float32)
    mu_k = np.zeros((B, H, d), np.float32)
    qb = np.zeros((B, H, n, d // 32), np.uint32)
    kb = np.zeros((B, H, n, d // 32), np.uint32)
    Vq = np.zeros((B, H, n, d), np.int8)
    vs = np.zeros((B, H, d), np.float32)
    rc = lib().hado_attention(_p(Q), _p(K), _p(V), B, H, n, d, _p(s), _p(t), gh, gw, pf, _p(aq), _p(ak), int(N),
                              int(mode), _p(r), nr if r is not None else 0, _p(O), _p(idx), _p(Aq), _p(P),
                              _p(mu_q), _p(mu_k), _p(qb), _p(kb), _p(Vq), _p(vs))
    _check(rc, "attention")
    if r is None:
        O = O.reshape(B, H, n, d)
    return OracleResult(O, idx, Aq, P, mu_q, mu_k, qb, kb, Vq, vs)


def dense_attention(Q, K, V, N=0, seqlens=None, bias=None, rows=None):
    """Standard (unbinarized) attention in fp64 on the given fp32 values."""
    Q, K, V = _f32(Q), _f32(K), _f32(V)
    B, H, n, d = Q.shape
    s = _seq(seqlens)
    t, gh, gw, pf = _bias_args(bias)
    r = None if rows is None else np.ascontiguousarray(rows, np.int64)
    nr = B * H * n if r is None else int(r.shape[0])
    O = np.zeros((nr, d), np.float64)
    rc = lib().hado_dense_attention(_p(Q), _p(K), _p(V), B, H, n, d, _p(s), _p(t), gh, gw, pf, int(N), _p(r),
                                    nr if r is not None else 0, _p(O))
    _check(rc, "dense_attention")
    if r is None:
        O = O.reshape(B, H, n, d)
    return O

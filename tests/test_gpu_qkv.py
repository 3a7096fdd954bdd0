"""GPU parity of the projection that precedes the path, binarized in its epilogue
(had_qkv_prepare): Q|K|V = X W^T on the tensor cores, the means of Q and K from
X's token means (mean_i(X_i) W^T), Q's sign bits and K's +-1 rows written into
the attention workspace, V in bf16; then the fused attention on that workspace.

Bars:
- sign bits of Q and K equal the oracle's (fp64 projection, fp64 means) on
  every entry whose distance to its mean exceeds the fp32 accumulation bound
  (2^-20 * sum_k |x_k w_k| + 2^-22 |mu|), where either sign is a correct result
  of an fp32 projection; those entries are a small fraction and are reported;
- K rows past L (up to n_pad) are +1; bits of tokens past L are 0;
- V within bf16 rounding of the fp64 projection (plus the accumulation bound);
- the attention that follows equals the oracle's attention on +-1 tensors that
  carry exactly the GPU's bits and its bf16 V: kept sets bit-exact, O within the
  usual bars.
"""
import numpy as np
import pytest

import workloads

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import binarized_qk_sparse_b200 as had  # noqa: E402


def _inputs(B, n, Dm, H, seed, scale=None):
    rng = np.random.default_rng(seed)
    X = workloads.bf16_round(rng.standard_normal((B, n, Dm)).astype(np.float32))
    W = workloads.bf16_round((rng.standard_normal((3 * H * 64, Dm)) * (scale or Dm ** -0.5)).astype(np.float32))
    return X, W


def _unpack(words, d=64):
    """[..., d/32] uint32 -> [..., d] bool (bit j of word w = channel 32w + j)."""
    w = words.astype(np.uint64)[..., None] >> np.arange(32, dtype=np.uint64)
    return (w & 1).astype(bool).reshape(words.shape[:-1] + (d,))


def _read_workspace(ws, B, H, n):
    """Q's sign bits and K's +-1 rows from the start of the attention workspace."""
    n_pad = (n + 63) // 64 * 64
    qbytes = B * H * n * 8
    qb = ws[:qbytes].view(torch.int32).cpu().numpy().view(np.uint32).reshape(B, H, n, 2)
    k0 = (qbytes + 255) // 256 * 256
    kpm = ws[k0:k0 + B * H * n_pad * 64].cpu().numpy().reshape(B, H, n_pad, 64)
    return qb, kpm


def _ambiguous(P, mu, X, W, H, t):
    """Entries whose sign an fp32 projection may legitimately take either way."""
    Wt = np.abs(W.astype(np.float64)).reshape(3, H, 64, -1)[t]  # [H, 64, Dm]
    mag = np.einsum("bik,hck->bhic", np.abs(X.astype(np.float64)), Wt, optimize=True)
    tol = 2.0 ** -20 * mag + 2.0 ** -22 * np.abs(mu.astype(np.float64))[:, :, None, :]
    return np.abs(P - mu.astype(np.float64)[:, :, None, :]) <= tol


def _check_bits(got, ref_bits, P, mu, X, W, H, t, L):
    g = _unpack(got)
    r = _unpack(ref_bits)
    amb = _ambiguous(P, mu, X, W, H, t)
    for b in range(len(L)):
        assert not g[b, :, L[b]:].any(), "tokens past L carry sign bits"
        amb[b, :, L[b]:] = False
    bad = (g != r) & ~amb
    assert not bad.any(), f"{bad.sum()} sign bits differ outside the rounding band"
    assert amb.mean() < 1e-3, amb.mean()


@pytest.mark.parametrize("B,n,Dm,H,seqlens,N,mode", [
    (2, 197, 256, 2, [197, 120], 0, "u8i8"),     # DeiT-like rows, ragged, dense uint8
    (1, 300, 192, 3, None, 30, "float"),         # 3 heads, top-30 float (n not a multiple of 128)
    (2, 70, 64, 1, [70, 9], 0, "float"),         # one panel, a short second sequence
    # 720 CTAs of 128 tokens x 4 heads (several waves, two CTAs per SM), ragged lengths
    (40, 197, 256, 12, list(range(197, 157, -1)), 0, "u8i8"),
])
def test_qkv_bits_rows_and_v(oracle_mod, B, n, Dm, H, seqlens, N, mode):
    X, W = _inputs(B, n, Dm, H, seed=100 + n)
    sl = None if seqlens is None else np.array(seqlens, np.int32)
    L = np.full(B, n) if sl is None else sl
    Xd = torch.from_numpy(X).to(torch.bfloat16).cuda()
    Wd = torch.from_numpy(W).to(torch.bfloat16).cuda()
    sd = None if sl is None else torch.from_numpy(sl).cuda()
    ws = had.had_qkv_workspace(Xd, H, N, mode, sd)
    O, V = had.had_qkv_attention(Xd, Wd, H, N=N, mode=mode, seqlens=sd, workspace=ws, return_v=True)
    torch.cuda.synchronize()
    assert had.had_get_device_status() == had.HAD_OK
    Q64, K64, V64, mq, mk, qb_ref, kb_ref = oracle_mod.qkv_project(X, W, H, 64, sl)
    qb, kpm = _read_workspace(ws, B, H, n)
    _check_bits(qb, qb_ref, Q64, mq, X, W, H, 0, L)
    # K: bit 7 of a +-1 byte is its sign (int8 0xFF or e4m3 0xB8 for -1)
    n_pad = kpm.shape[2]
    ksign = (kpm.view(np.uint8) >> 7).astype(bool)
    kwords = np.zeros((B, H, n, 2), np.uint32)
    for w in range(2):
        kwords[..., w] = (ksign[:, :, :n, 32 * w:32 * w + 32].astype(np.uint64)
                          << np.arange(32, dtype=np.uint64)).sum(axis=-1).astype(np.uint32)
    _check_bits(kwords, kb_ref, K64, mk, X, W, H, 1, L)
    for b in range(B):
        assert not ksign[b, :, L[b]:n_pad].any(), "K rows past L must be +1"
    # V: bf16 of the fp64 projection, within bf16 rounding and the accumulation bound
    Vg = V.float().cpu().numpy()
    mag = np.einsum("bik,hck->bhic", np.abs(X.astype(np.float64)),
                    np.abs(W.astype(np.float64)).reshape(3, H, 64, -1)[2], optimize=True)
    assert np.all(np.abs(Vg - V64) <= np.abs(V64) * 2.0 ** -8 + 2.0 ** -20 * mag + 1e-30)


@pytest.mark.parametrize("B,H,N,mode,with_bias", [(2, 2, 0, "u8i8", True), (2, 2, 0, "float", False),
                                                  (2, 2, 40, "float", True), (2, 2, 40, "u8i4", False),
                                                  (24, 12, 0, "u8i8", True)])  # 432 CTAs, V absmax over many
def test_qkv_attention_end_to_end(oracle_mod, B, H, N, mode, with_bias):
    """The attention on the fused workspace against the oracle's attention on +-1
    tensors that carry exactly the GPU's sign bits (their own means keep those signs)
    and the GPU's bf16 V: kept sets bit-exact, O within the usual bars."""
    n, Dm = 197, 256
    X, W = _inputs(B, n, Dm, H, seed=77)
    sl = np.array([197, 150] + [197 - 3 * i for i in range(B - 2)], np.int32)
    Xd = torch.from_numpy(X).to(torch.bfloat16).cuda()
    Wd = torch.from_numpy(W).to(torch.bfloat16).cuda()
    sd = torch.from_numpy(sl).cuda()
    bias = ob = None
    if with_bias:
        table = (np.random.default_rng(78).standard_normal((H, 27, 27)) * 0.1).astype(np.float32)
        bias = had.RelPosBias(torch.from_numpy(table).cuda(), 14, 14, 1)
        ob = oracle_mod.RelPosBias(table, 14, 14, 1)
    ws = had.had_qkv_workspace(Xd, H, N, mode, sd, bias)
    O, V = had.had_qkv_attention(Xd, Wd, H, N=N, mode=mode, seqlens=sd, bias=bias, workspace=ws,
                                 out_dtype=torch.float32, return_v=True)
    torch.cuda.synchronize()
    assert had.had_get_device_status() == had.HAD_OK
    qb, kpm = _read_workspace(ws, B, H, n)
    Qs = np.where(_unpack(qb), -1.0, 1.0).astype(np.float32)
    Ks = np.where((kpm[:, :, :n].view(np.uint8) >> 7).astype(bool), -1.0, 1.0).astype(np.float32)
    for b in range(B):  # padding tokens: any values (the oracle ignores them)
        Qs[b, :, sl[b]:] = 0.0
        Ks[b, :, sl[b]:] = 0.0
    Vg = V.float().cpu().numpy()
    m = {"float": 0, "u8i8": 1, "u8i4": 2}[mode]
    ref = oracle_mod.attention(Qs, Ks, Vg, N=N, mode=m, seqlens=sl, bias=ob, want_idx=N > 0)
    np.testing.assert_array_equal(ref.qbits, qb)  # the +-1 tensors keep the GPU's signs
    Og = O.cpu().numpy()
    tol = 1e-2 * float(np.max(np.abs(Vg))) * (1.0 if m == 0 else 1.5)
    assert np.max(np.abs(Og - ref.O)) <= tol
    if N > 0:
        idx = had.had_topn_indices(torch.from_numpy(Qs).cuda(), torch.from_numpy(Ks).cuda(), N, sd, bias)
        np.testing.assert_array_equal(idx.cpu().numpy(), ref.idx.reshape(B, H, n, N))
    # the separate path on the same signs and V (statistics pass for V's scales, packing) gives the same O
    # bit for bit: the epilogue's V absmax and the workspace it leaves are those of the prepare stage
    Qd = torch.from_numpy(Qs).to(torch.bfloat16).cuda()
    Kd = torch.from_numpy(Ks).to(torch.bfloat16).cuda()
    O2 = had.had_attention(Qd, Kd, V, N=N, mode=mode, seqlens=sd, bias=bias, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(O, O2)

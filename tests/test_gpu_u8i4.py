"""GPU parity of the 4-bit V mode (HAD_MODE_U8I4): uint8 attention codes times
per-channel 4-bit V, the int8 scheme of BinaryAttention §2.4 taken to 4 bits (its
conclusion names lower-bit V without defining it: codes in [-7, 7], scale
absmax / 7, round half to even).

Bars: the 4-bit codes and scales bit-exact against the oracle; O against the
oracle's mode 2 within the uint8 bars (max-abs 1e-2 * max|V| for bf16 V, plus
max|V| / 255 where a code may sit at a rounding tie of the top-N kept set); the
prepared two-stage call and the host entry point bit-identical to had_attention.
Workloads: DeiT (dense, relative-position bias), BERT (top-30, ragged lengths),
T5-1024 (top-120), the full-size stress workload on sampled rows (dense and
top-1920 with its 255x255 bias), bias grids whose rows hold 64k patches, edge
lengths, and head dim 128.
"""
import ctypes

import numpy as np
import pytest

import workloads

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import binarized_qk_sparse_b200 as had  # noqa: E402

MODE = 2  # the oracle's 4-bit V mode


def _dev(w, x):
    t = torch.from_numpy(np.ascontiguousarray(x))
    return (t.to(torch.bfloat16) if w.dtype == "bf16" else t).cuda()


def _inputs(w):
    Q, K, V = _dev(w, w.Q), _dev(w, w.K), _dev(w, w.V)
    seq = None if w.seqlens is None else torch.from_numpy(w.seqlens).cuda()
    bias = None
    if w.bias is not None:
        bias = had.RelPosBias(torch.from_numpy(w.bias.table).cuda(), w.bias.gh, w.bias.gw, w.bias.prefix)
    return Q, K, V, seq, bias


def _obias(oracle_mod, w):
    return None if w.bias is None else oracle_mod.RelPosBias(w.bias.table, w.bias.gh, w.bias.gw, w.bias.prefix)


def _tol(w):
    return (1e-3 if w.dtype == "f32" else 1e-2) * float(np.max(np.abs(w.V)))


def _tie(w):
    return float(np.max(np.abs(w.V))) / 255


def _flat(t):
    return t.reshape(-1, t.shape[-1])


def _rows(w, per_head, seed):
    rng = np.random.default_rng(seed)
    out = []
    for bh in range(w.B * w.H):
        L = w.n if w.seqlens is None else int(w.seqlens[bh // w.H])
        out.extend(bh * w.n + int(i) for i in sorted(rng.choice(L, size=min(per_head, L), replace=False)))
    return np.array(out, np.int64)


_cache = {}


def _workload(name):
    if name not in _cache:
        _cache[name] = workloads.by_name(name)
    return _cache[name]


def _sub(w, B):
    return workloads.Workload(w.name + f"_sub{B}", B, w.H, w.n, w.d, w.dtype, w.Q[:B], w.K[:B], w.V[:B],
                              None if w.seqlens is None else w.seqlens[:B], w.bias, w.passes, w.seed, w.recipe)


# ----------------------------------------------------------------------------- the quantizer

@pytest.mark.parametrize("name", ["tiny", "deit", "bert", "t5_1024"])
def test_v4_codes_and_scales_bit_exact(oracle_mod, name):
    w = _workload(name)
    _, _, V, seq, _ = _inputs(w)
    Vq, sc = had.had_quantize_v4(V, seq)
    Vq_o, sc_o = oracle_mod.v_quant(w.V, w.seqlens, bits=4)
    np.testing.assert_array_equal(sc.cpu().numpy(), sc_o)
    np.testing.assert_array_equal(Vq.cpu().numpy(), Vq_o)
    assert int(Vq.abs().max()) <= 7


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("seqlens", [None, [100, 37, 128]])
def test_v4_half_integer_ties_round_to_even(oracle_mod, d, seqlens):
    """Channels whose absmax is 7 * 2^e have scale 2^e, so V / scale is exact and
    values at k + 1/2 are genuine ties: both sides round them to the even code.
    128 tokens of bf16 (the short-head prep) and of fp32 with 600 tokens (the
    chunked prep)."""
    for n, dtype in ((128, "bf16"), (600, "f32")):
        rng = np.random.default_rng(7 + d + n)
        B = 1 if seqlens is None else len(seqlens)
        e = rng.integers(-3, 4, size=(B, 2, 1, d)).astype(np.float32)
        half = rng.integers(-14, 15, size=(B, 2, n, d)).astype(np.float32) / 2  # multiples of 1/2 in [-7, 7]
        V = np.ldexp(half, e.astype(np.int32)).astype(np.float32)
        V[:, :, 0, :] = np.ldexp(7.0, e[:, :, 0, :].astype(np.int32))  # absmax 7 * 2^e on the first (valid) token
        sl = None if seqlens is None else np.array([min(s, n) for s in seqlens], np.int32)
        Vd = torch.from_numpy(V).to(torch.bfloat16 if dtype == "bf16" else torch.float32).cuda()
        sd = None if sl is None else torch.from_numpy(sl).cuda()
        Vq, sc = had.had_quantize_v4(Vd, sd)
        Vq_o, sc_o = oracle_mod.v_quant(V, sl, bits=4)
        np.testing.assert_array_equal(sc.cpu().numpy(), sc_o)
        np.testing.assert_array_equal(Vq.cpu().numpy(), Vq_o)
        # the ties are there and went to even codes
        assert np.any(np.abs(Vq_o) % 2 == 0) and np.any(half % 1 != 0)


def test_v4_codes_stress_full_size(oracle_mod):
    w = _workload("stress")
    _, _, V, seq, _ = _inputs(w)
    Vq, sc = had.had_quantize_v4(V, seq)
    Vq_o, sc_o = oracle_mod.v_quant(w.V, w.seqlens, bits=4)
    np.testing.assert_array_equal(sc.cpu().numpy(), sc_o)
    np.testing.assert_array_equal(Vq.cpu().numpy(), Vq_o)


# ----------------------------------------------------------------------------- the fused kernel

@pytest.mark.parametrize("name", ["deit", "t5_1024", "stress", "deit_d128"])
def test_u8i4_top1_returns_the_kept_keys_codes(oracle_mod, name):
    """With N = 1 the kept key has p = 1, so A = 255 and O[c] = V4[j, c] * scale[c]
    up to fp32 rounding: every sampled row must give back, channel by channel, the
    oracle's 4-bit code of the key the oracle keeps.  This checks the codes the
    attention path prepares (the short-head and chunked prep kernels) and the
    order of the two keys in each packed byte, bit for bit."""
    w = _workload(name)
    if w.B > 4:
        w = _sub(w, 4)
    Q, K, V, seq, bias = _inputs(w)
    rows = _rows(w, 16 if w.n > 4096 else 64, 37)
    rows_t = torch.from_numpy(rows).cuda()
    O = _flat(had.had_attention(Q, K, V, N=1, mode="u8i4", seqlens=seq, bias=bias, out_dtype=torch.float32))
    O = O[rows_t].cpu().numpy()
    ref = oracle_mod.attention(w.Q, w.K, w.V, N=1, mode=MODE, seqlens=w.seqlens, bias=_obias(oracle_mod, w),
                               rows=rows, want_idx=True)
    bh = rows // w.n
    j = ref.idx[:, 0]
    Vq = ref.Vq.reshape(w.B * w.H, w.n, w.d)[bh, j]
    sc = ref.vscale.reshape(w.B * w.H, w.d)[bh]
    np.testing.assert_array_equal(np.rint(O / sc).astype(np.int32), Vq.astype(np.int32))


def test_u8i4_deit_dense_with_bias(oracle_mod):
    w = _workload("deit")
    Q, K, V, seq, bias = _inputs(w)
    O = had.had_attention(Q, K, V, N=0, mode="u8i4", seqlens=seq, bias=bias).float().cpu().numpy()
    ref = oracle_mod.attention(w.Q, w.K, w.V, N=0, mode=MODE, seqlens=w.seqlens, bias=_obias(oracle_mod, w))
    assert np.max(np.abs(O - ref.O)) <= _tol(w)
    # 4-bit V is coarser than int8 V: the two outputs differ, by about the 4-bit step
    O8 = had.had_attention(Q, K, V, N=0, mode="u8i8", seqlens=seq, bias=bias).float().cpu().numpy()
    assert np.max(np.abs(O - O8)) > _tie(w)


@pytest.mark.parametrize("name,N", [("bert", 30), ("t5_1024", 120), ("t5_256", 30)])
def test_u8i4_topn_without_bias(oracle_mod, name, N):
    w = _workload(name)
    if w.B > 4:
        w = _sub(w, 4)
    Q, K, V, seq, bias = _inputs(w)
    O = had.had_attention(Q, K, V, N=N, mode="u8i4", seqlens=seq).float().cpu().numpy()
    ref = oracle_mod.attention(w.Q, w.K, w.V, N=N, mode=MODE, seqlens=w.seqlens)
    assert np.max(np.abs(O - ref.O)) <= _tol(w)


def test_u8i4_stress_full_size(oracle_mod):
    w = _workload("stress")
    Q, K, V, seq, bias = _inputs(w)
    ob = _obias(oracle_mod, w)
    rows = _rows(w, 12, 19)
    rows_t = torch.from_numpy(rows).cuda()
    for N in (0, 1920):
        O = _flat(had.had_attention(Q, K, V, N=N, mode="u8i4", bias=bias))[rows_t].float().cpu().numpy()
        ref = oracle_mod.attention(w.Q, w.K, w.V, N=N, mode=MODE, bias=ob, rows=rows)
        assert np.max(np.abs(O - ref.O)) <= _tol(w) + (_tie(w) if N else 0.0), N


@pytest.mark.parametrize("gh,gw,seqlens", [(4, 64, None), (8, 128, [1024, 700])])
def test_u8i4_topn_bias_row_windows(oracle_mod, gh, gw, seqlens):
    B = 1 if seqlens is None else len(seqlens)
    w = workloads.grid(B, 2, gh, gw, 0, seqlens, seed=33)
    Q, K, V, seq, bias = _inputs(w)
    rows = _rows(w, 40, 23)
    rows_t = torch.from_numpy(rows).cuda()
    N = max(1, w.n // 8)
    ob = _obias(oracle_mod, w)
    for Nk in (N, 0):
        O = _flat(had.had_attention(Q, K, V, N=Nk, mode="u8i4", seqlens=seq, bias=bias))[rows_t].float().cpu().numpy()
        ref = oracle_mod.attention(w.Q, w.K, w.V, N=Nk, mode=MODE, seqlens=w.seqlens, bias=ob, rows=rows)
        assert np.max(np.abs(O - ref.O)) <= _tol(w) + _tie(w), Nk


def _small(seed, B=3, H=2, n=70):
    rng = np.random.default_rng(seed)
    X = [workloads.bf16_round(rng.standard_normal((B, H, n, 64)).astype(np.float32)) for _ in range(3)]
    return workloads.Workload(f"small{seed}", B, H, n, 64, "bf16", X[0], X[1], X[2], None, None, [], seed, "")


@pytest.mark.parametrize("n", [1, 5, 63, 64, 65, 130])
def test_u8i4_edge_lengths(oracle_mod, n):
    w = _small(60 + n, n=n)
    w.seqlens = np.array([n, max(1, n // 2), 1], np.int32)
    Q, K, V, seq, _ = _inputs(w)
    for N in (0, 1, 3, n + 2):
        O = had.had_attention(Q, K, V, N=N, mode="u8i4", seqlens=seq).float().cpu().numpy()
        ref = oracle_mod.attention(w.Q, w.K, w.V, N=N, mode=MODE, seqlens=w.seqlens).O
        assert np.max(np.abs(O - ref)) <= _tol(w), N
        # rows past a sequence's length are written as 0
        for b in range(w.B):
            assert not O[b, :, int(w.seqlens[b]):].any()


def test_u8i4_head_dim_128(oracle_mod):
    w = workloads.deit(128, B=4)
    Q, K, V, seq, bias = _inputs(w)
    ob = _obias(oracle_mod, w)
    rows = _rows(w, 24, 29)
    for N in (0, 16):
        O = _flat(had.had_attention(Q, K, V, N=N, mode="u8i4", bias=bias)).float().cpu().numpy()[rows]
        ref = oracle_mod.attention(w.Q, w.K, w.V, N=N, mode=MODE, bias=ob, rows=rows)
        assert np.max(np.abs(O - ref.O)) <= _tol(w) + (_tie(w) if N else 0.0), N
    g = workloads.grid(2, 2, 4, 128, 0, [512, 300], seed=47, d=128)
    Q, K, V, seq, bias = _inputs(g)
    rows = _rows(g, 32, 31)
    N = g.n // 8
    O = _flat(had.had_attention(Q, K, V, N=N, mode="u8i4", seqlens=seq, bias=bias)).float().cpu().numpy()[rows]
    ref = oracle_mod.attention(g.Q, g.K, g.V, N=N, mode=MODE, seqlens=g.seqlens, bias=_obias(oracle_mod, g), rows=rows)
    assert np.max(np.abs(O - ref.O)) <= _tol(g) + _tie(g)


# ----------------------------------------------------------------------------- the other entry points

def test_u8i4_prepared_and_host_entry_points_match(oracle_mod):
    w = _sub(_workload("deit"), 6)
    w.seqlens = np.array([197, 150, 65, 1, 197, 100], np.int32)
    Q, K, V, seq, bias = _inputs(w)
    L = had.lib()
    for N in (0, 30):
        ref = had.had_attention(Q, K, V, N=N, mode="u8i4", seqlens=seq, bias=bias)
        # two stages over one workspace
        shp = had.make_shape(Q, seq)
        bs = had._bias_struct(bias)
        nbytes = L.had_attention_workspace_size(ctypes.byref(shp), N, had.HAD_MODE_U8I4, bs)
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        out = torch.empty_like(ref)
        st = L.had_attention_prepare(ctypes.c_void_p(Q.data_ptr()), ctypes.c_void_p(K.data_ptr()),
                                     ctypes.c_void_p(V.data_ptr()), ctypes.byref(shp), bs, N, had.HAD_MODE_U8I4,
                                     ctypes.c_void_p(ws.data_ptr()), nbytes, None)
        assert st == had.HAD_OK
        st = L.had_attention_prepared(ctypes.c_void_p(V.data_ptr()), ctypes.byref(shp), bs, None, None, N,
                                      had.HAD_MODE_U8I4, ctypes.c_void_p(out.data_ptr()), 1,
                                      ctypes.c_void_p(ws.data_ptr()), nbytes, None)
        assert st == had.HAD_OK
        torch.cuda.synchronize()
        assert torch.equal(out, ref), N
        # host arrays in and out, in chunks of the batch
        hbias = had.RelPosBias(bias.table.cpu(), bias.gh, bias.gw, bias.prefix)
        for chunk in (0, 4):
            got = had.had_attention_host(Q.cpu(), K.cpu(), V.cpu(), N=N, mode="u8i4", seqlens=seq.cpu(), bias=hbias,
                                         chunk_b=chunk)
            assert torch.equal(got, ref.cpu()), (N, chunk)

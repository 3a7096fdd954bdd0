"""GPU parity at head dims other than 64 (BinaryAttention benchmarks its kernel at
head dim 128): the library, through its C ABI, against the oracle, which takes any
multiple of 32.

Pack and int8 V at d = 32 and 128; the fused kernel at d = 128 (64-channel panels
of the Q~, K~ and V tiles, 129 score levels, 128 O columns in tensor memory) on
tiny, DeiT-shaped and T5-1024-shaped inputs, with the same bars as at d = 64.
"""
import numpy as np
import pytest

import workloads

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import binarized_qk_sparse_b200 as had  # noqa: E402


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


def _sub(w, B):
    return workloads.Workload(w.name + f"_sub{B}", B, w.H, w.n, w.d, w.dtype, w.Q[:B], w.K[:B], w.V[:B],
                              None if w.seqlens is None else w.seqlens[:B], w.bias, w.passes, w.seed, w.recipe)


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


def _tiny():
    return _cache.setdefault("tiny", workloads.tiny(128))


def _deit():
    return _cache.setdefault("deit", workloads.deit(128, B=4))


def _t5():
    return _cache.setdefault("t5", workloads.t5(1024, 128, B=2))


@pytest.mark.parametrize("d", [32, 128])
@pytest.mark.parametrize("seqlens", [None, [100, 37, 128]])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_pack_and_int8_v_other_head_dims(oracle_mod, d, seqlens, dtype):
    rng = np.random.default_rng(d + (0 if seqlens is None else 1))
    B = 1 if seqlens is None else len(seqlens)
    X = rng.standard_normal((B, 3, 128, d), dtype=np.float32) + rng.standard_normal((1, 3, 1, d), dtype=np.float32)
    if dtype == "bf16":
        X = workloads.bf16_round(X)
    sl = None if seqlens is None else np.array(seqlens, np.int32)
    Xd = torch.from_numpy(X).to(torch.bfloat16 if dtype == "bf16" else torch.float32).cuda()
    sd = None if sl is None else torch.from_numpy(sl).cuda()
    bits, mu = had.had_binarize_pack(Xd, sd)
    mu_o = oracle_mod.channel_mean(X, sl)
    np.testing.assert_array_equal(mu.cpu().numpy(), mu_o)
    np.testing.assert_array_equal(bits.cpu().numpy().view(np.uint32), oracle_mod.sign_pack(X, mu_o, sl))
    bits2, mu2 = had.had_binarize_pack_noalloc(Xd, sd)
    np.testing.assert_array_equal(bits2.cpu().numpy(), bits.cpu().numpy())
    Vq, sc = had.had_quantize_v(Xd, sd)
    Vq_o, sc_o = oracle_mod.v_quant(X, sl)
    np.testing.assert_array_equal(sc.cpu().numpy(), sc_o)
    np.testing.assert_array_equal(Vq.cpu().numpy(), Vq_o)


@pytest.mark.parametrize("which", ["tiny", "t5"])
def test_d128_fused_kernel_scores(oracle_mod, which):
    w = _tiny() if which == "tiny" else _sub(_t5(), 1)
    Q, K, V, seq, _ = _inputs(w)
    S = had.had_attention_scores(Q, K, seq).cpu().numpy()
    ref = oracle_mod.attention(w.Q, w.K, w.V, N=0, seqlens=w.seqlens, rows=np.zeros(0, np.int64))
    np.testing.assert_array_equal(S, oracle_mod.binary_scores(ref.qbits, ref.kbits, 128, w.seqlens))


@pytest.mark.parametrize("N", [15, 0, 1, 127])
def test_d128_tiny(oracle_mod, N):
    w = _tiny()
    Q, K, V, seq, bias = _inputs(w)
    O = had.had_attention(Q, K, V, N=N, mode="float").cpu().numpy()
    ref = oracle_mod.attention(w.Q, w.K, w.V, N=N, want_idx=N > 0)
    assert np.max(np.abs(O - ref.O)) <= _tol(w)
    if N > 0:
        idx = had.had_topn_indices(Q, K, N).cpu().numpy().reshape(-1, N)
        np.testing.assert_array_equal(idx, ref.idx)


def test_d128_t5_1024_topn(oracle_mod):
    w = _t5()
    Q, K, V, seq, bias = _inputs(w)
    N = 120
    idx = had.had_topn_indices(Q, K, N).cpu().numpy().reshape(-1, N)
    rows = _rows(w, 48, 5)
    ref = oracle_mod.attention(w.Q, w.K, w.V, N=N, rows=rows, want_idx=True)
    np.testing.assert_array_equal(idx[rows], ref.idx)
    O = _flat(had.had_attention(Q, K, V, N=N, mode="float")).float().cpu().numpy()[rows]
    assert np.max(np.abs(O - ref.O)) <= _tol(w)


def test_d128_deit_dense_u8i8_and_topn_with_bias(oracle_mod):
    w = _deit()
    Q, K, V, seq, bias = _inputs(w)
    ob = _obias(oracle_mod, w)
    rows = _rows(w, 24, 6)
    Oq = _flat(had.had_attention(Q, K, V, N=0, mode="u8i8", bias=bias)).float().cpu().numpy()[rows]
    ref_q = oracle_mod.attention(w.Q, w.K, w.V, N=0, mode=1, bias=ob, rows=rows)
    assert np.max(np.abs(Oq - ref_q.O)) <= _tol(w)
    # every code of the first head of each sequence
    A = had.had_attention_codes_u8(Q, K, V, 0, w.n, N=0, bias=bias).cpu().numpy()
    A = A.reshape(w.B, w.H, w.n, w.n)[:, 0].reshape(-1, w.n)
    band = np.array([b * w.H * w.n + i for b in range(w.B) for i in range(w.n)], np.int64)
    ref_c = oracle_mod.attention(w.Q, w.K, w.V, N=0, mode=1, bias=ob, rows=band, want_codes=True).Aq
    diff = np.abs(A.astype(np.int32) - ref_c.astype(np.int32))
    assert diff.max() <= 1 and (diff > 0).mean() <= 1e-3
    for N in (16, 100):
        idx = _flat(had.had_topn_indices(Q, K, N, bias=bias)).cpu().numpy()[rows]
        ref_f = oracle_mod.attention(w.Q, w.K, w.V, N=N, bias=ob, rows=rows, want_idx=True)
        np.testing.assert_array_equal(idx, ref_f.idx)
        Of = _flat(had.had_attention(Q, K, V, N=N, mode="float", bias=bias)).float().cpu().numpy()[rows]
        assert np.max(np.abs(Of - ref_f.O)) <= _tol(w)


def test_d128_grid_rows_and_lengths(oracle_mod):
    """A 4x128 grid with ragged lengths: per-warp bias windows (top-N) and the
    global-memory exp(bias) path (dense), at head dim 128."""
    w = workloads.grid(2, 2, 4, 128, 0, [512, 300], seed=41, d=128)
    Q, K, V, seq, bias = _inputs(w)
    ob = _obias(oracle_mod, w)
    rows = _rows(w, 40, 7)
    N = w.n // 8
    for mode in (0, 1):
        O = _flat(had.had_attention(Q, K, V, N=N, mode="float" if mode == 0 else "u8i8", seqlens=seq,
                                    bias=bias)).float().cpu().numpy()[rows]
        ref = oracle_mod.attention(w.Q, w.K, w.V, N=N, mode=mode, seqlens=w.seqlens, bias=ob, rows=rows)
        assert np.max(np.abs(O - ref.O)) <= _tol(w) + mode * float(np.max(np.abs(w.V))) / 255
    idx = _flat(had.had_topn_indices(Q, K, N, seq, bias)).cpu().numpy()[rows]
    np.testing.assert_array_equal(
        idx, oracle_mod.attention(w.Q, w.K, w.V, N=N, seqlens=w.seqlens, bias=ob, rows=rows, want_idx=True).idx)
    Od = _flat(had.had_attention(Q, K, V, N=0, mode="u8i8", seqlens=seq, bias=bias)).float().cpu().numpy()[rows]
    ref_d = oracle_mod.attention(w.Q, w.K, w.V, N=0, mode=1, seqlens=w.seqlens, bias=ob, rows=rows)
    assert np.max(np.abs(Od - ref_d.O)) <= _tol(w)


@pytest.mark.parametrize("which", ["deit", "grid"])
def test_d128_dense_comparison_mode(oracle_mod, which):
    """The comparison mode (standard bf16 attention on the tcgen05 tensor cores) at
    head dim 128, against the oracle's fp64 attention on the same bf16 values."""
    if which == "deit":
        w = _deit()
    else:
        w = workloads.grid(2, 2, 4, 128, 0, [512, 300], seed=43, d=128)
    Q, K, V, seq, bias = _inputs(w)
    rows = _rows(w, 32, 8)
    O = _flat(had.had_dense_reference_mode(Q, K, V, seqlens=seq, bias=bias)).float().cpu().numpy()[rows]
    ref = oracle_mod.dense_attention(w.Q, w.K, w.V, seqlens=w.seqlens, bias=_obias(oracle_mod, w), rows=rows)
    assert np.max(np.abs(O - ref)) <= _tol(w)

"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle on the
same seeded inputs.

Bars: bit-exact packed bits, channel means, integer scores, top-N index sets
and int8 V; O within max-abs 1e-3*max|V| (fp32 V) or 1e-2*max|V| (bf16 V);
uint8 attention codes within 1 LSB on at most 0.1% of entries and never more.
The full-size stress workload (B2 H16 n16384) runs in the launch configuration
the benchmark times; the oracle checks seeded samples of its rows.
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
    if w.dtype == "bf16":
        t = t.to(torch.bfloat16)
    return t.cuda()


def _dev_inputs(w):
    Q, K, V = _dev(w, w.Q), _dev(w, w.K), _dev(w, w.V)
    seq = None if w.seqlens is None else torch.from_numpy(w.seqlens).cuda()
    bias = None
    if isinstance(w.bias, workloads.DenseBias):
        bias = had.DenseBias(torch.from_numpy(w.bias.table).cuda())
    elif w.bias is not None:
        bias = had.RelPosBias(torch.from_numpy(w.bias.table).cuda(), w.bias.gh, w.bias.gw, w.bias.prefix)
    return Q, K, V, seq, bias


def _oracle_bias(oracle_mod, w):
    if w.bias is None:
        return None
    if isinstance(w.bias, workloads.DenseBias):
        return oracle_mod.DenseBias(w.bias.table)
    return oracle_mod.RelPosBias(w.bias.table, w.bias.gh, w.bias.gw, w.bias.prefix)


def _tol(w):
    return (1e-3 if w.dtype == "f32" else 1e-2) * float(np.max(np.abs(w.V)))


_cache = {}


def _workload(name):
    if name not in _cache:
        _cache[name] = workloads.by_name(name)
    return _cache[name]


def _sample_rows(w, per_head, seed):
    rng = np.random.default_rng(seed)
    rows = []
    for bh in range(w.B * w.H):
        L = w.n if w.seqlens is None else int(w.seqlens[bh // w.H])
        ii = rng.choice(L, size=min(per_head, L), replace=False)
        rows.extend(bh * w.n + int(i) for i in sorted(ii))
    return np.array(rows, np.int64)


def _flat(t):
    return t.reshape(-1, t.shape[-1])


# ----------------------------------------------------------------------------- binarize + pack

@pytest.mark.parametrize("name", ["tiny", "deit", "bert", "t5_256"])
def test_binarize_pack_bit_exact(oracle_mod, name):
    w = _workload(name)
    Q, K, V, seq, _ = _dev_inputs(w)
    for X, Xn in ((Q, w.Q), (K, w.K)):
        bits, mu = had.had_binarize_pack(X, seq)
        mu_o = oracle_mod.channel_mean(Xn, w.seqlens)
        bits_o = oracle_mod.sign_pack(Xn, mu_o, w.seqlens)
        np.testing.assert_array_equal(mu.cpu().numpy(), mu_o)
        np.testing.assert_array_equal(bits.cpu().numpy().view(np.uint32), bits_o)
        # with the oracle's means passed in, the sign/pack step alone
        bits2, _ = had.had_binarize_pack(X, seq, mu_in=torch.from_numpy(mu_o).cuda())
        np.testing.assert_array_equal(bits2.cpu().numpy().view(np.uint32), bits_o)


def test_binarize_pack_stress_full_size(oracle_mod):
    w = _workload("stress")
    Q, K, V, seq, _ = _dev_inputs(w)
    bits, mu = had.had_binarize_pack(K, seq)
    mu_o = oracle_mod.channel_mean(w.K)
    np.testing.assert_array_equal(mu.cpu().numpy(), mu_o)
    got = bits.cpu().numpy().view(np.uint32)
    rng = np.random.default_rng(11)
    for b in range(w.B):
        for h in range(w.H):
            ii = np.sort(rng.choice(w.n, size=512, replace=False))
            ref = oracle_mod.sign_pack(w.K[b, h, ii][None, None], mu_o[b, h][None, None])
            np.testing.assert_array_equal(got[b, h, ii], ref[0, 0])


# ----------------------------------------------------------------------------- scores

@pytest.mark.parametrize("name", ["tiny", "bert", "t5_256"])
def test_integer_scores_bit_exact(oracle_mod, name):
    w = _workload(name)
    if name == "bert":  # keep the score matrix small: 4 sequences
        w = workloads.Workload(w.name, 4, w.H, w.n, w.d, w.dtype, w.Q[:4], w.K[:4], w.V[:4], w.seqlens[:4], None,
                               w.passes, w.seed, w.recipe)
    if name == "t5_256":
        w = workloads.Workload(w.name, 2, w.H, w.n, w.d, w.dtype, w.Q[:2], w.K[:2], w.V[:2], None, None, w.passes,
                               w.seed, w.recipe)
    Q, K, V, seq, _ = _dev_inputs(w)
    qb, _ = had.had_binarize_pack(Q, seq)
    kb, _ = had.had_binarize_pack(K, seq)
    S = had.had_scores_int(qb, kb, seq).cpu().numpy()
    S_o = oracle_mod.binary_scores(qb.cpu().numpy().view(np.uint32), kb.cpu().numpy().view(np.uint32), 64, w.seqlens)
    np.testing.assert_array_equal(S, S_o)


def _subset(w, B, name_suffix=""):
    return workloads.Workload(w.name + name_suffix, B, w.H, w.n, w.d, w.dtype, w.Q[:B], w.K[:B], w.V[:B],
                              None if w.seqlens is None else w.seqlens[:B], None, w.passes, w.seed, w.recipe)


@pytest.mark.parametrize("name,B", [("tiny", 1), ("bert", 4), ("t5_256", 2), ("t5_1024", 1)])
def test_fused_kernel_scores_bit_exact(oracle_mod, name, B):
    """The scores the fused kernel forms in tensor memory (+-1 int8 tcgen05 MMA),
    read back from it, against the oracle's d - 2*popcount on its own bits."""
    w = _subset(_workload(name), B)
    Q, K, V, seq, _ = _dev_inputs(w)
    S = had.had_attention_scores(Q, K, seq).cpu().numpy()
    ref = oracle_mod.attention(w.Q, w.K, w.V, N=0, seqlens=w.seqlens, rows=np.zeros(0, np.int64))
    S_o = oracle_mod.binary_scores(ref.qbits, ref.kbits, 64, w.seqlens)
    np.testing.assert_array_equal(S, S_o)


# ----------------------------------------------------------------------------- top-N index sets

def _oracle_full(oracle_mod, w, N, mode, rows=None, want_idx=False, want_codes=False):
    key = (w.name, N, mode, None if rows is None else rows.tobytes(), want_idx, want_codes)
    if key not in _cache:
        b = _oracle_bias(oracle_mod, w)
        _cache[key] = oracle_mod.attention(w.Q, w.K, w.V, N=N, mode=mode, seqlens=w.seqlens, bias=b, rows=rows,
                                           want_idx=want_idx, want_codes=want_codes)
    return _cache[key]


@pytest.mark.parametrize("name,N", [("tiny", 15), ("tiny", 1), ("tiny", 127), ("bert", 30), ("t5_128", 15),
                                    ("t5_256", 30), ("t5_512", 60), ("t5_1024", 120)])
def test_topn_sets_bit_exact(oracle_mod, name, N):
    w = _workload(name)
    Q, K, V, seq, bias = _dev_inputs(w)
    idx = had.had_topn_indices(Q, K, N, seq, bias).cpu().numpy().reshape(-1, N)
    ref = _oracle_full(oracle_mod, w, N, 0, want_idx=True).idx
    np.testing.assert_array_equal(idx, ref)


def test_topn_sets_with_bias_deit_shape(oracle_mod):
    w = _workload("deit")
    w = workloads.Workload(w.name + "_b4", 4, w.H, w.n, w.d, w.dtype, w.Q[:4], w.K[:4], w.V[:4], None, w.bias,
                           w.passes, w.seed, w.recipe)
    Q, K, V, seq, bias = _dev_inputs(w)
    for N in (1, 16, 100):
        idx = had.had_topn_indices(Q, K, N, seq, bias).cpu().numpy().reshape(-1, N)
        ref = _oracle_full(oracle_mod, w, N, 0, want_idx=True).idx
        np.testing.assert_array_equal(idx, ref)


def test_topn_sets_stress_full_size(oracle_mod):
    w = _workload("stress")
    Q, K, V, seq, bias = _dev_inputs(w)
    N = 1920
    idx = had.had_topn_indices(Q, K, N, seq, bias)
    rows = _sample_rows(w, 24, 12)
    got = _flat(idx)[torch.from_numpy(rows).cuda()].cpu().numpy()
    del idx
    ref = _oracle_full(oracle_mod, w, N, 0, rows=rows, want_idx=True).idx
    np.testing.assert_array_equal(got, ref)


# ----------------------------------------------------------------------------- outputs

@pytest.mark.parametrize("name,N", [("tiny", 15), ("tiny", 0), ("bert", 30), ("t5_128", 15), ("t5_256", 30),
                                    ("t5_512", 60), ("t5_1024", 120)])
def test_float_output_within_tolerance(oracle_mod, name, N):
    w = _workload(name)
    Q, K, V, seq, bias = _dev_inputs(w)
    O = had.had_attention(Q, K, V, N=N, mode="float", seqlens=seq, bias=bias).float().cpu().numpy()
    ref = _oracle_full(oracle_mod, w, N, 0).O
    err = np.max(np.abs(O - ref))
    assert err <= _tol(w), (err, _tol(w))


def test_float_output_dense_with_bias(oracle_mod):
    w = _workload("deit")
    w = workloads.Workload(w.name + "_b4", 4, w.H, w.n, w.d, w.dtype, w.Q[:4], w.K[:4], w.V[:4], None, w.bias,
                           w.passes, w.seed, w.recipe)
    Q, K, V, seq, bias = _dev_inputs(w)
    for N in (0, 50):
        O = had.had_attention(Q, K, V, N=N, mode="float", bias=bias).float().cpu().numpy()
        ref = _oracle_full(oracle_mod, w, N, 0).O
        assert np.max(np.abs(O - ref)) <= _tol(w)


def _codes_ok(got, ref):
    diff = np.abs(got.astype(np.int32) - ref.astype(np.int32))
    assert diff.max() <= 1, diff.max()
    assert (diff > 0).mean() <= 1e-3, (diff > 0).mean()


def test_u8i8_deit_full(oracle_mod):
    w = _workload("deit")
    Q, K, V, seq, bias = _dev_inputs(w)
    O = had.had_attention(Q, K, V, N=0, mode="u8i8", seqlens=seq, bias=bias).float().cpu().numpy()
    ref = _oracle_full(oracle_mod, w, 0, 1, want_codes=True)
    assert np.max(np.abs(O - ref.O)) <= _tol(w)
    A = had.had_attention_codes_u8(Q, K, V, 0, w.n, N=0, seqlens=seq, bias=bias).cpu().numpy()
    _codes_ok(A.reshape(-1, w.n), ref.Aq)
    Vq, sc = had.had_quantize_v(V, seq)
    np.testing.assert_array_equal(Vq.cpu().numpy(), ref.Vq)
    np.testing.assert_array_equal(sc.cpu().numpy(), ref.vscale)


def test_u8i8_topn_bert(oracle_mod):
    w = _workload("bert")
    Q, K, V, seq, bias = _dev_inputs(w)
    O = had.had_attention(Q, K, V, N=30, mode="u8i8", seqlens=seq).float().cpu().numpy()
    ref = _oracle_full(oracle_mod, w, 30, 1, want_codes=True)
    assert np.max(np.abs(O - ref.O)) <= _tol(w)
    A = had.had_attention_codes_u8(Q, K, V, 0, w.n, N=30, seqlens=seq).cpu().numpy()
    _codes_ok(A.reshape(-1, w.n), ref.Aq)


def test_stress_full_size_both_passes(oracle_mod):
    w = _workload("stress")
    Q, K, V, seq, bias = _dev_inputs(w)
    rows = _sample_rows(w, 16, 13)
    rows_t = torch.from_numpy(rows).cuda()
    Of = _flat(had.had_attention(Q, K, V, N=1920, mode="float", bias=bias))[rows_t].float().cpu().numpy()
    ref_f = _oracle_full(oracle_mod, w, 1920, 0, rows=rows)
    assert np.max(np.abs(Of - ref_f.O)) <= _tol(w)
    Oq = _flat(had.had_attention(Q, K, V, N=0, mode="u8i8", bias=bias))[rows_t].float().cpu().numpy()
    ref_q = _oracle_full(oracle_mod, w, 0, 1, rows=rows, want_codes=True)
    assert np.max(np.abs(Oq - ref_q.O)) <= _tol(w)
    # codes of a contiguous band of rows in every head
    r0, r1 = 5000, 5008
    A = had.had_attention_codes_u8(Q, K, V, r0, r1, N=0, bias=bias).cpu().numpy().reshape(-1, w.n)
    band = np.array([bh * w.n + i for bh in range(w.B * w.H) for i in range(r0, r1)], np.int64)
    ref_c = _oracle_full(oracle_mod, w, 0, 1, rows=band, want_codes=True)
    _codes_ok(A, ref_c.Aq)


# ----------------------------------------------------------------------------- bias layouts and lengths

def _check_grid(oracle_mod, w, per_head, seed):
    """Dense uint8 (O and codes), top-N float O and index sets, and dense index
    sets (N = n) of a relative-position-bias workload, on sampled rows."""
    Q, K, V, seq, bias = _dev_inputs(w)
    rows = _sample_rows(w, per_head, seed)
    rows_t = torch.from_numpy(rows).cuda()
    N = max(1, w.n // 8)
    Oq = _flat(had.had_attention(Q, K, V, N=0, mode="u8i8", seqlens=seq, bias=bias))[rows_t].float().cpu().numpy()
    ref_q = _oracle_full(oracle_mod, w, 0, 1, rows=rows)
    assert np.max(np.abs(Oq - ref_q.O)) <= _tol(w)
    Of = _flat(had.had_attention(Q, K, V, N=N, mode="float", seqlens=seq, bias=bias))[rows_t].float().cpu().numpy()
    ref_f = _oracle_full(oracle_mod, w, N, 0, rows=rows)
    assert np.max(np.abs(Of - ref_f.O)) <= _tol(w)
    for n_keep in (N, w.n):
        idx = _flat(had.had_topn_indices(Q, K, n_keep, seq, bias))[rows_t].cpu().numpy()
        ref_i = _oracle_full(oracle_mod, w, n_keep, 0, rows=rows, want_idx=True).idx
        np.testing.assert_array_equal(idx, ref_i)
    # codes of every row of the first head of each batch (keys past L must be 0)
    A = had.had_attention_codes_u8(Q, K, V, 0, w.n, N=0, seqlens=seq, bias=bias).cpu().numpy()
    A = A.reshape(w.B, w.H, w.n, w.n)[:, 0].reshape(-1, w.n)
    band = np.array([b * w.H * w.n + i for b in range(w.B) for i in range(w.n)], np.int64)
    ref_c = _oracle_full(oracle_mod, w, 0, 1, rows=band, want_codes=True)
    _codes_ok(A, ref_c.Aq)


@pytest.mark.parametrize("gh,gw,prefix,seqlens", [
    (14, 14, 1, [197, 150, 65, 1]),      # per-head offset table, class token, ragged lengths
    (16, 128, 0, None),                  # 64-key tiles inside one image row: closed-form offsets
    (16, 128, 0, [2048, 1000]),          # same grid with lengths: offsets computed per tile
    (8, 160, 0, None),                   # tiles crossing image rows, n > 1024: offsets per tile
    (6, 30, 2, [182, 97]),               # two class tokens, ragged lengths, table offsets
])
def test_relpos_bias_layouts(oracle_mod, gh, gw, prefix, seqlens):
    B = 1 if seqlens is None else len(seqlens)
    w = workloads.grid(B, 2, gh, gw, prefix, seqlens)
    _check_grid(oracle_mod, w, 24, 21)


@pytest.mark.parametrize("gh,gw,seqlens", [
    (4, 64, None),               # a CTA's 128 rows span two image rows (warps 0-1 and 2-3)
    (8, 128, [1024, 700]),       # one image row per CTA; ragged lengths (a partial last tile)
    (3, 192, None),              # image rows of 192 patches: CTAs straddle two rows
    (2, 256, [512, 333]),        # two CTAs per image row
])
def test_topn_bias_row_windows(oracle_mod, gh, gw, seqlens):
    """Top-N with a relative-position bias on grids whose rows hold a multiple of 64
    patches (each warp reads its bias from a window staged in shared memory): float
    and uint8 O, kept sets and the uint8 codes, against the oracle."""
    B = 1 if seqlens is None else len(seqlens)
    w = workloads.grid(B, 2, gh, gw, 0, seqlens, seed=31)
    Q, K, V, seq, bias = _dev_inputs(w)
    rows = _sample_rows(w, 40, 17)
    rows_t = torch.from_numpy(rows).cuda()
    N = max(1, w.n // 8)
    Of = _flat(had.had_attention(Q, K, V, N=N, mode="float", seqlens=seq, bias=bias))[rows_t].float().cpu().numpy()
    assert np.max(np.abs(Of - _oracle_full(oracle_mod, w, N, 0, rows=rows).O)) <= _tol(w)
    Oq = _flat(had.had_attention(Q, K, V, N=N, mode="u8i8", seqlens=seq, bias=bias))[rows_t].float().cpu().numpy()
    assert np.max(np.abs(Oq - _oracle_full(oracle_mod, w, N, 1, rows=rows).O)) <= _tol(w) + float(np.max(np.abs(w.V))) / 255
    idx = _flat(had.had_topn_indices(Q, K, N, seq, bias))[rows_t].cpu().numpy()
    np.testing.assert_array_equal(idx, _oracle_full(oracle_mod, w, N, 0, rows=rows, want_idx=True).idx)
    A = had.had_attention_codes_u8(Q, K, V, 0, w.n, N=N, seqlens=seq, bias=bias).cpu().numpy()
    A = A.reshape(w.B, w.H, w.n, w.n)[:, 1].reshape(-1, w.n)
    band = np.array([(b * w.H + 1) * w.n + i for b in range(w.B) for i in range(w.n)], np.int64)
    _codes_ok(A, _oracle_full(oracle_mod, w, N, 1, rows=band, want_codes=True).Aq)
    # dense float: the exp(bias) windows when the table is too large for shared memory
    Od = _flat(had.had_attention(Q, K, V, N=0, mode="float", seqlens=seq, bias=bias))[rows_t].float().cpu().numpy()
    assert np.max(np.abs(Od - _oracle_full(oracle_mod, w, 0, 0, rows=rows).O)) <= _tol(w)


# ----------------------------------------------------------------------------- comparison mode

@pytest.mark.parametrize("case", ["deit", "bert", "t5_1024", "grid_rows"])
def test_dense_reference_mode(oracle_mod, case):
    """The comparison mode: standard attention on the unbinarized bf16 inputs on the
    tcgen05 tensor cores, against the oracle's fp64 attention on the same values
    (relative-position bias in shared memory, ragged lengths, no bias, and per-warp
    bias windows on a 16x128 grid)."""
    if case == "grid_rows":
        w = workloads.grid(1, 2, 16, 128, 0, None, seed=13)
    else:
        w = _subset(_workload(case), 4 if case != "t5_1024" else 2)
        if case == "deit":
            w = workloads.Workload(w.name, w.B, w.H, w.n, w.d, w.dtype, w.Q, w.K, w.V, None, _workload("deit").bias,
                                   w.passes, w.seed, w.recipe)
    Q, K, V, seq, bias = _dev_inputs(w)
    rows = _sample_rows(w, 48, 3)
    O = _flat(had.had_dense_reference_mode(Q, K, V, seqlens=seq, bias=bias)).float().cpu().numpy()[rows]
    ref = oracle_mod.dense_attention(w.Q, w.K, w.V, seqlens=w.seqlens, bias=_oracle_bias(oracle_mod, w), rows=rows)
    assert np.max(np.abs(O - ref)) <= _tol(w)


# ----------------------------------------------------------------------------- edge cases

def _small(seed, B=3, H=2, n=70, dtype="bf16"):
    rng = np.random.default_rng(seed)
    Q = workloads.bf16_round(rng.standard_normal((B, H, n, 64)).astype(np.float32))
    K = workloads.bf16_round(rng.standard_normal((B, H, n, 64)).astype(np.float32))
    V = workloads.bf16_round(rng.standard_normal((B, H, n, 64)).astype(np.float32))
    return workloads.Workload(f"small{seed}", B, H, n, 64, dtype, Q, K, V, None, None, [], seed, "")


@pytest.mark.parametrize("n", [1, 5, 63, 64, 65, 130])
def test_edge_lengths(oracle_mod, n):
    w = _small(20 + n, n=n)
    w.seqlens = np.array([n, max(1, n // 2), 1], np.int32)
    Q, K, V, seq, bias = _dev_inputs(w)
    for N in (0, 1, 3, n + 2):
        O = had.had_attention(Q, K, V, N=N, seqlens=seq).float().cpu().numpy()
        ref = oracle_mod.attention(w.Q, w.K, w.V, N=N, seqlens=w.seqlens).O
        assert np.max(np.abs(O - ref)) <= _tol(w)
        Oq = had.had_attention(Q, K, V, N=N, mode="u8i8", seqlens=seq).float().cpu().numpy()
        refq = oracle_mod.attention(w.Q, w.K, w.V, N=N, mode=1, seqlens=w.seqlens).O
        assert np.max(np.abs(Oq - refq)) <= _tol(w)
        if N >= 1:
            idx = had.had_topn_indices(Q, K, N, seq).cpu().numpy().reshape(-1, N)
            np.testing.assert_array_equal(idx, oracle_mod.attention(w.Q, w.K, w.V, N=N, seqlens=w.seqlens,
                                                                    want_idx=True).idx)


def test_all_ties_keep_lowest_indices(oracle_mod):
    # constant Q and K: every score equals d, so the kept set must be keys 0..N-1
    w = _small(30, B=1, H=1, n=200)
    w.Q[:] = 1.0
    w.K[:] = -2.0
    Q, K, V, seq, bias = _dev_inputs(w)
    idx = had.had_topn_indices(Q, K, 17).cpu().numpy().reshape(-1, 17)
    assert (idx == np.arange(17)[None, :]).all()
    O = had.had_attention(Q, K, V, N=17).float().cpu().numpy()
    ref = oracle_mod.attention(w.Q, w.K, w.V, N=17).O
    assert np.max(np.abs(O - ref)) <= _tol(w)


@pytest.mark.parametrize("mode", ["float", "u8i8"])
def test_threshold_ties_across_chunks_and_tiles(oracle_mod, mode):
    # Integer score levels make many exact ties at the threshold; the values of N
    # put the cut in different 32-key chunks and tiles of a row (the two threads
    # of a row must keep ties in key order between them).  fp32 inputs make one
    # wrongly kept key visible against the 1e-3 bar.
    # Each case runs without and with per-sequence lengths (the library uses two
    # threads per row for short ragged batches, one otherwise).  In uint8 mode a
    # code may differ by one LSB from the oracle's fp64 rounding (the codes' own
    # bar), which moves O by up to max|V|/255, so that is added to the O bar.
    m = 1 if mode == "u8i8" else 0
    w = _small(77, B=2, H=2, n=200, dtype="f32")
    Q, K, V, seq, bias = _dev_inputs(w)
    bar = _tol(w) + (float(np.max(np.abs(w.V))) / 255.0 if m else 0.0)
    lens = np.array([200, 161], np.int32)
    for N in (20, 40, 70, 100, 131, 180):
        for sl in (None, lens):
            seqt = None if sl is None else torch.from_numpy(sl).cuda()
            O = had.had_attention(Q, K, V, N=N, mode=mode, seqlens=seqt).float().cpu().numpy()
            ref = oracle_mod.attention(w.Q, w.K, w.V, N=N, mode=m, seqlens=sl).O
            assert np.max(np.abs(O - ref)) <= bar, (N, sl, np.max(np.abs(O - ref)))
    # every score equal: the kept set is keys 0..N-1 for any N
    w = _small(78, B=1, H=1, n=200, dtype="f32")
    w.Q[:] = 1.0
    w.K[:] = -2.0
    Q, K, V, seq, bias = _dev_inputs(w)
    bar = _tol(w) + (float(np.max(np.abs(w.V))) / 255.0 if m else 0.0)
    for N in (40, 100, 150):
        for sl in (None, np.array([200], np.int32)):
            seqt = None if sl is None else torch.from_numpy(sl).cuda()
            O = had.had_attention(Q, K, V, N=N, mode=mode, seqlens=seqt).float().cpu().numpy()
            ref = oracle_mod.attention(w.Q, w.K, w.V, N=N, mode=m, seqlens=sl).O
            assert np.max(np.abs(O - ref)) <= bar, (N, sl, np.max(np.abs(O - ref)))


def test_alpha_and_bias_ties(oracle_mod):
    # a bias table of few distinct values makes many exact logit ties
    w = _small(31, B=2, H=2, n=65)
    gh, gw, prefix = 8, 8, 1
    rng = np.random.default_rng(5)
    table = (rng.integers(-2, 3, size=(2, 15, 15)) * 0.25).astype(np.float32)
    w.bias = workloads.Bias(table, gh, gw, prefix)
    Q, K, V, seq, bias = _dev_inputs(w)
    aq, ak = np.array([1.5, 0.5], np.float32), np.array([2.0, 1.0], np.float32)
    b = oracle_mod.RelPosBias(table, gh, gw, prefix)
    for N in (1, 7, 30, 64):
        idx = had.had_topn_indices(Q, K, N, bias=bias, alpha_q=aq, alpha_k=ak).cpu().numpy().reshape(-1, N)
        ref = oracle_mod.attention(w.Q, w.K, w.V, N=N, bias=b, alpha_q=aq, alpha_k=ak, want_idx=True)
        np.testing.assert_array_equal(idx, ref.idx)
        O = had.had_attention(Q, K, V, N=N, bias=bias, alpha_q=aq, alpha_k=ak).float().cpu().numpy()
        assert np.max(np.abs(O - ref.O)) <= _tol(w)


def _dense_bias_workload(B, H, n, seqlens, seed, dtype="bf16"):
    rng = np.random.default_rng(seed)
    Q = workloads.bf16_round(rng.standard_normal((B, H, n, 64)).astype(np.float32))
    K = workloads.bf16_round(rng.standard_normal((B, H, n, 64)).astype(np.float32))
    V = workloads.bf16_round(rng.standard_normal((B, H, n, 64)).astype(np.float32))
    table = (rng.standard_normal((H, n, n)) * 0.1).astype(np.float32)
    sl = None if seqlens is None else np.asarray(seqlens, np.int32)
    return workloads.Workload(f"dense_bias_b{B}_h{H}_n{n}", B, H, n, 64, dtype, Q, K, V, sl,
                              workloads.DenseBias(table), [], seed, "")


@pytest.mark.parametrize("n,seqlens", [
    (70, [70, 33]),          # extended tables staged in shared memory, key offsets from a table
    (197, None),             # DeiT length: tables in global memory
    (197, [197, 120]),
    (1100, [1100, 700]),     # n > 1024: key offsets computed per tile by each warp
])
def test_dense_bias_matrix(oracle_mod, n, seqlens):
    # BinaryAttention §2.3's dense learnable matrix, b_ij = table[h][i][j]:
    # dense uint8 and float O, top-N float O and kept sets, uint8 codes
    w = _dense_bias_workload(len(seqlens or [0]), 2, n, seqlens, 40 + n)
    Q, K, V, seq, bias = _dev_inputs(w)
    rows = _sample_rows(w, 24, 3)
    rows_t = torch.from_numpy(rows).cuda()
    N = max(1, n // 8)
    for Nk, mode in ((0, "u8i8"), (0, "float"), (N, "float")):
        m = 1 if mode == "u8i8" else 0
        O = _flat(had.had_attention(Q, K, V, N=Nk, mode=mode, seqlens=seq, bias=bias))[rows_t].float().cpu().numpy()
        ref = _oracle_full(oracle_mod, w, Nk, m, rows=rows)
        assert np.max(np.abs(O - ref.O)) <= _tol(w), (Nk, mode)
    idx = _flat(had.had_topn_indices(Q, K, N, seq, bias))[rows_t].cpu().numpy()
    np.testing.assert_array_equal(idx, _oracle_full(oracle_mod, w, N, 0, rows=rows, want_idx=True).idx)
    r0, r1 = 0, min(n, 64)
    A = had.had_attention_codes_u8(Q, K, V, r0, r1, N=0, seqlens=seq, bias=bias).cpu().numpy().reshape(-1, n)
    band = np.array([bh * n + i for bh in range(w.B * w.H) for i in range(r0, r1)], np.int64)
    _codes_ok(A, _oracle_full(oracle_mod, w, 0, 1, rows=band, want_codes=True).Aq)


def test_dense_bias_matrix_reference_mode_and_host_entry(oracle_mod):
    w = _dense_bias_workload(2, 2, 197, [197, 150], 77)
    Q, K, V, seq, bias = _dev_inputs(w)
    O = had.had_dense_reference_mode(Q, K, V, seqlens=seq, bias=bias).float().cpu().numpy()
    ref = oracle_mod.dense_attention(w.Q, w.K, w.V, seqlens=w.seqlens, bias=_oracle_bias(oracle_mod, w))
    assert np.max(np.abs(O - ref)) <= 1e-2 * np.max(np.abs(w.V))
    dev = had.had_attention(Q, K, V, N=25, seqlens=seq, bias=bias).cpu()
    hb = had.DenseBias(bias.table.cpu())
    got = had.had_attention_host(Q.cpu(), K.cpu(), V.cpu(), N=25, seqlens=seq.cpu(), bias=hb, chunk_b=1)
    assert torch.equal(got, dev)


@pytest.mark.parametrize("mode", ["float", "u8i8"])
def test_bias_ties_at_the_threshold_fp32(oracle_mod, mode):
    # A bias table of five values on a 14x14 grid with four class tokens (n = 200,
    # four 64-key tiles) makes many exact logit ties; the values of N put the
    # threshold in different tiles, and the radix search ends either on one
    # logit value or on a bin of keys ranked after the weight pass.  fp32 inputs
    # make one wrongly kept key visible against the 1e-3 bar (uint8 mode: plus
    # one code LSB).  Index sets are compared exactly.
    m = 1 if mode == "u8i8" else 0
    w = _small(79, B=2, H=2, n=200, dtype="f32")
    rng = np.random.default_rng(9)
    table = (rng.integers(-2, 3, size=(2, 27, 27)) * 0.25).astype(np.float32)
    w.bias = workloads.Bias(table, 14, 14, 4)
    Q, K, V, seq, bias = _dev_inputs(w)
    b = oracle_mod.RelPosBias(table, 14, 14, 4)
    bar = _tol(w) + (float(np.max(np.abs(w.V))) / 255.0 if m else 0.0)
    for N in (20, 70, 131, 180):
        for sl in (None, np.array([200, 161], np.int32)):
            seqt = None if sl is None else torch.from_numpy(sl).cuda()
            ref = oracle_mod.attention(w.Q, w.K, w.V, N=N, mode=m, seqlens=sl, bias=b, want_idx=True)
            O = had.had_attention(Q, K, V, N=N, mode=mode, seqlens=seqt, bias=bias).float().cpu().numpy()
            assert np.max(np.abs(O - ref.O)) <= bar, (N, sl, np.max(np.abs(O - ref.O)))
            idx = had.had_topn_indices(Q, K, N, seqt, bias).cpu().numpy().reshape(-1, N)
            np.testing.assert_array_equal(idx, ref.idx)


@pytest.mark.parametrize("pinned", [True, False])
def test_host_entry_point_matches_the_device_call(oracle_mod, pinned):
    # had_attention_host cuts the batch into chunks that run the same kernels as
    # had_attention: O is bit-identical for every chunk size, pinned or not
    w = _workload("deit")
    B = 6
    sub = workloads.Workload(w.name + "_b6", B, w.H, w.n, w.d, w.dtype, w.Q[:B], w.K[:B], w.V[:B],
                             np.array([197, 150, 65, 1, 197, 100], np.int32), w.bias, w.passes, w.seed, w.recipe)
    Q, K, V, seq, bias = _dev_inputs(sub)

    def host(t):
        t = t.cpu()
        return t.pin_memory() if pinned else t

    hQ, hK, hV = host(Q), host(K), host(V)
    hseq = sub_seq = torch.from_numpy(sub.seqlens)
    hbias = had.RelPosBias(host(bias.table), bias.gh, bias.gw, bias.prefix)
    for N, mode in ((0, "u8i8"), (0, "float"), (30, "float"), (30, "u8i8")):
        ref = had.had_attention(Q, K, V, N=N, mode=mode, seqlens=seq, bias=bias).cpu()
        for chunk in (0, 1, 4, 6):
            got = had.had_attention_host(hQ, hK, hV, N=N, mode=mode, seqlens=hseq, bias=hbias, chunk_b=chunk)
            assert got.device.type == "cpu"
            assert torch.equal(got, ref), (N, mode, chunk)
    # and against the oracle once, on fp32 output
    got = had.had_attention_host(hQ, hK, hV, N=30, mode="float", seqlens=sub_seq, bias=hbias, chunk_b=4,
                                 out_dtype=torch.float32).numpy()
    rows = _sample_rows(sub, 24, 5)
    ref = _oracle_full(oracle_mod, sub, 30, 0, rows=rows).O
    assert np.max(np.abs(got.reshape(-1, 64)[rows] - ref)) <= _tol(sub)


@pytest.mark.parametrize("L,code", [(6, 43), (30, 9), (102, 3), (510, 1)])
def test_u8_codes_round_half_up_at_exact_ties(oracle_mod, L, code):
    """Rows of L equal logits (identical Q rows and K rows: every score is d) have
    p = 1/L, and 255/L = k + 1/2 exactly: the codes must be floor(255 p + 0.5) = k + 1
    on both sides, bit for bit."""
    n, d = 512, 64
    rng = np.random.default_rng(5)
    q = workloads.bf16_round(rng.standard_normal(d).astype(np.float32))
    k = workloads.bf16_round(rng.standard_normal(d).astype(np.float32))
    Qn = np.broadcast_to(q, (1, 1, n, d)).copy()
    Kn = np.broadcast_to(k, (1, 1, n, d)).copy()
    Vn = workloads.bf16_round(rng.standard_normal((1, 1, n, d)).astype(np.float32))
    seq_n = np.array([L], np.int32)
    Q, K, V = (torch.from_numpy(x).to(torch.bfloat16).cuda() for x in (Qn, Kn, Vn))
    A = had.had_attention_codes_u8(Q, K, V, 0, n, N=0, seqlens=torch.from_numpy(seq_n).cuda()).cpu().numpy()
    ref = oracle_mod.attention(Qn, Kn, Vn, N=0, mode=1, seqlens=seq_n, want_codes=True)
    np.testing.assert_array_equal(A.reshape(n, n), ref.Aq.reshape(n, n))
    assert (A.reshape(n, n)[:L, :L] == code).all()


def test_timeout_path_reports_and_recovers(oracle_mod):
    """The fused kernel's bounded waits: with the test hook, one thread of every CTA
    waits on a barrier nothing completes; its bound (2e6 clocks, about 1 ms)
    expires, the CTAs wind down with zero output, and the status word says
    HAD_ERR_TIMEOUT.  The next normal call matches the oracle again."""
    w = _workload("tiny")
    Q, K, V, seq, bias = _dev_inputs(w)
    assert had.had_get_device_status() == had.HAD_OK
    try:
        had.had_debug_bounded_wait(2_000_000, True)
        O = had.had_attention(Q, K, V, N=15, mode="float")
        torch.cuda.synchronize()
    finally:
        had.had_debug_bounded_wait(0, False)
    assert had.had_get_device_status() == had.HAD_ERR_TIMEOUT
    assert not O.cpu().numpy().any()
    O2 = had.had_attention(Q, K, V, N=15, mode="float").cpu().numpy()
    assert had.had_get_device_status() == had.HAD_OK
    ref = _oracle_full(oracle_mod, w, 15, 0).O
    assert np.max(np.abs(O2 - ref)) <= _tol(w)


def test_bad_seqlens_raise_device_status():
    w = _small(32, B=2, H=1, n=64)
    Q, K, V, _, _ = _dev_inputs(w)
    assert had.had_get_device_status() == had.HAD_OK
    seq = torch.tensor([64, 0], dtype=torch.int32, device="cuda")
    O = had.had_attention(Q, K, V, N=5, seqlens=seq)
    assert had.had_get_device_status() == had.HAD_ERR_DEVICE
    assert had.had_get_device_status() == had.HAD_OK   # cleared on read
    assert not O[1].float().abs().sum().item()

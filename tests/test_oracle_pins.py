"""Pins for the CPU oracle: each test checks it against something other than itself.

What pins what (sources: "Hamming Attention Distillation" = HAD, abstract and
method summary; "BinaryAttention: One-Bit QK-Attention" = BA, §2.1-§2.4):
  - channel mean: closed forms on integer-valued inputs; exact fsum.
  - sign + pack: brute-force unpacking vs x < mu, bit-order probes, shift invariance.
  - score: the identity dot(sign q, sign k) = d - 2*Hamming (BA §2.1 distance
    view, §2.2 XNOR + popcount; HAD abstract) via numpy +-1 matmuls and an
    exhaustive 8-bit sweep; Theorem 1 (BA §2.1) statistically.
  - logit: bias indexing with an injective table (relative-position and dense
    matrix, BA §2.3); a dense matrix built from a relative-position table gives
    the same result as the table; alpha scale.
  - top-N: numpy lexsort brute force; N >= L reduces to dense; nesting; alpha invariance.
  - softmax / A.V: rows sum to 1; exp(-Hamming) shift form; independent dense
    attention in numpy; padded batch == each sequence alone.
  - quantization (BA §2.4): V reconstruction within s/2; |A_q/255 - p| <= 0.5/255;
    closed-form bound |O_q - O_f|; a one-key row gives A_q = 255.
"""
import math

import numpy as np
import pytest

import workloads


def _signs(X, mu, L):
    """+-1 matrix of sign(X - mu) over valid tokens (x < mu -> -1, else +1)."""
    return np.where(X[:L] < mu[None, :], -1, 1).astype(np.int64)


def _rng(seed):
    return np.random.default_rng(1000 + seed)


# ----------------------------------------------------------------------------- mean

def test_mean_closed_form_integer_inputs(oracle_mod):
    B, H, n, d = 2, 3, 40, 64
    X = np.zeros((B, H, n, d), np.float32)
    i = np.arange(n, dtype=np.float32)[:, None]
    c = np.arange(d, dtype=np.float32)[None, :]
    for b in range(B):
        for h in range(H):
            X[b, h] = i + c + 100 * h + 1000 * b
    seqlens = np.array([40, 17], np.int32)
    X[1, :, 17:, :] = 1e6  # padding must not enter the mean
    mu = oracle_mod.channel_mean(X, seqlens)
    for b, L in enumerate(seqlens):
        for h in range(H):
            expect = (L - 1) / 2.0 + np.arange(d) + 100 * h + 1000 * b
            np.testing.assert_array_equal(mu[b, h], expect.astype(np.float32))


def test_mean_matches_exact_sum(oracle_mod):
    rng = _rng(1)
    X = (rng.standard_normal((2, 2, 300, 64)) * 3 + 0.25).astype(np.float32)
    mu = oracle_mod.channel_mean(X)
    for b in range(2):
        for h in range(2):
            for c in range(64):
                exact = math.fsum(float(v) for v in X[b, h, :, c]) / 300.0
                assert mu[b, h, c] == np.float32(exact)


# ----------------------------------------------------------------------------- sign + pack

def test_pack_brute_force_and_padding(oracle_mod):
    rng = _rng(2)
    X = rng.standard_normal((2, 2, 70, 64)).astype(np.float32)
    seqlens = np.array([70, 33], np.int32)
    mu = oracle_mod.channel_mean(X, seqlens)
    bits = oracle_mod.sign_pack(X, mu, seqlens)
    assert bits.shape == (2, 2, 70, 2) and bits.dtype == np.uint32
    for b in range(2):
        L = seqlens[b]
        for h in range(2):
            unpacked = ((bits[b, h][:, :, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(70, 64)
            np.testing.assert_array_equal(unpacked[:L], (X[b, h, :L] < mu[b, h][None, :]).astype(np.uint32))
            assert not unpacked[L:].any()


def test_pack_bit_order_probe(oracle_mod):
    n, d = 64, 64
    X = np.zeros((1, 1, n, d), np.float32)
    for t in range(n):
        X[0, 0, t, t] = -1.0          # token t: only channel t below the mean
    mu = np.zeros((1, 1, d), np.float32) - np.float32(1.0 / n) * 0.5  # mean of each column is -1/64
    bits = oracle_mod.sign_pack(X, mu)
    for t in range(n):
        w, j = divmod(t, 32)
        assert bits[0, 0, t, w] == (1 << j) and bits[0, 0, t, 1 - w] == 0


def test_pack_shift_invariance(oracle_mod):
    rng = _rng(3)
    X = rng.integers(-50, 50, size=(1, 2, 90, 64)).astype(np.float32)
    shift = rng.integers(-1000, 1000, size=(1, 2, 1, 64)).astype(np.float32)
    b1 = oracle_mod.sign_pack(X, oracle_mod.channel_mean(X))
    Y = X + shift
    b2 = oracle_mod.sign_pack(Y, oracle_mod.channel_mean(Y))
    np.testing.assert_array_equal(b1, b2)


# ----------------------------------------------------------------------------- score

def test_score_equals_pm1_dot_product(oracle_mod):
    rng = _rng(4)
    B, H, n, d = 2, 3, 50, 64
    Q = rng.standard_normal((B, H, n, d)).astype(np.float32)
    K = rng.standard_normal((B, H, n, d)).astype(np.float32)
    seqlens = np.array([50, 21], np.int32)
    mq, mk = oracle_mod.channel_mean(Q, seqlens), oracle_mod.channel_mean(K, seqlens)
    S = oracle_mod.binary_scores(oracle_mod.sign_pack(Q, mq, seqlens), oracle_mod.sign_pack(K, mk, seqlens), d,
                                 seqlens)
    for b in range(B):
        L = seqlens[b]
        for h in range(H):
            ref = _signs(Q[b, h], mq[b, h], L) @ _signs(K[b, h], mk[b, h], L).T
            np.testing.assert_array_equal(S[b, h, :L, :L], ref)
            assert not S[b, h, L:].any() and not S[b, h, :, L:].any()


def test_score_exhaustive_byte_patterns(oracle_mod):
    # every pair of 8-bit patterns, placed in channels 20..27 (straddling no word)
    # and in channels 28..35 (straddling the two words); the rest of the bits agree.
    pats = np.arange(256, dtype=np.uint64)
    for start in (20, 28):
        full = (pats << np.uint64(start)) | np.uint64(0x5A5A5A5A00000000 & ~(0xFF << start) & 0xFFFFFFFFFFFFFFFF)
        words = np.stack([(full & np.uint64(0xFFFFFFFF)).astype(np.uint32), (full >> np.uint64(32)).astype(np.uint32)],
                         axis=-1).reshape(1, 1, 256, 2)
        S = oracle_mod.binary_scores(words, words, 64)[0, 0]
        pm = 1 - 2 * ((full[:, None] >> np.arange(64, dtype=np.uint64)[None, :]) & np.uint64(1)).astype(np.int64)
        np.testing.assert_array_equal(S, pm @ pm.T)


def test_theorem1_arcsine_law(oracle_mod):
    """BA §2.1 Theorem 1: E[sign q sign k] = (2/pi) arcsin(rho) for zero-mean jointly Gaussian q, k."""
    w = workloads.t5(1024)
    Q, K = w.Q[:1], w.K[:1]
    pi = w.extra["pi"][:1]
    mq, mk = oracle_mod.channel_mean(Q), oracle_mod.channel_mean(K)
    S = oracle_mod.binary_scores(oracle_mod.sign_pack(Q, mq), oracle_mod.sign_pack(K, mk), 64)
    H, n = Q.shape[1], Q.shape[2]
    matched = np.array([S[0, h, pi[0, h, j], j] for h in range(H) for j in range(n)], np.float64) / 64
    expect = 2 / np.pi * np.arcsin(0.6)
    assert abs(matched.mean() - expect) < 0.01, (matched.mean(), expect)
    rng = _rng(5)
    ii, jj = rng.integers(0, n, 20000), rng.integers(0, n, 20000)
    hh = rng.integers(0, H, 20000)
    keep = pi[0, hh, jj] != ii
    indep = S[0, hh[keep], ii[keep], jj[keep]] / 64.0
    assert abs(indep.mean()) < 0.01


# ----------------------------------------------------------------------------- logits / bias

def test_relpos_bias_indexing(oracle_mod):
    gh, gw, prefix = 3, 4, 2
    n, d, H = prefix + gh * gw, 64, 2
    table = np.zeros((H, 2 * gh - 1, 2 * gw - 1), np.float32)
    for h in range(H):
        for a in range(2 * gh - 1):
            for c in range(2 * gw - 1):
                table[h, a, c] = 100 * h + 10 * a + c + 1   # injective, not symmetric
    bits = np.zeros((1, H, n, 2), np.uint32)                # all scores = d = 64
    l = oracle_mod.logits(bits, bits, d, bias=oracle_mod.RelPosBias(table, gh, gw, prefix))
    for h in range(H):
        for i in range(n):
            for j in range(n):
                if i < prefix or j < prefix:
                    b = 0.0
                else:
                    yi, xi = divmod(i - prefix, gw)
                    yj, xj = divmod(j - prefix, gw)
                    b = 100 * h + 10 * (yi - yj + gh - 1) + (xi - xj + gw - 1) + 1
                assert l[0, h, i, j] == np.float32(8.0 + b)


def test_dense_bias_matrix_indexing(oracle_mod):
    # BA §2.3's dense learnable matrix: b_ij = table[h][i][j] for query i, key j
    n, d, H = 9, 64, 2
    table = np.zeros((H, n, n), np.float32)
    for h in range(H):
        for i in range(n):
            for j in range(n):
                table[h, i, j] = 1000 * h + 37 * i + j + 1   # injective, not symmetric
    bits = np.zeros((1, H, n, 2), np.uint32)                 # all scores = d = 64
    l = oracle_mod.logits(bits, bits, d, bias=oracle_mod.DenseBias(table))
    for h in range(H):
        for i in range(n):
            for j in range(n):
                assert l[0, h, i, j] == np.float32(8.0 + 1000 * h + 37 * i + j + 1)


def test_dense_bias_matrix_of_a_relpos_table_matches_the_table(oracle_mod):
    Q, K, V, bias = _small_case(19, with_bias=True)
    B, H, n, d = Q.shape
    Bm = _bias_matrix(bias, H, n).astype(np.float32)
    seq = np.array([40, 23], np.int32)
    for N, mode in ((0, 0), (7, 0), (0, 1), (12, 1)):
        a = oracle_mod.attention(Q, K, V, N=N, mode=mode, seqlens=seq, bias=bias, want_idx=N > 0)
        b = oracle_mod.attention(Q, K, V, N=N, mode=mode, seqlens=seq, bias=oracle_mod.DenseBias(Bm), want_idx=N > 0)
        np.testing.assert_array_equal(a.O, b.O)
        if N > 0:
            np.testing.assert_array_equal(a.idx, b.idx)


def test_logit_is_single_rounding_of_scaled_score_plus_bias(oracle_mod):
    rng = _rng(6)
    H, gh, gw = 2, 5, 5
    n = gh * gw
    bits = rng.integers(0, 2 ** 32, size=(1, H, n, 2), dtype=np.uint64).astype(np.uint32)
    table = rng.standard_normal((H, 9, 9)).astype(np.float32)
    aq = np.array([1.3, 0.7], np.float32)
    ak = np.array([0.9, 2.1], np.float32)
    l = oracle_mod.logits(bits, bits, 64, bias=oracle_mod.RelPosBias(table, gh, gw, 0), alpha_q=aq, alpha_k=ak)
    S = oracle_mod.binary_scores(bits, bits, 64)
    for h in range(H):
        c = np.float32(float(aq[h]) * float(ak[h]) / 8.0)
        for i in range(n):
            yi, xi = divmod(i, gw)
            for j in range(n):
                yj, xj = divmod(j, gw)
                b = table[h, yi - yj + gh - 1, xi - xj + gw - 1]
                exact = float(S[0, h, i, j]) * float(c) + float(b)   # exact in fp64
                assert l[0, h, i, j] == np.float32(exact)


# ----------------------------------------------------------------------------- top-N

def _brute_topn(lrow, L, N):
    keff = L if (N == 0 or N >= L) else N
    order = np.lexsort((np.arange(L), -lrow[:L].astype(np.float64)))
    return np.sort(order[:keff])


@pytest.mark.parametrize("with_bias", [False, True])
def test_topn_matches_full_sort(oracle_mod, with_bias):
    rng = _rng(7 + with_bias)
    B, H, gh, gw, d = 2, 2, 6, 6, 64
    n = gh * gw
    Q = rng.standard_normal((B, H, n, d)).astype(np.float32)
    K = rng.standard_normal((B, H, n, d)).astype(np.float32)
    V = rng.standard_normal((B, H, n, d)).astype(np.float32)
    seqlens = np.array([n, 23], np.int32) if not with_bias else None
    bias = oracle_mod.RelPosBias(rng.standard_normal((H, 11, 11)).astype(np.float32) * 0.1, gh, gw, 0) \
        if with_bias else None
    for N in (1, 5, 9, 22, 30):
        r = oracle_mod.attention(Q, K, V, N=N, seqlens=seqlens, bias=bias, want_idx=True)
        lg = oracle_mod.logits(r.qbits, r.kbits, d, seqlens, bias)
        for b in range(B):
            L = n if seqlens is None else int(seqlens[b])
            for h in range(H):
                for i in range(n):
                    got = r.idx[(b * H + h) * n + i]
                    if i >= L:
                        assert (got == -1).all()
                        continue
                    ref = _brute_topn(lg[b, h, i], L, N)
                    np.testing.assert_array_equal(got[:len(ref)], ref)
                    assert (got[len(ref):] == -1).all()


def test_topn_invariants(oracle_mod):
    rng = _rng(9)
    B, H, n, d = 1, 2, 48, 64
    Q = rng.standard_normal((B, H, n, d)).astype(np.float32)
    K = rng.standard_normal((B, H, n, d)).astype(np.float32)
    V = rng.standard_normal((B, H, n, d)).astype(np.float32)
    prev = None
    for N in range(1, n + 3):
        r = oracle_mod.attention(Q, K, V, N=N, want_idx=True)
        sets = [set(int(x) for x in row if x >= 0) for row in r.idx]
        if N >= n:
            assert all(s == set(range(n)) for s in sets)
        if prev is not None:
            assert all(p <= s for p, s in zip(prev, sets))      # nested
            assert all(len(s) == min(N, n) for s in sets)
        prev = sets
    # without a bias the kept set does not depend on alpha > 0
    a = oracle_mod.attention(Q, K, V, N=7, want_idx=True)
    b = oracle_mod.attention(Q, K, V, N=7, want_idx=True, alpha_q=np.array([3.7, 0.2], np.float32),
                             alpha_k=np.array([0.05, 9.0], np.float32))
    np.testing.assert_array_equal(a.idx, b.idx)
    # N >= L reproduces the dense pass exactly
    dense = oracle_mod.attention(Q, K, V, N=0)
    big = oracle_mod.attention(Q, K, V, N=n + 5)
    np.testing.assert_array_equal(dense.O, big.O)


# ----------------------------------------------------------------------------- softmax / A.V

def _small_case(seed, B=2, H=2, n=40, with_bias=False):
    rng = _rng(seed)
    d = 64
    Q = rng.standard_normal((B, H, n, d)).astype(np.float32)
    K = rng.standard_normal((B, H, n, d)).astype(np.float32)
    V = (rng.standard_normal((B, H, n, d)) * 2).astype(np.float32)
    bias = None
    if with_bias:
        gh, gw = 5, 8
        assert gh * gw == n
        bias = workloads.Bias((rng.standard_normal((H, 9, 15)) * 0.3).astype(np.float32), gh, gw, 0)
    return Q, K, V, bias


def _bias_matrix(bias, H, n):
    Bm = np.zeros((H, n, n), np.float64)
    if bias is None:
        return Bm
    for i in range(bias.prefix, n):
        yi, xi = divmod(i - bias.prefix, bias.gw)
        for j in range(bias.prefix, n):
            yj, xj = divmod(j - bias.prefix, bias.gw)
            Bm[:, i, j] = bias.table[:, yi - yj + bias.gh - 1, xi - xj + bias.gw - 1]
    return Bm


@pytest.mark.parametrize("with_bias", [False, True, "dense"])
def test_dense_equals_independent_numpy_attention(oracle_mod, with_bias):
    Q, K, V, bias = _small_case(10 + (with_bias is True), with_bias=with_bias is True)
    B, H, n, d = Q.shape
    if with_bias == "dense":
        bias = oracle_mod.DenseBias((_rng(29).standard_normal((H, n, n)) * 0.3).astype(np.float32))
        Bm = bias.table.astype(np.float64)
    else:
        Bm = _bias_matrix(bias, H, n)
    r = oracle_mod.attention(Q, K, V, N=0, bias=bias)
    for b in range(B):
        for h in range(H):
            mq = np.float32(np.sum(Q[b, h].astype(np.float64), axis=0) / n)
            mk = np.float32(np.sum(K[b, h].astype(np.float64), axis=0) / n)
            S = (np.where(Q[b, h] < mq, -1.0, 1.0) @ np.where(K[b, h] < mk, -1.0, 1.0).T)
            l = (S * np.float64(np.float32(1 / 8.0)) + Bm[h]).astype(np.float32).astype(np.float64)
            p = np.exp(l - l.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            ref = p @ V[b, h].astype(np.float64)
            assert np.max(np.abs(r.O[b, h] - ref)) <= 1e-12 * np.max(np.abs(V))


@pytest.mark.parametrize("d", [32, 128])
def test_other_head_dims_equal_independent_numpy_attention(oracle_mod, d):
    # the oracle's d is any multiple of 32 (the pages' kernel benchmark uses
    # head dim 128); pinned against the same independent numpy attention
    rng = _rng(40 + d)
    B, H, n = 1, 2, 24
    Q = rng.standard_normal((B, H, n, d)).astype(np.float32)
    K = rng.standard_normal((B, H, n, d)).astype(np.float32)
    V = rng.standard_normal((B, H, n, d)).astype(np.float32)
    r = oracle_mod.attention(Q, K, V, N=0)
    c = np.float64(np.float32(1.0 / math.sqrt(d)))
    for h in range(H):
        mq = np.float32(np.sum(Q[0, h].astype(np.float64), axis=0) / n)
        mk = np.float32(np.sum(K[0, h].astype(np.float64), axis=0) / n)
        S = np.where(Q[0, h] < mq, -1.0, 1.0) @ np.where(K[0, h] < mk, -1.0, 1.0).T
        l = (S * c).astype(np.float32).astype(np.float64)
        p = np.exp(l - l.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        assert np.max(np.abs(r.O[0, h] - p @ V[0, h].astype(np.float64))) <= 1e-12 * np.max(np.abs(V))


def test_probabilities_sum_to_one_and_exp_hamming_form(oracle_mod):
    Q, K, V, _ = _small_case(12)
    B, H, n, d = Q.shape
    for N in (0, 6):
        r = oracle_mod.attention(Q, K, V, N=N, want_probs=True, want_idx=N > 0)
        np.testing.assert_allclose(r.P.sum(axis=1), 1.0, rtol=0, atol=1e-12)
        # BA §2.1: softmax of (d - 2h)c equals softmax of -2hc (shift by the constant d*c)
        ham = np.zeros((B, H, n, n))
        for w in range(2):
            x = r.qbits[..., w][..., :, None] ^ r.kbits[..., w][..., None, :]
            ham += np.unpackbits(x.view(np.uint8).reshape(B, H, n, n, 4), axis=-1).sum(axis=-1)
        l = (-2.0 * ham * 0.125)
        for row in range(B * H * n):
            b, h, i = row // (H * n), (row // n) % H, row % n
            keep = np.arange(n) if N == 0 else r.idx[row]
            e = np.exp(l[b, h, i, keep] - l[b, h, i, keep].max())
            p = np.zeros(n)
            p[keep] = e / e.sum()
            np.testing.assert_allclose(r.P[row], p, rtol=0, atol=1e-13)


def test_padded_batch_equals_sequences_alone(oracle_mod):
    rng = _rng(13)
    H, n, d = 2, 48, 64
    seqlens = np.array([48, 17, 1], np.int32)
    Q = rng.standard_normal((3, H, n, d)).astype(np.float32)
    K = rng.standard_normal((3, H, n, d)).astype(np.float32)
    V = rng.standard_normal((3, H, n, d)).astype(np.float32)
    for N, mode in ((5, 0), (0, 1), (0, 0)):
        full = oracle_mod.attention(Q, K, V, N=N, mode=mode, seqlens=seqlens)
        for b, L in enumerate(seqlens):
            alone = oracle_mod.attention(Q[b:b + 1, :, :L], K[b:b + 1, :, :L], V[b:b + 1, :, :L], N=N, mode=mode)
            np.testing.assert_array_equal(full.O[b, :, :L], alone.O[0])
            assert not full.O[b, :, L:].any()


def test_alpha_scales_the_logits(oracle_mod):
    Q, K, V, _ = _small_case(14, B=1, H=2)
    a1 = oracle_mod.attention(Q, K, V, N=0, alpha_q=np.array([2.0, 4.0], np.float32),
                              alpha_k=np.array([0.5, 0.25], np.float32))
    a0 = oracle_mod.attention(Q, K, V, N=0)
    np.testing.assert_array_equal(a1.O, a0.O)         # alpha_q * alpha_k = 1 -> same c
    a2 = oracle_mod.attention(Q, K, V, N=0, alpha_q=np.array([3.0, 3.0], np.float32))
    assert np.max(np.abs(a2.O - a0.O)) > 1e-3


# ----------------------------------------------------------------------------- quantization

def test_v_quant_reconstruction(oracle_mod):
    w = workloads.deit()
    V = w.V[:2]
    Vq, s = oracle_mod.v_quant(V)
    assert Vq.dtype == np.int8 and (np.abs(Vq.astype(np.int32)) <= 127).all()
    rec = Vq.astype(np.float64) * s[:, :, None, :].astype(np.float64)
    # rint of the fp32 quotient V/s, whose rounding error is at most 127 * 2^-24 in units of s
    assert (np.abs(rec - V) <= s[:, :, None, :] * (0.5 + 127 * 2.0 ** -24)).all()
    # the channel's absmax maps to +-127
    assert (np.abs(Vq).max(axis=2) == 127).all()


def test_quant_codes_and_output_bounds(oracle_mod):
    Q, K, V, bias = _small_case(15, with_bias=True)
    B, H, n, d = Q.shape
    V[0, 1, :, 5] *= 20.0   # an outlier channel
    for N in (0, 9):
        rq = oracle_mod.attention(Q, K, V, N=N, mode=1, bias=bias, want_codes=True, want_probs=True)
        rf = oracle_mod.attention(Q, K, V, N=N, mode=0, bias=bias)
        assert np.all(np.abs(rq.Aq / 255.0 - rq.P) <= 0.5 / 255 + 1e-15)
        s = rq.vscale.astype(np.float64)
        for row in range(B * H * n):
            b, h, i = row // (H * n), (row // n) % H, row % n
            p = rq.P[row]
            diff = np.abs(rq.O.reshape(-1, d)[row] - rf.O.reshape(-1, d)[row])
            kept = p > 0
            bound = (0.5 / 255) * (np.abs(V[b, h][kept]) + s[b, h] / 2).sum(axis=0) \
                + (p[kept][:, None] * s[b, h][None, :] / 2).sum(axis=0)
            assert np.all(diff <= bound + 1e-12)


def test_one_key_row_gives_full_code(oracle_mod):
    rng = _rng(16)
    Q = rng.standard_normal((2, 1, 8, 64)).astype(np.float32)
    K = rng.standard_normal((2, 1, 8, 64)).astype(np.float32)
    V = rng.standard_normal((2, 1, 8, 64)).astype(np.float32)
    r = oracle_mod.attention(Q, K, V, N=1, mode=1, want_codes=True)
    assert (r.Aq.max(axis=1) == 255).all() and ((r.Aq > 0).sum(axis=1) == 1).all()
    r = oracle_mod.attention(Q, K, V, N=0, mode=1, seqlens=np.array([1, 8], np.int32), want_codes=True)
    assert r.Aq[0, 0] == 255 and (r.Aq[1:8] == 0).all()
    np.testing.assert_allclose(r.O[0, 0, 0], r.Vq[0, 0, 0].astype(np.float64) * r.vscale[0, 0].astype(np.float64),
                               rtol=1e-12)


# ----------------------------------------------------------------------------- dense comparison mode

def test_standard_dense_attention(oracle_mod):
    Q, K, V, bias = _small_case(17, with_bias=True)
    B, H, n, d = Q.shape
    O = oracle_mod.dense_attention(Q, K, V, bias=bias)
    Bm = _bias_matrix(bias, H, n)
    for b in range(B):
        for h in range(H):
            l = Q[b, h].astype(np.float64) @ K[b, h].astype(np.float64).T / 8.0 + Bm[h]
            p = np.exp(l - l.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            np.testing.assert_allclose(O[b, h], p @ V[b, h].astype(np.float64), rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------- rounding ties (constructed)

def test_v_quant_rounds_half_to_even(oracle_mod):
    """int8 V takes rint (half to even) of V / s: with absmax 127 the scale is
    exactly 1 (and 0.5 for absmax 63.5), so halves land exactly on ties and a
    half-away or floor(x + 0.5) rounding would give other codes."""
    d, n = 64, 12
    V = np.zeros((1, 1, n, d), np.float32)
    V[0, 0, :, 0] = [127.0, 0.5, -0.5, 1.5, -1.5, 2.5, -2.5, 3.5, -3.5, 126.5, -126.5, 0.0]
    V[0, 0, :, 1] = [63.5, 0.25, -0.25, 0.75, -0.75, 1.25, -1.25, 31.75, -31.75, 0.0, 0.0, 0.0]
    V[0, 0, :, 2:] = 1.0                       # absmax 1: scale 1/127 (no ties asserted there)
    Vq, sc = oracle_mod.v_quant(V)
    assert sc[0, 0, 0] == np.float32(1.0) and sc[0, 0, 1] == np.float32(0.5)
    np.testing.assert_array_equal(Vq[0, 0, :, 0], [127, 0, 0, 2, -2, 2, -2, 4, -4, 126, -126, 0])
    np.testing.assert_array_equal(Vq[0, 0, :, 1], [127, 0, 0, 2, -2, 2, -2, 64, -64, 0, 0, 0])


@pytest.mark.parametrize("L,code", [(6, 43), (30, 9), (102, 3), (510, 1), (2, 128), (10, 26)])
def test_attention_codes_round_half_up(oracle_mod, L, code):
    """A_q = floor(255 p + 0.5): a row of L equal logits has p = 1/L, and for
    L in {6, 30, 102, 510} 255/L is exactly k + 1/2 with k even, where rint
    (half to even) and floor(255 p) give k, and floor(255 p + 0.5) gives k + 1.
    Identical Q rows and identical K rows make every score d and every logit equal."""
    n, d = 512, 64
    rng = _rng(77)
    q = rng.standard_normal(d).astype(np.float32)
    k = rng.standard_normal(d).astype(np.float32)
    Q = np.broadcast_to(q, (1, 1, n, d)).copy()
    K = np.broadcast_to(k, (1, 1, n, d)).copy()
    V = rng.standard_normal((1, 1, n, d)).astype(np.float32)
    res = oracle_mod.attention(Q, K, V, N=0, mode=1, seqlens=np.array([L], np.int32), want_codes=True,
                               want_probs=True)
    A = res.Aq.reshape(n, n)
    np.testing.assert_array_equal(A[:L, :L], np.full((L, L), code, np.uint8))
    assert not A[:, L:].any() and not A[L:].any()
    assert 255.0 / L == code - 0.5


# ----------------------------------------------------------------------------- 4-bit V (mode 2)

def test_v_quant4_rounds_half_to_even_and_reconstructs(oracle_mod):
    """4-bit V: absmax 7 gives scale exactly 1, so halves are exact ties: rint
    (half to even), not half-away or floor(x + 0.5); every value reconstructs
    within s/2, and the codes stay in [-7, 7]."""
    n, d = 10, 64
    V = _rng(41).standard_normal((2, 3, n, d)).astype(np.float32)
    V[0, 0, :, 0] = [7.0, 0.5, -0.5, 1.5, -1.5, 2.5, -2.5, 6.5, -6.5, 0.0]
    Vq, sc = oracle_mod.v_quant(V, bits=4)
    assert sc[0, 0, 0] == np.float32(1.0)
    np.testing.assert_array_equal(Vq[0, 0, :, 0], [7, 0, 0, 2, -2, 2, -2, 6, -6, 0])
    assert np.abs(Vq).max() <= 7
    err = np.abs(Vq.astype(np.float64) * sc[:, :, None, :] - V)
    assert np.all(err <= sc[:, :, None, :] * (0.5 + 1e-6))
    # the scale is absmax / 7 per (batch, head, channel)
    np.testing.assert_array_equal(sc, (np.abs(V).max(axis=2) / np.float32(7.0)).astype(np.float32))


def test_u8i4_output_equals_independent_numpy(oracle_mod):
    """Mode 2 (uint8 A x 4-bit V) against numpy: p from an independent dense
    attention, A_q = floor(255 p + 0.5), V_q = clip(rint(V / (absmax / 7)), -7, 7),
    O = (A_q @ V_q) * s / 255."""
    Q, K, V, bias = _small_case(12, with_bias=False)
    B, H, n, d = Q.shape
    r = oracle_mod.attention(Q, K, V, N=0, mode=2)
    for b in range(B):
        for h in range(H):
            mq = np.float32(np.sum(Q[b, h].astype(np.float64), axis=0) / n)
            mk = np.float32(np.sum(K[b, h].astype(np.float64), axis=0) / n)
            S = (np.where(Q[b, h] < mq, -1.0, 1.0) @ np.where(K[b, h] < mk, -1.0, 1.0).T)
            l = (S * np.float64(np.float32(1 / 8.0))).astype(np.float32).astype(np.float64)
            p = np.exp(l - l.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            A = np.floor(255.0 * p + 0.5)
            s4 = (np.abs(V[b, h]).max(axis=0) / np.float32(7.0)).astype(np.float32)
            Vq = np.clip(np.rint(V[b, h] / s4), -7, 7)
            ref = (A @ Vq) * s4.astype(np.float64) / 255.0
            assert np.max(np.abs(r.O[b, h] - ref)) <= 1e-9 * np.max(np.abs(V))
    # and it stays within the closed-form bound of the float output
    rf = oracle_mod.attention(Q, K, V, N=0, mode=0, want_probs=True)
    s4 = (np.abs(V).max(axis=2) / 7.0)
    bound = (0.5 / 255) * np.abs(V).sum(axis=2, keepdims=True) + 0.5 * s4[:, :, None, :] * 1.0
    assert np.all(np.abs(r.O - rf.O) <= bound + 1e-9)


# ----------------------------------------------------------------------------- the projection before the path

def _np_pack_lsb(mask):
    """[..., d] bool -> [..., d/32] uint32, channel 32w + j at bit j of word w (numpy, no oracle code)."""
    d = mask.shape[-1]
    m = mask.reshape(mask.shape[:-1] + (d // 32, 32)).astype(np.uint64)
    return (m << np.arange(32, dtype=np.uint64)).sum(axis=-1).astype(np.uint32)


@pytest.mark.parametrize("seqlens", [None, [70, 33, 1]])
def test_qkv_projection_against_independent_numpy(oracle_mod, seqlens):
    """Projection, means and sign bits of the step before the path, against numpy:
    P = X W^T in fp64 (einsum), the mean over the valid tokens, and the LSB-first packing
    of P < mu; tokens past L carry zero words."""
    rng = np.random.default_rng(41)
    B, n, Dm, H, d = 3, 70, 192, 2, 64
    X = workloads.bf16_round(rng.standard_normal((B, n, Dm)).astype(np.float32))
    W = workloads.bf16_round((rng.standard_normal((3 * H * d, Dm)) * 0.05).astype(np.float32))
    sl = None if seqlens is None else np.array(seqlens, np.int32)
    Q, K, V, mq, mk, qb, kb = oracle_mod.qkv_project(X, W, H, d, sl)
    P = np.einsum("bik,ok->bio", X.astype(np.float64), W.astype(np.float64)).reshape(B, n, 3, H, d)
    P = P.transpose(2, 0, 3, 1, 4)  # [t][b][h][i][c]
    for t, got in enumerate((Q, K, V)):
        np.testing.assert_allclose(got, P[t], rtol=0, atol=1e-12)
    L = np.full(B, n) if sl is None else sl
    for t, (mu, bits) in enumerate(((mq, qb), (mk, kb))):
        ref_mu = np.stack([P[t][b, :, :L[b]].mean(axis=1) for b in range(B)]).astype(np.float32)
        np.testing.assert_array_equal(mu, ref_mu)
        mask = P[t] < mu[:, :, None, :].astype(np.float64)
        for b in range(B):
            mask[b, :, L[b]:] = False
        np.testing.assert_array_equal(bits, _np_pack_lsb(mask))


def test_qkv_means_are_the_projected_token_mean(oracle_mod):
    """The mean of a linear map's outputs is the map of the mean input: mu_t = mean_i(X_i) W_t^T.
    This is the identity the fused projection uses to binarize in its epilogue; in fp64 both
    sides agree to rounding, so the fp32 means agree to one unit in the last place."""
    rng = np.random.default_rng(43)
    B, n, Dm, H, d = 2, 197, 256, 3, 64
    X = workloads.bf16_round(rng.standard_normal((B, n, Dm)).astype(np.float32))
    W = workloads.bf16_round((rng.standard_normal((3 * H * d, Dm)) * 0.05).astype(np.float32))
    sl = np.array([197, 120], np.int32)
    _, _, _, mq, mk, _, _ = oracle_mod.qkv_project(X, W, H, d, sl)
    for b in range(B):
        xbar = X[b, :sl[b]].astype(np.float64).mean(axis=0)
        lin = (W.astype(np.float64) @ xbar).reshape(3, H, d)
        for t, mu in enumerate((mq, mk)):
            np.testing.assert_array_max_ulp(mu[b], lin[t].astype(np.float32), maxulp=1)

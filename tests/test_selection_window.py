"""The top-N threshold with a bias lies in [fmaf(s_N, c, b_min), fmaf(s_N, c, b_max)],
where s_N is the score level that holds rank N.

At least N keys score s_N or more, so their logits reach the low end. Fewer than
N score above s_N, and only those can pass the high end (fmaf rounding is
monotone).  The fused kernel searches only that window.  Checked here against
the oracle's full sort, on random rows and on rows with many ties.
"""
import numpy as np
import pytest


def _fmaf(x, y, z):
    # x*y + z is exact in fp64 for these operands (|s| <= 64 integer, fp32 c and b
    # of nearby magnitude), so one fp32 rounding of it is fmaf
    return np.float32(np.float64(x) * np.float64(y) + np.float64(z))


@pytest.mark.parametrize("seed,levels", [(0, None), (1, None), (2, 5)])
def test_threshold_lies_in_the_score_level_window(oracle_mod, seed, levels):
    rng = np.random.default_rng(300 + seed)
    H, gh, gw = 2, 6, 6
    n, d = gh * gw, 64
    Q = rng.standard_normal((1, H, n, d)).astype(np.float32)
    K = rng.standard_normal((1, H, n, d)).astype(np.float32)
    if levels is None:
        table = (rng.standard_normal((H, 2 * gh - 1, 2 * gw - 1)) * 0.3).astype(np.float32)
    else:   # few distinct bias values: many exact logit ties
        table = (rng.integers(-2, 3, size=(H, 2 * gh - 1, 2 * gw - 1)) * 0.25).astype(np.float32)
    bias = oracle_mod.RelPosBias(table, gh, gw, 0)
    qb = oracle_mod.sign_pack(Q, oracle_mod.channel_mean(Q))
    kb = oracle_mod.sign_pack(K, oracle_mod.channel_mean(K))
    S = oracle_mod.binary_scores(qb, kb, d)
    Lg = oracle_mod.logits(qb, kb, d, bias=bias)
    c = np.float32(1.0 / 8.0)
    for h in range(H):
        bmin, bmax = float(table[h].min()), float(table[h].max())
        for i in range(n):
            for N in (1, 5, 17, n - 1):
                F = np.sort(Lg[0, h, i])[::-1][N - 1]          # the N-th largest logit
                sN = np.sort(S[0, h, i])[::-1][N - 1]          # the level holding rank N
                lo, hi = _fmaf(sN, c, bmin), _fmaf(sN, c, bmax)
                assert lo <= F <= hi, (h, i, N, lo, F, hi)
                # and fewer than N logits lie above the window
                assert int(np.sum(Lg[0, h, i] > hi)) < N

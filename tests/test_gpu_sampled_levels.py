"""GPU parity of top-N with a bias on long rows (64 tiles of 64 keys or more),
where the fused kernel's first level pass reads one tile in eight and each row
brackets its threshold from that sample; the float-binned pass verifies the
bracket with exact counts and a missed bracket reruns the level pass over every
tile.  The kept sets must be the oracle's bit for bit whether the sample is
representative (random grids) or built to mislead it (every sampled key scores +d,
or -d, while the threshold lies elsewhere), and O must stay within its bars.
"""
import numpy as np
import pytest

import workloads

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import binarized_qk_sparse_b200 as had  # noqa: E402

STRIDE = 8  # one sampled tile in eight: tile 8u + u % 8


def _sampled_tiles(ntiles):
    return [8 * u + (u % 8) for u in range(ntiles) if 8 * u + (u % 8) < ntiles]


def _inputs(w):
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).cuda()  # noqa: E731
    seq = None if w.seqlens is None else torch.from_numpy(w.seqlens).cuda()
    bias = had.RelPosBias(torch.from_numpy(w.bias.table).cuda(), w.bias.gh, w.bias.gw, w.bias.prefix)
    return dev(w.Q), dev(w.K), dev(w.V), seq, bias


def _obias(oracle_mod, w):
    return oracle_mod.RelPosBias(w.bias.table, w.bias.gh, w.bias.gw, w.bias.prefix)


def _rows(w, per_head, seed):
    rng = np.random.default_rng(seed)
    out = []
    for bh in range(w.B * w.H):
        L = w.n if w.seqlens is None else int(w.seqlens[bh // w.H])
        out.extend(bh * w.n + int(i) for i in sorted(rng.choice(L, size=min(per_head, L), replace=False)))
    return np.array(out, np.int64)


def _check(oracle_mod, w, N, rows, modes=(0, 1)):
    Q, K, V, seq, bias = _inputs(w)
    ob = _obias(oracle_mod, w)
    rows_t = torch.from_numpy(rows).cuda()
    idx = had.had_topn_indices(Q, K, N, seq, bias).reshape(-1, N)[rows_t].cpu().numpy()
    ref_i = oracle_mod.attention(w.Q, w.K, w.V, N=N, seqlens=w.seqlens, bias=ob, rows=rows, want_idx=True)
    np.testing.assert_array_equal(idx, ref_i.idx)
    vmax = float(np.max(np.abs(w.V)))
    for mode in modes:
        name = "float" if mode == 0 else "u8i8"
        O = had.had_attention(Q, K, V, N=N, mode=name, seqlens=seq, bias=bias).reshape(-1, w.d)[rows_t]
        ref = ref_i.O if mode == 0 else oracle_mod.attention(w.Q, w.K, w.V, N=N, mode=1, seqlens=w.seqlens,
                                                             bias=ob, rows=rows).O
        assert np.max(np.abs(O.float().cpu().numpy() - ref)) <= 1e-2 * vmax + mode * vmax / 255, name


@pytest.mark.parametrize("gh,gw,prefix,seqlens", [
    (64, 128, 0, [8192, 5000]),   # per-warp bias windows; a ragged second sequence (79 tiles)
    (64, 96, 1, None),            # a class token: extended-table gathers (97 tiles)
])
def test_sampled_bracket_on_random_grids(oracle_mod, gh, gw, prefix, seqlens):
    B = 1 if seqlens is None else len(seqlens)
    w = workloads.grid(B, 2, gh, gw, prefix, seqlens, seed=51)
    for N in (w.n // 8, 100):
        _check(oracle_mod, w, N, _rows(w, 48, 3))


@pytest.mark.parametrize("sign", [1.0, -1.0])
def test_misleading_sample_falls_back_to_every_tile(oracle_mod, sign):
    """Identical query rows sign-bin to q~ = +1, so a key's score is d minus twice
    its count of channels below the key mean.  The keys of the sampled tiles are set
    to +4 (every channel above the mean: score +d) or -4 (score -d), the others drawn
    from N(0, 1).  sign = +1: the sample puts the threshold at the top level, but only
    1/8 of the keys are there and N asks for more, so the rank falls below the bracket
    (bin 0).  sign = -1: the sample puts it at the bottom level, and more than N keys lie
    above the bracket (bin 127).  Either way the kernel must count every tile again."""
    gh, gw = 64, 128
    seqlens = np.array([8192, 4500], np.int32)
    w = workloads.grid(2, 2, gh, gw, 0, seqlens, seed=57)
    rng = np.random.default_rng(58)
    Q = np.repeat(rng.standard_normal((2, 2, 1, 64), dtype=np.float32), w.n, axis=2)
    K = rng.standard_normal((2, 2, w.n, 64), dtype=np.float32)
    for b, L in enumerate(seqlens):
        for t in _sampled_tiles((int(L) + 63) // 64):
            K[b, :, 64 * t:64 * (t + 1)] = 4.0 * sign
    w = workloads.Workload(w.name + f"_mislead{int(sign)}", w.B, w.H, w.n, w.d, w.dtype, workloads.bf16_round(Q),
                           workloads.bf16_round(K), w.V, w.seqlens, w.bias, w.passes, w.seed, w.recipe)
    _check(oracle_mod, w, 2000, _rows(w, 32, 5), modes=(0,))

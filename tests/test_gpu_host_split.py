"""had_attention_host on sequences too long for one chunk: with chunk_b = 0 the
library splits each sequence into equal groups of heads, computes consecutive
chunks on two streams, and copies each group's O back on its own.  Every (b, h)
runs the same kernels as in had_attention, so O must be bit-identical to the
device call, with a relative-position bias table and per-head alphas offset to
each group's heads.
"""
import numpy as np
import pytest

import workloads

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import binarized_qk_sparse_b200 as had  # noqa: E402


@pytest.mark.parametrize("N,mode", [(1920, "float"), (0, "u8i8")])
def test_head_groups_match_the_device_call(N, mode):
    # B2 H8 n16384 (128 x 128 patches): 100 MB of inputs per sequence, split into two groups of 4 heads
    w = workloads.grid(2, 8, 128, 128, 0, seqlens=[16384, 12000], seed=41)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16)  # noqa: E731
    hQ, hK, hV = (dev(x).pin_memory() for x in (w.Q, w.K, w.V))
    Q, K, V = hQ.cuda(), hK.cuda(), hV.cuda()
    seq = torch.from_numpy(w.seqlens)
    table = torch.from_numpy(w.bias.table)
    alpha_q = torch.linspace(0.8, 1.2, 8)
    alpha_k = torch.linspace(1.1, 0.9, 8)
    ref = had.had_attention(Q, K, V, N=N, mode=mode, seqlens=seq.cuda(),
                            bias=had.RelPosBias(table.cuda(), 128, 128, 0),
                            alpha_q=alpha_q, alpha_k=alpha_k).cpu()
    got = had.had_attention_host(hQ, hK, hV, N=N, mode=mode, seqlens=seq,
                                 bias=had.RelPosBias(table.pin_memory(), 128, 128, 0),
                                 alpha_q=alpha_q, alpha_k=alpha_k)
    assert had.had_get_device_status() == had.HAD_OK
    assert torch.equal(got, ref)
    assert got[1, :, 12000:].abs().max().item() == 0.0  # rows past L

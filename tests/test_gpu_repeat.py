"""Repeated calls give the same output bit for bit.

Top-N with a bias keeps each row's final radix bin as a list of recorded keys,
filled by the row's two threads in whatever order they reach them; the weights
of the kept keys are then summed over that list.  The list is put in key order
before any sum, so the same inputs give the same O on every call, in every
mode.  Each case runs three times (with the launches of other cases between
them) and compares the outputs with torch.equal.
"""
import numpy as np
import pytest

import workloads

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import binarized_qk_sparse_b200 as had  # noqa: E402


def _dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).cuda()


@pytest.mark.parametrize("B,H,gh,gw,prefix,seqlens,N,mode", [
    (2, 2, 14, 14, 1, [197, 150], 40, "float"),      # DeiT rows, ragged, top-40 float
    (2, 2, 14, 14, 1, None, 24, "float"),            # top-24 float
    (1, 2, 48, 48, 0, None, 288, "float"),           # 2304 keys: the sampled level pass
    (2, 2, 14, 14, 1, [197, 120], 40, "u8i8"),       # top-40, uint8 A x int8 V
    (2, 2, 14, 14, 1, None, 0, "u8i4"),              # dense, 4-bit V
])
def test_same_output_on_every_call(B, H, gh, gw, prefix, seqlens, N, mode):
    w = workloads.grid(B, H, gh, gw, prefix, seqlens, seed=31)
    Q, K, V = _dev(w.Q), _dev(w.K), _dev(w.V)
    sd = None if w.seqlens is None else torch.from_numpy(w.seqlens).cuda()
    bias = had.RelPosBias(torch.from_numpy(w.bias.table).cuda(), w.bias.gh, w.bias.gw, w.bias.prefix)
    outs = []
    for rep in range(3):
        outs.append(had.had_attention(Q, K, V, N=N, mode=mode, seqlens=sd, bias=bias, out_dtype=torch.float32))
        # other launches in between, so that the runs do not see the same timing
        had.had_attention(Q, K, V, N=max(1, N // 2), mode="float", seqlens=sd, bias=bias)
    torch.cuda.synchronize()
    assert had.had_get_device_status() == had.HAD_OK
    for o in outs[1:]:
        assert torch.equal(o, outs[0])

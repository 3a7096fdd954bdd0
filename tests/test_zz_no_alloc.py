"""had_binarize_pack_noalloc against had_binarize_pack (the workspace entry point).

The no-allocation variant serves callers that cannot allocate device memory
when they call into the library, so it keeps its scratch in a fixed array
inside the library.  Its results must equal the workspace entry point's
bit for bit (packed sign bits and fp32 channel means, the tolerance the other
pack tests use), on two calls in a row -- the second one runs over the scratch
the first one left behind.  This file is collected last on purpose.
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


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    bert = workloads.bert()       # padded sequences (seqlens) ...
    tiny = workloads.tiny()       # ... then fp32 inputs of another shape
    cases = [(_dev(bert, bert.K), torch.from_numpy(bert.seqlens).cuda()),
             (_dev(tiny, tiny.Q), None),
             (_dev(bert, bert.Q), torch.from_numpy(bert.seqlens).cuda())]
    for X, seq in cases:
        bits_ref, mu_ref = had.had_binarize_pack(X, seq)
        bits, mu = had.had_binarize_pack_noalloc(X, seq)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(bits.cpu().numpy(), bits_ref.cpu().numpy())
        np.testing.assert_array_equal(mu.cpu().numpy(), mu_ref.cpu().numpy())
    assert had.had_get_device_status() == had.HAD_OK


def test_noalloc_rejects_shapes_beyond_its_scratch():
    X = torch.zeros((1, 64, 16384, 64), dtype=torch.bfloat16, device="cuda")   # 64 * 256 chunks > 8192
    with pytest.raises(had.HadError) as e:
        had.had_binarize_pack_noalloc(X)
    assert e.value.status == had.HAD_ERR_UNSUPPORTED
    assert b"static scratch limit" in had.lib().had_last_cuda_error()

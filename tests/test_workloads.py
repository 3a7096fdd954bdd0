"""The seeded input generators that both sides use: shapes, dtypes, recipes and
reproducibility (the same call gives the same arrays)."""
import numpy as np
import pytest

import workloads


@pytest.mark.parametrize("name", ["tiny", "deit", "bert", "t5_128", "t5_256", "t5_512", "t5_1024",
                                  "deit_dense_bias"])
def test_generators_are_seeded_and_shaped(name):
    a, b = workloads.by_name(name), workloads.by_name(name)
    for x, y in ((a.Q, b.Q), (a.K, b.K), (a.V, b.V)):
        assert x.shape == (a.B, a.H, a.n, a.d) and x.dtype == np.float32
        np.testing.assert_array_equal(x, y)
        if a.dtype == "bf16":   # bf16-valued fp32: the low 16 bits are zero
            assert not np.any(x.view(np.uint32) & 0xFFFF)
    if a.seqlens is not None:
        np.testing.assert_array_equal(a.seqlens, b.seqlens)
        assert a.seqlens.min() >= 1 and a.seqlens.max() <= a.n
    if isinstance(a.bias, workloads.Bias):
        assert a.bias.table.shape == (a.H, 2 * a.bias.gh - 1, 2 * a.bias.gw - 1)
        assert a.bias.gh * a.bias.gw + a.bias.prefix == a.n
    elif isinstance(a.bias, workloads.DenseBias):
        assert a.bias.table.shape == (a.H, a.n, a.n)
    assert a.recipe


def test_dense_bias_workload_reuses_the_deit_tensors():
    d, m = workloads.by_name("deit"), workloads.by_name("deit_dense_bias")
    np.testing.assert_array_equal(d.Q, m.Q)
    np.testing.assert_array_equal(d.V, m.V)
    assert abs(float(np.std(m.bias.table)) - 0.1) < 0.005   # ~N(0, 0.1)

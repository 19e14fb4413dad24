"""The threaded driver of the oracle quantize runs the same C steps over
disjoint row ranges; it must give the sequential oracle's result bit for bit
(codes, scale bytes including padding, tensor scale, status)."""
import numpy as np
import pytest
import torch

import oracle


def _same(x, layout, threads):
    st1, r1 = oracle.quantize(x, layout)
    st2, r2 = oracle.quantize_parallel(x, layout, threads=threads)
    assert st1 == st2
    if st1 == oracle.OK:
        assert np.float32(r1.g) == np.float32(r2.g)
        assert np.array_equal(r1.codes, r2.codes)
        assert np.array_equal(r1.scales, r2.scales)


@pytest.mark.parametrize("rows,cols", [(1, 16), (127, 48), (128, 64), (129, 80), (300, 1040),
                                       (1000, 32), (2049, 272)])
@pytest.mark.parametrize("layout", [oracle.SF_SWIZZLED, oracle.SF_LINEAR])
@pytest.mark.parametrize("threads", [1, 3, 8])
def test_parallel_equals_sequential(rows, cols, layout, threads):
    g = torch.Generator().manual_seed(rows * 7 + cols)
    x = torch.randn(rows, cols, generator=g) * torch.exp2(
        torch.randint(-8, 8, (rows, 1), generator=g).float())
    _same(x.to(torch.bfloat16), layout, threads)


def test_parallel_special_tensors():
    z = torch.zeros(300, 64, dtype=torch.bfloat16)
    _same(z, oracle.SF_SWIZZLED, 4)
    st, r = oracle.quantize_parallel(z, threads=4)
    assert st == oracle.OK and r.g == 1.0
    x = torch.randn(400, 64).to(torch.bfloat16)
    x[333, 5] = float("nan")                      # in the last range only
    assert oracle.quantize_parallel(x, threads=4)[0] == oracle.ERR_NONFINITE
    tiny = torch.full((256, 32), 1e-37, dtype=torch.bfloat16)
    assert oracle.quantize_parallel(tiny, threads=2)[0] == oracle.ERR_RANGE
    assert oracle.quantize_parallel(torch.zeros(0, 16, dtype=torch.bfloat16))[0] == oracle.OK


def test_parallel_amax_and_gemm_reference():
    g = torch.Generator().manual_seed(99)
    x = (torch.randn(700, 96, generator=g) * 3).to(torch.bfloat16)
    assert oracle.tensor_amax_parallel(x, threads=5) == oracle.tensor_amax(x)
    st, qa = oracle.quantize(x[:37])
    st2, qw = oracle.quantize(x[100:300])
    rng = np.random.default_rng(0)
    i, j = rng.integers(0, 37, 501), rng.integers(0, 200, 501)
    r1, a1 = oracle.gemm_ref(qa, qw, i, j)
    r2, a2 = oracle.gemm_ref_parallel(qa, qw, i, j, threads=7)
    assert np.array_equal(r1, r2) and np.array_equal(a1, a2)

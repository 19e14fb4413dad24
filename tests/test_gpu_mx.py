"""GPU parity of MXFP4 quantize / dequantize (block 32, UE8M0 scales; the
format the pages compare NVFP4 with) against the oracle: codes and scales
bit for bit, dequantized BF16 bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_block_scaled_22_b200 import binding as nb
from nvfp4_block_scaled_22_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    nb.lib()
    yield
    assert nb.nvfp4_check_status() == 0


def _rand(rows, cols, seed, scale=1.0, outliers=0.01):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, cols, generator=g) * scale
    n = x.numel()
    idx = torch.randint(0, n, (max(1, int(outliers * n)),), generator=g)
    x.view(-1)[idx] *= 40
    return x.to(torch.bfloat16)


def _check(x_cpu, layout, what=""):
    q = nb.nvfp4_quantize_mx(x_cpu.to(DEV), layout=layout)
    st, ref = oracle.quantize_mx(x_cpu, layout)
    assert st == oracle.OK
    assert nb.nvfp4_check_status() == 0
    torch.cuda.synchronize()
    assert np.array_equal(q.scales.cpu().numpy(), ref.scales), f"{what}: scales"
    assert np.array_equal(q.codes.cpu().numpy(), ref.codes), f"{what}: codes"
    y = nb.nvfp4_dequantize_mx(q)
    assert np.array_equal(y.cpu().view(torch.int16).numpy().view(np.uint16), ref.dequantize()), \
        f"{what}: dequantize"
    return q, ref


@pytest.mark.parametrize("rows,cols", [(1, 32), (7, 96), (129, 160), (300, 1056), (64, 8192), (1000, 4096)])
@pytest.mark.parametrize("layout", [nb.SF_SWIZZLED, nb.SF_LINEAR])
def test_ragged_shapes(rows, cols, layout):
    _check(_rand(rows, cols, rows + cols), layout, f"{rows}x{cols}")


def test_dynamic_range_zero_blocks_subnormals():
    x = _rand(128, 256, 3)
    x[0] = 0.0
    x[1, :32] = 2.0 ** -133                 # BF16 subnormals only
    x[2, :64] *= 1e30
    x[3, :32] *= 1e-30
    _check(x, nb.SF_SWIZZLED, "range")
    _check(x, nb.SF_LINEAR, "range linear")


def test_nonfinite_is_reported():
    x = _rand(16, 64, 4)
    x[2, 3] = float("nan")
    nb.nvfp4_quantize_mx(x.to(DEV))
    assert nb.nvfp4_check_status() == 4


def test_sweep_full_size_compare():
    x = inputs.sweep_tensor(1 << 24, device=DEV)
    _check(x.cpu(), nb.SF_SWIZZLED, "sweep 2^24")


def _gemm_check(m, n, k, seed):
    from tests.gpu_util import bf16_to_f64, gemm_tolerance
    a = _rand(m, k, seed)
    w = _rand(n, k, seed + 1, 0.05)
    qa = nb.nvfp4_quantize_mx(a.to(DEV))
    qw = nb.nvfp4_quantize_mx(w.to(DEV))
    d = nb.nvfp4_gemm_mx(qa, qw)
    assert nb.nvfp4_check_status() == 0
    _, ra = oracle.quantize_mx(a)
    _, rw = oracle.quantize_mx(w)
    rng = np.random.default_rng(seed)
    cnt = min(m * n, 2000)
    ii, jj = rng.integers(0, m, cnt), rng.integers(0, n, cnt)
    ref, ab = oracle.gemm_ref_mx(ra, rw, ii, jj)
    got = bf16_to_f64(d)[ii, jj]
    bad = np.abs(got - ref) > gemm_tolerance(ref, ab)
    assert not bad.any(), f"{bad.sum()} of {cnt} outside tolerance, e.g. got {got[bad][:4]} ref {ref[bad][:4]}"


@pytest.mark.parametrize("m,n,k", [(128, 256, 256), (640, 384, 192), (257, 257, 320), (16, 1024, 2048),
                                   (1024, 2048, 4096)])
def test_gemm(m, n, k):
    _gemm_check(m, n, k, m + n + k)

"""GPU parity of column-wise quantization (NVFP4 of x^T read from a
row-major x) against the oracle applied to an explicit BF16 x^T: codes,
scales and tensor scale bit for bit, with and without the 16x16 random
Hadamard transform, in both scale layouts."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_block_scaled_22_b200 import binding as nb
from nvfp4_block_scaled_22_b200 import inputs
from tests.gpu_util import assert_quantized_equal, bf16_to_f64, gemm_tolerance

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


def _check(x_cpu, layout=nb.SF_SWIZZLED, mask=None, what=""):
    q = nb.nvfp4_quantize_t(x_cpu.to(DEV), layout=layout, sign_mask=mask)
    xt = x_cpu.t().contiguous()
    st, ref = oracle.quantize(xt, layout) if mask is None else oracle.quantize_rht(xt, mask, layout)
    assert st == oracle.OK
    assert nb.nvfp4_check_status() == 0
    assert_quantized_equal(q, ref, what)
    return q, ref


SHAPES = [(16, 8), (48, 24), (80, 136), (64, 128), (1040, 296), (4096, 1000), (208, 2056)]


@pytest.mark.parametrize("rows,cols", SHAPES)
@pytest.mark.parametrize("layout", [nb.SF_SWIZZLED, nb.SF_LINEAR])
def test_ragged_shapes(rows, cols, layout):
    _check(_rand(rows, cols, rows + 3 * cols), layout, what=f"{rows}x{cols}")


@pytest.mark.parametrize("rows,cols", SHAPES)
@pytest.mark.parametrize("layout", [nb.SF_SWIZZLED, nb.SF_LINEAR])
def test_ragged_shapes_rht(rows, cols, layout):
    _check(_rand(rows, cols, 7 * rows + cols), layout, inputs.rht_sign_mask(rows), f"rht {rows}x{cols}")


def test_pitch_wider_than_columns_and_supplied_scale():
    big = _rand(320, 512, 5)
    x = big.to(DEV)[:, 128:128 + 200]                 # ld = 512 > 200 columns
    assert x.stride(0) == 512
    q = nb.nvfp4_quantize_t(x)
    st, ref = oracle.quantize(big[:, 128:328].t().contiguous())
    assert_quantized_equal(q, ref, "strided view")
    out = nb.NVFP4Tensor.empty(200, 320, device=DEV)
    out.global_scale.fill_(float(ref.g) * 0.5)
    nb.nvfp4_quantize_t(x, out=out, global_supplied=True)
    assert_quantized_equal(out, oracle.quantize_with_global(big[:, 128:328].t().contiguous(),
                                                            float(np.float32(ref.g) * np.float32(0.5))),
                           "supplied g")


def test_errors_zero_and_empty():
    x = _rand(64, 64, 9)
    x[3, 5] = float("inf")
    nb.nvfp4_quantize_t(x.to(DEV))
    assert nb.nvfp4_check_status() == 4
    nb.nvfp4_quantize_t(x.to(DEV), sign_mask=0x00FF)
    assert nb.nvfp4_check_status() == 4
    z = nb.nvfp4_quantize_t(torch.zeros(32, 40, dtype=torch.bfloat16, device=DEV))
    assert float(z.global_scale[0]) == 1.0 and not z.codes.any() and not z.scales.any()
    e = nb.nvfp4_quantize_t(torch.zeros(0, 64, dtype=torch.bfloat16, device=DEV))
    assert e.rows == 64 and e.cols == 0
    assert nb.nvfp4_check_status() == 0


def test_wgrad_from_forward_layouts_full_size():
    """dW = dY^T X with dY [8192 x 20480] and X [8192 x 5120] in their forward
    layouts: both operands quantized column-wise with the Hadamard transform
    (same signs), compared in full with the oracle on explicit transposes;
    the GEMM on sampled outputs."""
    mask = inputs.rht_sign_mask(0)
    dy_t = inputs.wgrad_grad_output_t(device=DEV)
    x_t = inputs.wgrad_activation_t(device=DEV)
    dy, x = dy_t.t().contiguous(), x_t.t().contiguous()     # forward layouts
    qa = nb.nvfp4_quantize_t(dy, sign_mask=mask)
    qw = nb.nvfp4_quantize_t(x, sign_mask=mask)
    d = nb.nvfp4_gemm(qa, qw)
    assert nb.nvfp4_check_status() == 0
    st, ra = oracle.quantize_rht(dy_t.cpu(), mask)
    assert st == oracle.OK
    assert_quantized_equal(qa, ra, "dY column-wise")
    st, rw = oracle.quantize_rht(x_t.cpu(), mask)
    assert_quantized_equal(qw, rw, "X column-wise")
    rng = np.random.default_rng(12)
    ii, jj = rng.integers(0, qa.rows, 500), rng.integers(0, qw.rows, 500)
    ref, ab = oracle.gemm_ref(ra, rw, ii, jj)
    assert np.all(np.abs(bf16_to_f64(d)[ii, jj] - ref) <= gemm_tolerance(ref, ab))

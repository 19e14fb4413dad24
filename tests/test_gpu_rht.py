"""GPU parity of quantization after the 16x16 random Hadamard transform
("NVFP4: how NVIDIA pre-trained a 12B model on 10T tokens", section "Four
stabilisation devices") against the CPU oracle, and of the Wgrad GEMM that
consumes two such operands.

Codes, scales and the tensor scale must match bit for bit; the GEMM within
the GEMM tolerance of the oracle's FP64 product of the same quantized
operands.
"""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_block_scaled_22_b200 import binding as nb
from nvfp4_block_scaled_22_b200 import inputs
from tests.gpu_util import assert_quantized_equal, bf16_to_f64, gemm_tolerance, tile_samples

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


def _check(x_cpu, mask, layout=nb.SF_SWIZZLED, what=""):
    q = nb.nvfp4_quantize_rht(x_cpu.to(DEV), mask, layout=layout)
    st, ref = oracle.quantize_rht(x_cpu, mask, layout)
    assert st == oracle.OK
    assert nb.nvfp4_check_status() == 0
    assert_quantized_equal(q, ref, what)
    return q, ref


@pytest.mark.parametrize("rows,cols", [(1, 16), (7, 48), (129, 80), (300, 1040), (257, 4112),
                                       (1000, 512), (64, 16384)])
@pytest.mark.parametrize("layout", [nb.SF_SWIZZLED, nb.SF_LINEAR])
def test_ragged_shapes(rows, cols, layout):
    mask = inputs.rht_sign_mask(rows + cols)
    _check(_rand(rows, cols, rows * 7 + cols), mask, layout, f"{rows}x{cols}")


@pytest.mark.parametrize("mask", [0x0000, 0xFFFF, 0x0001, 0x8000, 0x5A5A])
def test_sign_masks(mask):
    _check(_rand(130, 256, 3), mask, what=f"mask {mask:#06x}")


def test_wide_dynamic_range_signed_zeros_and_subnormal_results():
    x = _rand(256, 512, 5)
    x[0] = 0.0                                   # -0 after the flips, signed zero codes
    x[1] = -0.0
    x[2, :64] = 1e-30                            # transformed values far below g's reach
    x[3, :32] = torch.tensor([2.0 ** -133] * 32)  # BF16 subnormals
    x[4] *= 1e4
    _check(x, 0xFFFF, what="zeros/range")
    _check(x, 0x0F0F, nb.SF_LINEAR, "zeros/range linear")


def test_errors_and_supplied_scale():
    x = _rand(64, 128, 9)
    _, ref = oracle.quantize_rht(x, 0x1234)
    out = nb.NVFP4Tensor.empty(64, 128, device=DEV)
    out.global_scale.fill_(float(ref.g))
    nb.nvfp4_quantize_rht(x.to(DEV), 0x1234, out=out, global_supplied=True)
    assert nb.nvfp4_check_status() == 0
    assert_quantized_equal(out, ref, "supplied g")
    bad = x.clone()
    bad[5, 9] = float("nan")
    nb.nvfp4_quantize_rht(bad.to(DEV), 0x1234)
    assert nb.nvfp4_check_status() == 4
    # finite input whose transform overflows FP32: 16 values near the BF16 max
    big = torch.full((2, 32), 3.0e38).to(torch.bfloat16)
    assert oracle.quantize_rht(big, 0)[0] == oracle.ERR_NONFINITE
    nb.nvfp4_quantize_rht(big.to(DEV), 0)
    assert nb.nvfp4_check_status() == 4
    q = nb.nvfp4_quantize_rht(torch.zeros(0, 64, dtype=torch.bfloat16, device=DEV), 7)
    assert nb.nvfp4_check_status() == 0 and float(q.global_scale[0]) == 1.0


def test_wgrad_operands_full_size_and_gemm():
    """dW = dY^T X at M = 8192 tokens: both operands quantized after the
    transform with the same signs, full compare of codes and scales, then the
    Wgrad GEMM (20480 x 5120, K = 8192, run in N-fastest tile order) on
    sampled outputs that touch every output tile."""
    mask = inputs.rht_sign_mask(0)
    dy_t = inputs.wgrad_grad_output_t(device=DEV)
    x_t = inputs.wgrad_activation_t(device=DEV)
    qa = nb.nvfp4_quantize_rht(dy_t, mask)
    qw = nb.nvfp4_quantize_rht(x_t, mask)
    d = nb.nvfp4_gemm(qa, qw)
    assert nb.nvfp4_check_status() == 0
    st, ra = oracle.quantize_rht(dy_t.cpu(), mask)
    assert st == oracle.OK
    assert_quantized_equal(qa, ra, "dY^T")
    st, rw = oracle.quantize_rht(x_t.cpu(), mask)
    assert st == oracle.OK
    assert_quantized_equal(qw, rw, "X^T")
    rng = np.random.default_rng(11)
    ti, tj = tile_samples(qa.rows, qw.rows, rng)
    ii = np.concatenate([rng.integers(0, qa.rows, 600), ti])
    jj = np.concatenate([rng.integers(0, qw.rows, 600), tj])
    ref, ab = oracle.gemm_ref(ra, rw, ii, jj)
    got = bf16_to_f64(d)[ii, jj]
    assert np.all(np.abs(got - ref) <= gemm_tolerance(ref, ab))


def test_transform_cancels_in_the_gemm():
    """Same signs on both operands along K: the quantized GEMM approximates
    the product of the untransformed BF16 operands about as well as the
    GEMM without the transform does."""
    a = _rand(256, 1024, 21, outliers=0.002)
    w = _rand(256, 1024, 22, 0.02, outliers=0.002)
    exact = a.double() @ w.double().t()
    mask = 0x3C96
    d_rht = nb.nvfp4_gemm(nb.nvfp4_quantize_rht(a.to(DEV), mask),
                          nb.nvfp4_quantize_rht(w.to(DEV), mask)).double().cpu()
    d_plain = nb.nvfp4_gemm(nb.nvfp4_quantize(a.to(DEV)), nb.nvfp4_quantize(w.to(DEV))).double().cpu()
    assert nb.nvfp4_check_status() == 0
    err_rht = (d_rht - exact).norm() / exact.norm()
    err_plain = (d_plain - exact).norm() / exact.norm()
    assert err_rht < 0.2 and err_rht < 1.5 * err_plain

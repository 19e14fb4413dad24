"""GPU parity of stochastically rounded quantization (gradients, "NVFP4: how
NVIDIA pre-trained a 12B model on 10T tokens", section "Four stabilisation
devices") against the oracle: the draws come from the same counter-based
generator on both sides, so codes, scales and the tensor scale must match
bit for bit, row-wise and column-wise, with and without the Hadamard
transform."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_block_scaled_22_b200 import binding as nb
from nvfp4_block_scaled_22_b200 import inputs
from tests.gpu_util import assert_quantized_equal

pytestmark = pytest.mark.gpu
DEV = "cuda"
SEED = 0x0DDBA11CAFEF00D5


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


ROW_SHAPES = [(1, 16), (7, 48), (129, 80), (300, 1040), (1000, 512), (64, 4112)]


@pytest.mark.parametrize("rows,cols", ROW_SHAPES)
@pytest.mark.parametrize("layout", [nb.SF_SWIZZLED, nb.SF_LINEAR])
@pytest.mark.parametrize("rht", [False, True])
def test_rowwise(rows, cols, layout, rht):
    x = _rand(rows, cols, rows * 5 + cols)
    mask = inputs.rht_sign_mask(rows) if rht else None
    q = nb.nvfp4_quantize_sr(x.to(DEV), SEED + rows, sign_mask=mask, layout=layout)
    st, ref = oracle.quantize_sr(x, SEED + rows, layout, sign_mask=mask)
    assert st == oracle.OK
    assert nb.nvfp4_check_status() == 0
    assert_quantized_equal(q, ref, f"sr {rows}x{cols} rht={rht}")


COL_SHAPES = [(16, 8), (80, 136), (1040, 296), (208, 2056)]


@pytest.mark.parametrize("rows,cols", COL_SHAPES)
@pytest.mark.parametrize("layout", [nb.SF_SWIZZLED, nb.SF_LINEAR])
@pytest.mark.parametrize("rht", [False, True])
def test_columnwise(rows, cols, layout, rht):
    x = _rand(rows, cols, rows + 11 * cols)
    mask = inputs.rht_sign_mask(cols) if rht else None
    q = nb.nvfp4_quantize_sr(x.to(DEV), SEED ^ cols, transposed=True, sign_mask=mask, layout=layout)
    st, ref = oracle.quantize_sr(x.t().contiguous(), SEED ^ cols, layout, sign_mask=mask)
    assert st == oracle.OK
    assert nb.nvfp4_check_status() == 0
    assert_quantized_equal(q, ref, f"sr^T {rows}x{cols} rht={rht}")


def test_same_seed_same_codes_other_seed_other_codes():
    x = _rand(256, 512, 9).to(DEV)
    a = nb.nvfp4_quantize_sr(x, 1)
    b = nb.nvfp4_quantize_sr(x, 1)
    c = nb.nvfp4_quantize_sr(x, 2)
    torch.cuda.synchronize()
    assert torch.equal(a.codes, b.codes) and torch.equal(a.scales, c.scales)
    assert not torch.equal(a.codes, c.codes)


def test_gradients_full_size():
    """The gradient of the ffn linear at 8192 tokens: row-wise for Dgrad and
    column-wise with the transform for Wgrad, full compare."""
    dy_t = inputs.wgrad_grad_output_t(device=DEV)
    dy = dy_t.t().contiguous()                                  # 8192 x 20480
    mask = inputs.rht_sign_mask(0)
    q = nb.nvfp4_quantize_sr(dy, 11)
    qt = nb.nvfp4_quantize_sr(dy, 12, transposed=True, sign_mask=mask)
    assert nb.nvfp4_check_status() == 0
    st, ref = oracle.quantize_sr(dy.cpu(), 11)
    assert_quantized_equal(q, ref, "dY row-wise SR")
    st, ref_t = oracle.quantize_sr(dy_t.cpu(), 12, sign_mask=mask)
    assert_quantized_equal(qt, ref_t, "dY column-wise SR + RHT")

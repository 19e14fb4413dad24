"""GPU parity of 2D (16x16 block) weight quantization against the oracle:
W's NVFP4 tensor against the oracle's 2D quantization of W, W^T's against
the oracle's 2D quantization of an explicit BF16 W^T (bit for bit), and the
Fprop / Dgrad GEMMs that consume them within the GEMM tolerance."""
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


@pytest.mark.parametrize("rows,cols", [(16, 16), (48, 80), (256, 1040), (144, 4096), (1040, 208)])
@pytest.mark.parametrize("layout", [nb.SF_SWIZZLED, nb.SF_LINEAR])
def test_both_orientations(rows, cols, layout):
    w = _rand(rows, cols, rows + cols)
    q, qt = nb.nvfp4_quantize_2d(w.to(DEV), transposed=True, layout=layout)
    assert nb.nvfp4_check_status() == 0
    st, ref = oracle.quantize_2d(w, layout)
    assert st == oracle.OK
    assert_quantized_equal(q, ref, f"W {rows}x{cols}")
    st, ref_t = oracle.quantize_2d(w.t().contiguous(), layout)
    assert_quantized_equal(qt, ref_t, f"W^T {rows}x{cols}")


@pytest.mark.parametrize("rows,cols", [(1, 16), (130, 96), (7, 4112)])
@pytest.mark.parametrize("layout", [nb.SF_SWIZZLED, nb.SF_LINEAR])
def test_partial_row_groups(rows, cols, layout):
    w = _rand(rows, cols, 3 * rows + cols)
    q = nb.nvfp4_quantize_2d(w.to(DEV), layout=layout)
    st, ref = oracle.quantize_2d(w, layout)
    assert_quantized_equal(q, ref, f"W {rows}x{cols}")


def test_supplied_scale_and_errors():
    w = _rand(64, 128, 5)
    st, ref = oracle.quantize_2d(w)
    out = nb.NVFP4Tensor.empty(64, 128, device=DEV)
    out.global_scale.fill_(float(ref.g))
    out_t = nb.NVFP4Tensor.empty(128, 64, device=DEV)
    nb.nvfp4_quantize_2d(w.to(DEV), out=out, out_t=out_t, global_supplied=True)
    assert nb.nvfp4_check_status() == 0
    assert_quantized_equal(out, ref, "supplied g")
    assert_quantized_equal(out_t, oracle.quantize_2d(w.t().contiguous())[1], "supplied g, W^T")
    bad = w.clone()
    bad[9, 9] = float("nan")
    nb.nvfp4_quantize_2d(bad.to(DEV), transposed=True)
    assert nb.nvfp4_check_status() == 4


def test_ffn_weight_full_size_fprop_and_dgrad():
    """W 20480 x 5120 (the ffn weight): both orientations in full; Fprop
    D = X W^T-contraction (A = X, B = W) and Dgrad dX = dY W (A = dY, B = W^T)
    on sampled outputs."""
    w = inputs.ffn_weight(device=DEV)
    q, qt = nb.nvfp4_quantize_2d(w, transposed=True)
    assert nb.nvfp4_check_status() == 0
    wc = w.cpu()
    st, rw = oracle.quantize_2d(wc)
    assert_quantized_equal(q, rw, "W")
    st, rwt = oracle.quantize_2d(wc.t().contiguous())
    assert_quantized_equal(qt, rwt, "W^T")
    rng = np.random.default_rng(13)
    x = inputs.ffn_activation(512, device=DEV)
    qx = nb.nvfp4_quantize(x)
    d = nb.nvfp4_gemm(qx, q)                                   # 512 x 20480
    _, rx = oracle.quantize(x.cpu())
    ii, jj = rng.integers(0, 512, 300), rng.integers(0, 20480, 300)
    ref, ab = oracle.gemm_ref(rx, rw, ii, jj)
    assert np.all(np.abs(bf16_to_f64(d)[ii, jj] - ref) <= gemm_tolerance(ref, ab))
    dy = inputs.wgrad_grad_output_t(512, device=DEV).t().contiguous()   # 512 x 20480
    qdy = nb.nvfp4_quantize(dy)
    dx = nb.nvfp4_gemm(qdy, qt)                                # 512 x 5120
    assert nb.nvfp4_check_status() == 0
    _, rdy = oracle.quantize(dy.cpu())
    ii, jj = rng.integers(0, 512, 300), rng.integers(0, 5120, 300)
    ref, ab = oracle.gemm_ref(rdy, rwt, ii, jj)
    assert np.all(np.abs(bf16_to_f64(dx)[ii, jj] - ref) <= gemm_tolerance(ref, ab))

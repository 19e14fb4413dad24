"""GPU parity of quantize / dequantize / gather against the CPU oracle.

Codes, scales and the tensor scale must match bit for bit (they are
integer/byte results of one fixed FP32 convention); dequantized BF16 too.
"""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_block_scaled_22_b200 import binding as nb
from nvfp4_block_scaled_22_b200 import inputs
from tests.gpu_util import assert_quantized_equal

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    nb.lib()
    yield
    assert nb.nvfp4_check_status() == 0


def _check(x_cpu, layout=nb.SF_SWIZZLED, what=""):
    x = x_cpu.to(DEV)
    q = nb.nvfp4_quantize(x, layout=layout)
    st, ref = oracle.quantize(x_cpu, layout)
    assert st == oracle.OK
    assert nb.nvfp4_check_status() == 0
    assert_quantized_equal(q, ref, what)
    return q, ref


def _rand(rows, cols, seed, scale=1.0, outliers=0.01):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, cols, generator=g) * scale
    n = x.numel()
    k = max(1, int(outliers * n))
    idx = torch.randint(0, n, (k,), generator=g)
    x.view(-1)[idx] *= 40
    return x.to(torch.bfloat16)


def test_tiny_linear_operands():
    for which in ("A", "W"):
        _check(inputs.tiny_operand(which), what=which)


@pytest.mark.parametrize("rows,cols", [(1, 16), (7, 48), (129, 80), (128, 64), (300, 1040),
                                       (2, 4096), (257, 16), (33, 144)])
@pytest.mark.parametrize("layout", [nb.SF_SWIZZLED, nb.SF_LINEAR])
def test_ragged_shapes(rows, cols, layout):
    _check(_rand(rows, cols, rows * 1000 + cols), layout, f"{rows}x{cols}")


def test_wide_dynamic_range_and_subnormals():
    g = torch.Generator().manual_seed(3)
    x = torch.randn(256, 512, generator=g) * torch.exp2(torch.randint(-60, 20, (256, 512), generator=g).float())
    x[5, :] = 1e-39          # BF16 subnormals
    x[6, :32] = -0.0
    _check(x.to(torch.bfloat16), what="wide range")


@pytest.mark.parametrize("n", inputs.SWEEP_SIZES[:2])
def test_sweep_sizes(n):
    _check(inputs.sweep_tensor(n), what=f"sweep {n}")


def test_sweep_largest_full_compare():
    n = inputs.SWEEP_SIZES[2]
    x = inputs.sweep_tensor(n, device=DEV)
    q = nb.nvfp4_quantize(x)
    assert nb.nvfp4_check_status() == 0
    st, ref = oracle.quantize_parallel(x.cpu())
    assert st == oracle.OK
    assert_quantized_equal(q, ref, "sweep 2^28")


@pytest.mark.parametrize("m", inputs.FFN_M)
def test_ffn_activation(m):
    _check(inputs.ffn_activation(m), what=f"ffn A m={m}")


def test_ffn_weight():
    _check(inputs.ffn_weight(), what="ffn W")


def test_kv_tensor_linear_layout():
    x = inputs.kv_tensor(0, 1, device=DEV).view(-1, inputs.KV_HEADS * inputs.KV_HEAD_DIM)
    q = nb.nvfp4_quantize(x, layout=nb.SF_LINEAR)
    assert nb.nvfp4_check_status() == 0
    st, ref = oracle.quantize_parallel(x.cpu(), oracle.SF_LINEAR)
    assert_quantized_equal(q, ref, "kv layer0 V")
    # 0.5625 bytes per value, no padding
    assert q.nbytes() == x.numel() * 9 // 16
    # dequantize round trip of the full tensor, bit for bit
    y = nb.nvfp4_dequantize(q)
    assert np.array_equal(y.cpu().view(torch.int16).numpy().view(np.uint16), ref.dequantize())


def test_kv_cache_every_tensor():
    """All 64 tensors of the KV workload (32 layers x K, V), one at a time,
    each bit for bit against the oracle, in the workspace and output buffers
    a cache would reuse."""
    T, C = inputs.KV_TOKENS, inputs.KV_HEADS * inputs.KV_HEAD_DIM
    q = nb.NVFP4Tensor.empty(T, C, nb.SF_LINEAR, DEV)
    ws = nb.Workspace(DEV)
    total = 0
    for layer in range(inputs.KV_LAYERS):
        for kv in (0, 1):
            x = inputs.kv_tensor(layer, kv, device=DEV).view(T, C)
            nb.nvfp4_quantize(x, out=q, workspace=ws)
            assert nb.nvfp4_check_status(ws) == 0
            st, ref = oracle.quantize_parallel(x.cpu(), oracle.SF_LINEAR)
            assert st == oracle.OK
            assert_quantized_equal(q, ref, f"kv layer {layer} {'KV'[kv]}")
            total += q.nbytes()
    # the KV page's worked example: 36 KiB per token over the 64 tensors
    assert total == T * 36 * 1024


def test_zero_tensor_and_empty():
    q = nb.nvfp4_quantize(torch.zeros(130, 64, dtype=torch.bfloat16, device=DEV))
    assert nb.nvfp4_check_status() == 0
    assert float(q.global_scale[0]) == 1.0
    assert int(q.codes.count_nonzero()) == 0 and int(q.scales.count_nonzero()) == 0
    q = nb.nvfp4_quantize(torch.zeros(0, 64, dtype=torch.bfloat16, device=DEV))
    assert nb.nvfp4_check_status() == 0
    assert float(q.global_scale[0]) == 1.0


def test_nonfinite_and_range_are_reported():
    x = _rand(64, 64, 9).to(DEV)
    x[3, 7] = float("nan")
    nb.nvfp4_quantize(x)
    assert nb.nvfp4_check_status() == 4
    x[3, 7] = float("-inf")
    nb.nvfp4_quantize(x)
    assert nb.nvfp4_check_status() == 4
    tiny = torch.full((16, 32), 1e-37, dtype=torch.bfloat16, device=DEV)
    nb.nvfp4_quantize(tiny)
    assert nb.nvfp4_check_status() == 5
    assert oracle.quantize(tiny.cpu())[0] == oracle.ERR_RANGE
    # supplied tensor scale: Inf in the data still reported
    x[3, 7] = float("inf")
    q = nb.NVFP4Tensor.empty(64, 64, device=DEV)
    q.global_scale.fill_(1.0)
    nb.nvfp4_quantize(x, out=q, global_supplied=True)
    assert nb.nvfp4_check_status() == 4


def test_supplied_global_scale():
    x = _rand(200, 256, 11)
    st, ref_full = oracle.quantize(x)
    g = np.float32(ref_full.g) * np.float32(0.75)   # any caller-chosen g
    ref = oracle.quantize_with_global(x, float(g))
    q = nb.NVFP4Tensor.empty(200, 256, device=DEV)
    q.global_scale.fill_(float(g))
    nb.nvfp4_quantize(x.to(DEV), out=q, global_supplied=True)
    assert nb.nvfp4_check_status() == 0
    assert_quantized_equal(q, ref, "supplied g")


def test_global_scale_entry():
    x = _rand(333, 512, 12)
    g = nb.nvfp4_global_scale(x.to(DEV))
    assert nb.nvfp4_check_status() == 0
    st, amax = oracle.tensor_amax(x)
    assert float(g[0]) == oracle.global_scale(amax)[1]


@pytest.mark.parametrize("layout", [nb.SF_SWIZZLED, nb.SF_LINEAR])
def test_dequantize_parity(layout):
    x = _rand(300, 1040, 13, scale=2.0)
    q, ref = _check(x, layout)
    y = nb.nvfp4_dequantize(q)
    yr = ref.dequantize()
    got = y.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, yr)


def test_dequantize_exact_round_trip():
    rng = np.random.default_rng(5)
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float32)
    c = grid[rng.integers(0, 8, (128, 16, 16))] * rng.choice([-1, 1], (128, 16, 16))
    c[:, :, 0] = 6.0
    k = rng.integers(-10, 4, (128, 16, 1))
    x = torch.from_numpy((c * np.exp2(k)).reshape(128, 256).astype(np.float32)).to(torch.bfloat16)
    q = nb.nvfp4_quantize(x.to(DEV))
    y = nb.nvfp4_dequantize(q)
    assert torch.equal(y.cpu(), x)


def test_quantize_gather_moe_parity():
    r = inputs.MoeRouting()
    x = inputs.moe_activation()
    gather = r.gather.to(DEV)
    xd = x.to(DEV)
    gx = nb.nvfp4_global_scale(xd)
    q = nb.NVFP4Tensor.empty(r.padded_rows, x.shape[1], device=DEV, global_scale=gx)
    nb.nvfp4_quantize_gather(xd, gather, out=q, global_supplied=True)
    assert nb.nvfp4_check_status() == 0
    gathered = torch.zeros(r.padded_rows, x.shape[1], dtype=torch.bfloat16)
    real = r.gather >= 0
    gathered[real] = x[r.gather[real].long()]
    st, amax = oracle.tensor_amax(x)
    ref = oracle.quantize_with_global(gathered, oracle.global_scale(amax)[1])
    assert_quantized_equal(q, ref, "moe gather")


def test_quantize_gather_own_amax():
    x = _rand(50, 128, 14)
    gather = torch.tensor([3, -1, 0, 49, 49, -1, 7] * 20, dtype=torch.int32)
    q = nb.nvfp4_quantize_gather(x.to(DEV), gather.to(DEV))
    assert nb.nvfp4_check_status() == 0
    gathered = torch.zeros(len(gather), 128, dtype=torch.bfloat16)
    real = gather >= 0
    gathered[real] = x[gather[real].long()]
    st, ref = oracle.quantize(gathered)
    assert_quantized_equal(q, ref, "gather own amax")


@pytest.mark.parametrize("src_layout", [nb.SF_SWIZZLED, nb.SF_LINEAR])
def test_gather_rows_moe_parity(src_layout):
    """Quantize X once, then gather its NVFP4 rows into the expert slots:
    bit for bit the oracle's quantization of the gathered rows with X's
    tensor scale, and the same bytes as the gathered quantize."""
    r = inputs.MoeRouting()
    x = inputs.moe_activation()
    xd = x.to(DEV)
    gather = r.gather.to(DEV)
    qx = nb.nvfp4_quantize(xd, layout=src_layout)
    q = nb.nvfp4_gather_rows(qx, gather)
    qg = nb.NVFP4Tensor.empty(r.padded_rows, x.shape[1], device=DEV, global_scale=nb.nvfp4_global_scale(xd))
    nb.nvfp4_quantize_gather(xd, gather, out=qg, global_supplied=True)
    assert nb.nvfp4_check_status() == 0
    gathered = torch.zeros(r.padded_rows, x.shape[1], dtype=torch.bfloat16)
    real = r.gather >= 0
    gathered[real] = x[r.gather[real].long()]
    st, amax = oracle.tensor_amax(x)
    ref = oracle.quantize_with_global(gathered, oracle.global_scale(amax)[1])
    assert_quantized_equal(q, ref, "gathered rows")
    assert torch.equal(q.codes, qg.codes) and torch.equal(q.scales, qg.scales)


@pytest.mark.parametrize("src_layout,dst_layout", [(nb.SF_SWIZZLED, nb.SF_SWIZZLED),
                                                   (nb.SF_LINEAR, nb.SF_SWIZZLED),
                                                   (nb.SF_SWIZZLED, nb.SF_LINEAR),
                                                   (nb.SF_LINEAR, nb.SF_LINEAR)])
@pytest.mark.parametrize("cols", [16, 48, 1040, 8448])
def test_gather_rows_layouts_ragged_and_bad_entries(src_layout, dst_layout, cols):
    x = _rand(70, cols, cols + src_layout)
    qs = nb.nvfp4_quantize(x.to(DEV), layout=src_layout)
    gather = torch.tensor([69, -1, 0, 5, 5, 130, -1, 33] * 17, dtype=torch.int32)   # 130: out of range
    q = nb.nvfp4_gather_rows(qs, gather.to(DEV), layout=dst_layout)
    assert nb.nvfp4_check_status() == 1                                              # NVFP4_ERR_INVALID_ARG
    rows = torch.zeros(len(gather), cols, dtype=torch.bfloat16)
    ok = (gather >= 0) & (gather < 70)
    rows[ok] = x[gather[ok].long()]
    st, amax = oracle.tensor_amax(x)
    ref = oracle.quantize_with_global(rows, oracle.global_scale(amax)[1], dst_layout)
    assert_quantized_equal(q, ref, f"gather {src_layout}->{dst_layout}")

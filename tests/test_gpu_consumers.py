"""GPU parity of the consumer steps against the oracle: the MoE per-token
combine (bit for bit: the same FMA chain in the same order) and the NVFP4
-> FP8 conversion for attention reads (bit for bit, after the quantize of
the same input is itself checked against the oracle)."""
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


def test_moe_combine_full_routing():
    r = inputs.MoeRouting()
    g = torch.Generator(device=DEV).manual_seed(inputs.seed_for("moe", 9100))
    out = torch.randn((r.padded_rows, inputs.MOE_HIDDEN), generator=g, device=DEV).to(torch.bfloat16)
    slots = r.token_slots.to(DEV)
    w = r.combine_weights.to(DEV)
    y = nb.nvfp4_moe_combine(out, slots, w)
    torch.cuda.synchronize()
    ref = oracle.moe_combine(out.cpu(), r.token_slots.numpy(), r.combine_weights.numpy())
    assert np.array_equal(y.cpu().view(torch.int16).numpy().view(np.uint16), ref)


@pytest.mark.parametrize("tokens,topk,hidden", [(1, 1, 8), (37, 3, 2056), (300, 8, 6144)])
def test_moe_combine_shapes_and_skipped_slots(tokens, topk, hidden):
    rng = np.random.default_rng(tokens + topk)
    rows = 64
    out = torch.from_numpy(rng.standard_normal((rows, hidden)).astype(np.float32)).to(torch.bfloat16)
    slots = rng.integers(-1, rows + 5, (tokens, topk)).astype(np.int32)   # -1 and out-of-range skipped
    w = rng.random((tokens, topk)).astype(np.float32)
    y = nb.nvfp4_moe_combine(out.to(DEV), torch.from_numpy(slots).to(DEV), torch.from_numpy(w).to(DEV))
    s2 = np.where(slots >= rows, -1, slots)
    ref = oracle.moe_combine(out, s2, w)
    assert np.array_equal(y.cpu().view(torch.int16).numpy().view(np.uint16), ref)


def _fp8_case(x_dev, layout, what):
    """GPU quantize then GPU NVFP4 -> FP8, against the oracle's own quantize
    of the same BF16 input followed by the oracle's conversion: both steps
    are checked, and no oracle input comes from the GPU."""
    q = nb.nvfp4_quantize(x_dev, layout=layout)
    y, sc = nb.nvfp4_dequantize_fp8(q)
    torch.cuda.synchronize()
    assert nb.nvfp4_check_status() == 0
    st, r = oracle.quantize(x_dev.cpu(), layout)
    assert st == oracle.OK
    assert_quantized_equal(q, r, what)
    ref, rsc = oracle.dequantize_fp8(r)
    assert np.float32(sc.item()) == np.float32(rsc)
    assert np.array_equal(y.cpu().numpy(), ref)


@pytest.mark.parametrize("layout", [nb.SF_SWIZZLED, nb.SF_LINEAR])
def test_fp8_conversion_kv_tensor(layout):
    x = inputs.kv_tensor(0, 1, device=DEV).view(inputs.KV_TOKENS, -1)[:8192].contiguous()
    _fp8_case(x, layout, "kv rows for fp8")


def test_fp8_conversion_ragged_and_tiny_scales():
    g = torch.Generator().manual_seed(5)
    x = torch.randn(130, 96, generator=g)
    x[3] *= 1e-6                                      # tiny block scales: FP8 underflow
    x[4] *= 1e4
    _fp8_case(x.to(torch.bfloat16).to(DEV), nb.SF_SWIZZLED, "ragged fp8")


@pytest.mark.parametrize("rows,inter", [(1, 16), (37, 80), (300, 1040), (4096, 2048)])
@pytest.mark.parametrize("layout", [nb.SF_SWIZZLED, nb.SF_LINEAR])
def test_swiglu_quantize(rows, inter, layout):
    g = torch.Generator().manual_seed(rows + inter)
    gu = (torch.randn(rows, 2 * inter, generator=g) * 3).to(torch.bfloat16)
    gu[0, :4] = torch.tensor([90.0, -90.0, 0.0, -0.0])          # clamp ends and zeros
    q = nb.nvfp4_quantize_swiglu(gu.to(DEV), layout=layout)
    assert nb.nvfp4_check_status() == 0
    st, ref = oracle.quantize_swiglu(gu, layout)
    assert st == oracle.OK
    assert_quantized_equal(q, ref, f"swiglu {rows}x{inter}")


def _swiglu_edge_tensor(case):
    """Gate|up rows (256 x 2*160, BF16) for one screening edge case."""
    rows, inter = 256, 160
    g = torch.Generator().manual_seed(77)
    gate = torch.randn(rows, inter, generator=g) * 3
    up = torch.randn(rows, inter, generator=g) * 3
    if case == "subnormal_gates":
        # g * r below the normal range against ups that make h ~ 1e-10
        sub = torch.randint(1, 128, (rows // 2, inter), generator=g).float() * 2.0 ** -133
        gate[: rows // 2] = sub * torch.sign(gate[: rows // 2])
        up[: rows // 2] = torch.sign(up[: rows // 2]) * torch.exp(
            torch.rand(rows // 2, inter, generator=g) * 3 + 64)
        gate[rows // 2:] *= 1e-5
        up[rows // 2:] *= 1e-5
    elif case == "tiny":
        # every block max below 2^-90: all h from the defined formula
        gate *= 1e-15
        up *= 1e-15
    elif case == "large":
        gate *= 1e17
        up *= 1e17
    elif case == "clamp_zeros_ties":
        gate[5] = torch.linspace(-120.0, -60.0, inter)     # exp clamp, deep negative gates
        gate[6] = torch.linspace(60.0, 120.0, inter)
        gate[7, ::2] = 0.0
        gate[7, 1::2] = -0.0
        up[8, ::3] = -0.0
        gate[11, :16] = 2.0                                # sixteen values tie the block max
        up[11, :16] = 1.5
        gate[12, :16] = torch.tensor([2.0, 2.0078125] * 8)  # near-ties one BF16 step apart
        up[12, :16] = 3.0
        gate[13, :16] *= 1e-30                             # a tiny block in a normal row
    return torch.cat([gate, up], dim=1).to(torch.bfloat16)


@pytest.mark.parametrize("case", ["subnormal_gates", "tiny", "large", "clamp_zeros_ties"])
@pytest.mark.parametrize("layout", [nb.SF_SWIZZLED, nb.SF_LINEAR])
def test_swiglu_quantize_screening_edges(case, layout):
    """Inputs that the kernel's cheap screening of h cannot decide alone:
    subnormal gates (g * r not a normal number), blocks of tiny values (every
    h from the defined formula), large finite h, gates at and beyond the exp
    clamp, signed zeros and ties of the block maximum; codes, scales and g
    must still equal the oracle's."""
    gu = _swiglu_edge_tensor(case)
    q = nb.nvfp4_quantize_swiglu(gu.to(DEV), layout=layout)
    assert nb.nvfp4_check_status() == 0
    st, ref = oracle.quantize_swiglu(gu, layout)
    assert st == oracle.OK
    assert_quantized_equal(q, ref, f"swiglu screening {case}")

"""MoE expert block at full size (256 experts, top-8 of 4096 tokens, hidden
6144, intermediate 2048) against the oracle on sampled experts and outputs.

Oracle inputs come only from the seeded generators: the down projection is
checked on a generated intermediate (not on the GPU's up-projection output).
"""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_block_scaled_22_b200 import binding as nb
from nvfp4_block_scaled_22_b200 import inputs
from tests.gpu_util import assert_quantized_equal, bf16_to_f64, gemm_tolerance

pytestmark = pytest.mark.gpu
DEV = "cuda"
E, H, I = inputs.MOE_EXPERTS, inputs.MOE_HIDDEN, inputs.MOE_INTER
SAMPLE_EXPERTS = (0, 17, 128, 255)


@pytest.fixture(scope="module")
def routing():
    return inputs.MoeRouting()


def _stacked(which, n, k):
    q = nb.NVFP4Tensor.empty(E * n, k, device=DEV)
    g = torch.zeros(E, dtype=torch.float32, device=DEV)
    sfb = nb.nvfp4_scales_bytes(n, k)
    for e in range(E):
        w = inputs.moe_expert_weight(which, e, device=DEV)
        sub = nb.NVFP4Tensor(q.codes[e * n:(e + 1) * n], q.scales[e * sfb:(e + 1) * sfb],
                             g[e:e + 1], n, k, nb.SF_SWIZZLED)
        nb.nvfp4_quantize(w, out=sub)
    assert nb.nvfp4_check_status() == 0
    return q, g, sfb


def _expert_ref(which, e, n, k, q, g, sfb):
    """Oracle quantization of expert e's weight, checked against the GPU slice."""
    w = inputs.moe_expert_weight(which, e, device=DEV).cpu()
    st, ref = oracle.quantize(w)
    assert st == oracle.OK
    sub = nb.NVFP4Tensor(q.codes[e * n:(e + 1) * n], q.scales[e * sfb:(e + 1) * sfb],
                         g[e:e + 1], n, k, nb.SF_SWIZZLED)
    assert_quantized_equal(sub, ref, f"W_{which}[{e}]")
    return ref


def _sample_rows(routing, e, count, rng):
    o = int(routing.slot_offsets[e])
    r = int(routing.rows[e])
    return o + rng.integers(0, r, count)


def test_routing_structure(routing):
    assert routing.real_rows == inputs.MOE_TOKENS * inputs.MOE_TOPK
    assert int(routing.rows.sum()) == routing.real_rows
    assert int(routing.slot_offsets[-1]) == routing.padded_rows
    assert np.all(np.diff(routing.slot_offsets.numpy()) % 128 == 0)
    # every token appears exactly top-k times, each within one expert once
    g = routing.gather[routing.gather >= 0].long()
    assert torch.equal(torch.bincount(g, minlength=inputs.MOE_TOKENS),
                       torch.full((inputs.MOE_TOKENS,), inputs.MOE_TOPK))
    assert routing.rows.min() >= 0 and routing.rows.max() > routing.rows.min()   # uneven batches


def test_up_projection_full_size(routing):
    x = inputs.moe_activation(device=DEV)
    gx = nb.nvfp4_global_scale(x)
    qx = nb.NVFP4Tensor.empty(routing.padded_rows, H, device=DEV, global_scale=gx)
    nb.nvfp4_quantize_gather(x, routing.gather.to(DEV), out=qx, global_supplied=True)
    wu, gu, sfb = _stacked("up", I, H)
    h = torch.zeros((routing.padded_rows, I), dtype=torch.bfloat16, device=DEV)
    nb.nvfp4_grouped_gemm(routing.slot_offsets.to(DEV), routing.rows.to(DEV), qx, wu, gu, I, out=h)
    assert nb.nvfp4_check_status() == 0

    xc = x.cpu()
    st, amax = oracle.tensor_amax(xc)
    g = oracle.global_scale(amax)[1]
    assert float(gx[0]) == g
    rng = np.random.default_rng(1)
    qx_codes = qx.codes.cpu().numpy()
    for e in SAMPLE_EXPERTS:
        ref_w = _expert_ref("up", e, I, H, wu, gu, sfb)
        rows = _sample_rows(routing, e, 6, rng)
        src = routing.gather[rows].long()
        qa = oracle.quantize_with_global(xc[src], g)
        assert np.array_equal(qa.codes, qx_codes[rows]), f"gathered codes, expert {e}"
        cols = rng.integers(0, I, 40)
        ii = np.repeat(np.arange(len(rows)), len(cols))
        jj = np.tile(cols, len(rows))
        ref, ab = oracle.gemm_ref(qa, ref_w, ii, jj)
        got = bf16_to_f64(h)[rows[ii], jj]
        assert np.all(np.abs(got - ref) <= gemm_tolerance(ref, ab)), f"expert {e}"


def test_down_projection_full_size(routing):
    # generated intermediate in the padded expert layout (zeros in padding rows)
    gen = torch.Generator(device=DEV).manual_seed(inputs.seed_for("moe", 9000))
    hmid = torch.randn((routing.padded_rows, I), generator=gen, device=DEV).to(torch.bfloat16)
    real = (routing.gather >= 0).to(DEV)
    hmid[~real] = 0
    ident = torch.where(routing.gather >= 0, torch.arange(routing.padded_rows, dtype=torch.int32),
                        torch.full_like(routing.gather, -1)).to(DEV)
    qh = nb.nvfp4_quantize_gather(hmid, ident)
    wd, gd, sfb = _stacked("down", H, I)
    y = torch.zeros((routing.padded_rows, H), dtype=torch.bfloat16, device=DEV)
    nb.nvfp4_grouped_gemm(routing.slot_offsets.to(DEV), routing.rows.to(DEV), qh, wd, gd, H, out=y)
    assert nb.nvfp4_check_status() == 0

    hc = hmid.cpu()
    st, rq = oracle.quantize(hc)                 # padding rows are zero: same amax
    assert_quantized_equal(qh, rq, "intermediate")
    rng = np.random.default_rng(2)
    for e in SAMPLE_EXPERTS:
        ref_w = _expert_ref("down", e, H, I, wd, gd, sfb)
        rows = _sample_rows(routing, e, 5, rng)
        cols = rng.integers(0, H, 40)
        ii = np.repeat(rows, len(cols))
        jj = np.tile(cols, len(rows))
        ref, ab = oracle.gemm_ref(rq, ref_w, ii, jj)
        got = bf16_to_f64(y)[ii, jj]
        assert np.all(np.abs(got - ref) <= gemm_tolerance(ref, ab)), f"expert {e}"

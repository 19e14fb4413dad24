"""MoE expert block at full size (256 experts, top-8 of 4096 tokens, hidden
6144, intermediate 2048) against the oracle, on every expert.

Per expert: its tensor scale and the sampled weight rows are checked bit for
bit against the oracle (four experts' weights in full), and outputs are
sampled so that every expert's first and last real row and every 256-column
output tile are touched.  Oracle inputs come only from the seeded generators:
the down projection is checked on a generated intermediate (not on the GPU's
up-projection output).
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
FULL_EXPERTS = (0, 17, 128, 255)


@pytest.fixture(scope="module")
def routing():
    return inputs.MoeRouting()


def _stacked(which, n, k):
    q = nb.NVFP4Tensor.empty(E * n, k, device=DEV)
    g = torch.zeros(E, dtype=torch.float32, device=DEV)
    sfb = nb.nvfp4_scales_bytes(n, k)
    for e in range(E):
        w = inputs.moe_expert_weight(which, e, device=DEV)
        nb.nvfp4_quantize(w, out=_slice(q, g, e, n, k, sfb))
    assert nb.nvfp4_check_status() == 0
    return q, g, sfb


def _slice(q, g, e, n, k, sfb):
    return nb.NVFP4Tensor(q.codes[e * n:(e + 1) * n], q.scales[e * sfb:(e + 1) * sfb],
                          g[e:e + 1], n, k, nb.SF_SWIZZLED)


def _sf_table(n, k):
    """Byte offset of block (row, block column) in one expert's 128x4 scale
    slice, from the oracle's layout function."""
    t = np.empty((n, k // 16), np.int64)
    for r in range(n):
        for c in range(k // 16):
            t[r, c] = oracle.sf_offset(r, c, n, k, oracle.SF_SWIZZLED)
    return t


def _tile_cols(n, rng):
    """One random column in every 256-column output tile, plus the last."""
    c = np.arange(0, n, 256) + rng.integers(0, 256, -(-n // 256))
    return np.unique(np.concatenate([np.minimum(c, n - 1), [n - 1]]))


def _edge_rows(routing, e, rng):
    """First, last and one random real row of expert e's slot (global rows)."""
    o, r = int(routing.slot_offsets[e]), int(routing.rows[e])
    if r == 0:
        return np.zeros(0, np.int64)
    return np.unique(np.array([o, o + r - 1, o + int(rng.integers(0, r))], np.int64))


def _at(d, i, j):
    """D[i, j] as float64, gathered on the device."""
    it = torch.from_numpy(np.ascontiguousarray(i, np.int64)).to(DEV)
    jt = torch.from_numpy(np.ascontiguousarray(j, np.int64)).to(DEV)
    return bf16_to_f64(d[it, jt])


def _expert_check(which, e, n, k, q, g, sfb, cols, sf_table):
    """Oracle tensor scale of expert e's weight (over all of it) and the
    oracle quantization of weight rows `cols` under it, both checked bit for
    bit against the GPU's stacked tensor.  Returns those rows as an oracle
    tensor (row-major scales) for the GEMM reference."""
    w = inputs.moe_expert_weight(which, e, device=DEV).cpu()
    if e in FULL_EXPERTS:
        st, full = oracle.quantize_parallel(w)
        assert st == oracle.OK
        assert_quantized_equal(_slice(q, g, e, n, k, sfb), full, f"W_{which}[{e}]")
    st, amax = oracle.tensor_amax(w)
    assert st == oracle.OK
    st, gw = oracle.global_scale(amax)
    assert st == oracle.OK
    assert np.float32(g[e].item()) == np.float32(gw), f"W_{which}[{e}] tensor scale"
    sub = oracle.quantize_with_global(w[torch.from_numpy(cols)], gw, oracle.SF_LINEAR)
    rows = torch.from_numpy(e * n + cols).to(DEV)
    assert np.array_equal(q.codes[rows].cpu().numpy(), sub.codes), f"W_{which}[{e}] codes"
    sf = q.scales[e * sfb:(e + 1) * sfb].cpu().numpy()
    assert np.array_equal(sf[sf_table[cols]].ravel(), sub.scales), f"W_{which}[{e}] scales"
    return sub


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
    sf_table = _sf_table(I, H)
    for e in range(E):
        cols = _tile_cols(I, rng)
        ref_w = _expert_check("up", e, I, H, wu, gu, sfb, cols, sf_table)
        rows = _edge_rows(routing, e, rng)
        if rows.size == 0:
            continue
        src = routing.gather[torch.from_numpy(rows)].long()
        qa = oracle.quantize_with_global(xc[src], g)
        assert np.array_equal(qa.codes, qx.codes[torch.from_numpy(rows).to(DEV)].cpu().numpy()), \
            f"gathered codes, expert {e}"
        ii = np.repeat(np.arange(len(rows)), len(cols))
        jj = np.tile(np.arange(len(cols)), len(rows))
        ref, ab = oracle.gemm_ref(qa, ref_w, ii, jj)
        got = _at(h, rows[ii], cols[jj])
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
    st, rq = oracle.quantize_parallel(hc)        # padding rows are zero: same amax
    assert st == oracle.OK
    assert_quantized_equal(qh, rq, "intermediate")
    rng = np.random.default_rng(2)
    sf_table = _sf_table(H, I)
    for e in range(E):
        cols = _tile_cols(H, rng)
        ref_w = _expert_check("down", e, H, I, wd, gd, sfb, cols, sf_table)
        rows = _edge_rows(routing, e, rng)
        if rows.size == 0:
            continue
        ii = np.repeat(rows, len(cols))
        jj = np.tile(np.arange(len(cols)), len(rows))
        ref, ab = oracle.gemm_ref(rq, ref_w, ii, jj)
        got = _at(y, ii, cols[jj])
        assert np.all(np.abs(got - ref) <= gemm_tolerance(ref, ab)), f"expert {e}"


def _ident(routing):
    return torch.where(routing.gather >= 0, torch.arange(routing.padded_rows, dtype=torch.int32),
                       torch.full_like(routing.gather, -1)).to(DEV)


@pytest.mark.parametrize("n", [256, 384])
def test_out_scale_small_groups(n):
    """The grouped GEMM's tensor scale of its output (max over real rows and
    the n columns, from the epilogue) equals the one the intermediate's
    quantize computes in its own amax pass over the same rows, bit for bit;
    the output itself is unchanged.  n = 384: a 256-column tile reaches into
    the next group's weights, which must not count."""
    rows, k = [5, 130, 0, 128], 512
    offs = np.concatenate([[0], np.cumsum([-(-r // 128) * 128 for r in rows])]).astype(np.int32)
    gen = torch.Generator().manual_seed(77 + n)
    a = torch.zeros(int(offs[-1]), k, dtype=torch.bfloat16)
    for g, r in enumerate(rows):
        a[offs[g]:offs[g] + r] = torch.randn(r, k, generator=gen).to(torch.bfloat16)
    w = (torch.randn(len(rows) * n, k, generator=gen) * 0.02).to(torch.bfloat16)
    w[2 * n:3 * n] *= 50.0                 # the group with no rows has the largest weights
    qa, qw = nb.nvfp4_quantize(a.to(DEV)), nb.nvfp4_quantize(w.to(DEV))
    gws = qw.global_scale.repeat(len(rows))
    off_d, rows_d = torch.from_numpy(offs).to(DEV), torch.tensor(rows, dtype=torch.int32, device=DEV)
    d0 = torch.zeros((a.shape[0], n), dtype=torch.bfloat16, device=DEV)
    d1 = torch.zeros_like(d0)
    nb.nvfp4_grouped_gemm(off_d, rows_d, qa, qw, gws, n, out=d0)
    _, g1 = nb.nvfp4_grouped_gemm_out_scale(off_d, rows_d, qa, qw, gws, n, out=d1)
    assert nb.nvfp4_check_status() == 0
    assert torch.equal(d0, d1)
    real = torch.zeros(a.shape[0], dtype=torch.bool)
    for g, r in enumerate(rows):
        real[offs[g]:offs[g] + r] = True
    ident = torch.where(real, torch.arange(a.shape[0], dtype=torch.int32),
                        torch.full((a.shape[0],), -1, dtype=torch.int32)).to(DEV)
    q_own = nb.nvfp4_quantize_gather(d1, ident)
    assert nb.nvfp4_check_status() == 0
    assert g1.item() == q_own.global_scale.item()


def test_out_scale_full_size(routing):
    """At the MoE shape: the up projection's output tensor scale equals the
    intermediate quantize's own, and quantizing with it supplied gives the
    same bytes."""
    x = inputs.moe_activation(device=DEV)
    qx = nb.nvfp4_quantize_gather(x, routing.gather.to(DEV))
    wu, gu, _ = _stacked("up", I, H)
    off_d, rows_d = routing.slot_offsets.to(DEV), routing.rows.to(DEV)
    h, g1 = nb.nvfp4_grouped_gemm_out_scale(off_d, rows_d, qx, wu, gu, I)
    assert nb.nvfp4_check_status() == 0
    ident = _ident(routing)
    q_own = nb.nvfp4_quantize_gather(h, ident)
    q_sup = nb.NVFP4Tensor.empty(routing.padded_rows, I, device=DEV, global_scale=g1.clone())
    nb.nvfp4_quantize_gather(h, ident, out=q_sup, global_supplied=True)
    assert nb.nvfp4_check_status() == 0
    assert g1.item() == q_own.global_scale.item()
    assert torch.equal(q_sup.codes, q_own.codes) and torch.equal(q_sup.scales, q_own.scales)

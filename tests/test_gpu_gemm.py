"""GPU parity of the block-scaled NVFP4 GEMM and grouped GEMM against the
oracle's FP64 GEMM over the dequantized operands.

Bar: |D - ref| <= 1e-3 * sum_k |a_ik w_jk| + half a BF16 ulp of ref per
element.  Operands are quantized by the CUDA path; they are bit-identical to
the oracle's (checked here too), so both sides multiply the same numbers.
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


def _rand(rows, cols, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, cols, generator=g) * scale
    if x.numel():
        idx = torch.randint(0, x.numel(), (max(1, x.numel() // 200),), generator=g)
        x.view(-1)[idx] *= 30
    return x.to(torch.bfloat16)


def _quant_both(x_cpu, what):
    q = nb.nvfp4_quantize(x_cpu.to(DEV))
    st, ref = oracle.quantize(x_cpu)
    assert st == oracle.OK
    assert_quantized_equal(q, ref, what)
    return q, ref


def _check_full(a_cpu, w_cpu, what):
    qa, ra = _quant_both(a_cpu, what + " A")
    qw, rw = _quant_both(w_cpu, what + " W")
    d = nb.nvfp4_gemm(qa, qw)
    assert nb.nvfp4_check_status() == 0
    m, n = a_cpu.shape[0], w_cpu.shape[0]
    ii, jj = np.meshgrid(np.arange(m), np.arange(n), indexing="ij")
    ref, ab = oracle.gemm_ref(ra, rw, ii.ravel(), jj.ravel())
    got = bf16_to_f64(d).ravel()
    err = np.abs(got - ref)
    tol = gemm_tolerance(ref, ab)
    bad = np.nonzero(err > tol)[0]
    assert bad.size == 0, (f"{what}: {bad.size}/{err.size} outside tolerance; first "
                           f"(i,j)={ii.ravel()[bad[:4]]},{jj.ravel()[bad[:4]]} got {got[bad[:4]]} "
                           f"ref {ref[bad[:4]]}")
    return d


def test_tiny_linear():
    _check_full(inputs.tiny_operand("A"), inputs.tiny_operand("W"), "tiny")


@pytest.fixture(params=[True, False], ids=["pairs", "single"])
def pairs(request):
    prev = nb.nvfp4_set_gemm_pairs(request.param)
    yield request.param
    nb.nvfp4_set_gemm_pairs(prev)


@pytest.mark.parametrize("m,n,k", [(1, 1, 64), (7, 9, 64), (129, 300, 128), (128, 256, 320),
                                   (300, 513, 1088), (256, 512, 4096), (64, 1000, 256),
                                   (1, 256, 5120), (640, 384, 192), (257, 257, 320)])
def test_ragged_shapes(m, n, k, pairs):
    _check_full(_rand(m, k, m + 7 * n + k), _rand(n, k, 3 * m + n + k, 0.02), f"{m}x{n}x{k}")


def test_output_pitch_and_untouched_padding():
    a, w = _rand(130, 256, 1), _rand(200, 256, 2)
    qa, ra = _quant_both(a, "A")
    qw, rw = _quant_both(w, "W")
    out = torch.full((130, 264), 7.0, dtype=torch.bfloat16, device=DEV)
    nb.nvfp4_gemm(qa, qw, out=out[:, :200])
    assert nb.nvfp4_check_status() == 0
    assert torch.all(out[:, 200:] == 7.0)
    ii, jj = np.meshgrid(np.arange(130), np.arange(200), indexing="ij")
    ref, ab = oracle.gemm_ref(ra, rw, ii.ravel(), jj.ravel())
    got = bf16_to_f64(out[:, :200]).ravel()
    assert np.all(np.abs(got - ref) <= gemm_tolerance(ref, ab))


def _sampled(d, ra, rw, m, n, count, seed, gw=None, rows_map=None):
    rng = np.random.default_rng(seed)
    i = rng.integers(0, m, count)
    j = rng.integers(0, n, count)
    ti, tj = tile_samples(m, n, rng)
    i = np.concatenate([i, ti])
    j = np.concatenate([j, tj])
    wj = j if rows_map is None else rows_map(i, j)
    ref, ab = oracle.gemm_ref(ra, rw, i, wj, gw=None if gw is None else gw(i))
    got = bf16_to_f64(d[torch.from_numpy(i).to(d.device), torch.from_numpy(j).to(d.device)])
    tol = gemm_tolerance(ref, ab)
    bad = np.nonzero(np.abs(got - ref) > tol)[0]
    assert bad.size == 0, f"{bad.size} sampled outputs outside tolerance, e.g. {i[bad[:4]]},{j[bad[:4]]}"


@pytest.fixture(scope="module")
def ffn_weight():
    w = inputs.ffn_weight()
    return _quant_both(w, "ffn W")


@pytest.mark.parametrize("m", inputs.FFN_M)
def test_ffn_linear_full_size(m, ffn_weight, pairs):
    qw, rw = ffn_weight
    qa, ra = _quant_both(inputs.ffn_activation(m), f"ffn A {m}")
    d = nb.nvfp4_gemm(qa, qw)
    assert nb.nvfp4_check_status() == 0
    _sampled(d, ra, rw, m, inputs.FFN_N, 1500, m)
    assert torch.isfinite(d.float()).all()


def _grouped_case(rows_per_group, n, k, seed):
    groups = len(rows_per_group)
    padded = [((r + 127) // 128) * 128 for r in rows_per_group]
    offs = np.concatenate([[0], np.cumsum(padded)]).astype(np.int32)
    total = int(offs[-1])
    a = torch.zeros(total, k, dtype=torch.bfloat16)
    for g, r in enumerate(rows_per_group):
        a[offs[g]:offs[g] + r] = _rand(r, k, seed + g)
    w_list = [_rand(n, k, seed + 1000 + g, 0.02) for g in range(groups)]
    return offs, a, w_list


@pytest.mark.parametrize("rows_per_group,n,k", [([5, 0, 130, 128, 1], 256, 256),
                                                ([300, 17], 384, 192),
                                                ([1, 2, 3, 4, 5, 6, 7, 8], 128, 64)])
def test_grouped_small_full(rows_per_group, n, k):
    offs, a, w_list = _grouped_case(rows_per_group, n, k, 77)
    groups = len(rows_per_group)
    qa, ra = _quant_both(a, "grouped A")
    w_all = torch.cat(w_list, 0)
    qw = nb.NVFP4Tensor.empty(groups * n, k, device=DEV)
    gws = torch.zeros(groups, dtype=torch.float32, device=DEV)
    refs = []
    sf_per_group = nb.nvfp4_scales_bytes(n, k)
    for g in range(groups):
        sub = nb.NVFP4Tensor(qw.codes[g * n:(g + 1) * n], qw.scales[g * sf_per_group:(g + 1) * sf_per_group],
                             gws[g:g + 1], n, k, nb.SF_SWIZZLED)
        nb.nvfp4_quantize(w_list[g].to(DEV), out=sub)
        st, rg = oracle.quantize(w_list[g])
        assert_quantized_equal(sub, rg, f"W[{g}]")
        refs.append(rg)
    assert nb.nvfp4_check_status() == 0
    out = torch.full((a.shape[0], n), 3.0, dtype=torch.bfloat16, device=DEV)
    nb.nvfp4_grouped_gemm(torch.from_numpy(offs).to(DEV),
                          torch.tensor(rows_per_group, dtype=torch.int32, device=DEV),
                          qa, qw, gws, n, out=out)
    assert nb.nvfp4_check_status() == 0
    got = bf16_to_f64(out)
    for g, r in enumerate(rows_per_group):
        o = int(offs[g])
        if r:
            ii, jj = np.meshgrid(np.arange(o, o + r), np.arange(n), indexing="ij")
            ref, ab = oracle.gemm_ref(ra, refs[g], ii.ravel(), jj.ravel())
            assert np.all(np.abs(got[o:o + r].ravel() - ref) <= gemm_tolerance(ref, ab)), f"group {g}"
        # padding rows of the slot are not written
        assert np.all(got[o + r:int(offs[g + 1])] == 3.0)


def test_grouped_bad_offsets_rejected_on_device():
    k, n = 64, 128
    qa = nb.nvfp4_quantize(_rand(256, k, 5).to(DEV))
    qw = nb.nvfp4_quantize(_rand(2 * n, k, 6).to(DEV))
    gws = torch.ones(2, dtype=torch.float32, device=DEV)
    out = torch.full((256, n), 3.0, dtype=torch.bfloat16, device=DEV)
    offs = torch.tensor([0, 100, 256], dtype=torch.int32, device=DEV)   # 100 not a multiple of 128
    rows = torch.tensor([10, 10], dtype=torch.int32, device=DEV)
    nb.nvfp4_grouped_gemm(offs, rows, qa, qw, gws, n, out=out)
    assert nb.nvfp4_check_status() == 3
    assert torch.all(out == 3.0)
    offs = torch.tensor([0, 128, 512], dtype=torch.int32, device=DEV)   # beyond A's rows
    nb.nvfp4_grouped_gemm(offs, rows, qa, qw, gws, n, out=out)
    assert nb.nvfp4_check_status() == 3


@pytest.mark.parametrize("m,n,k", [(16, 2048, 5120), (100, 4096, 1024), (128, 256, 2048), (1, 512, 256)])
def test_split_k_against_oracle_and_unsplit(m, n, k):
    """Small-M GEMMs split K across SMs when the workspace holds the FP32
    slices: within tolerance of the oracle, deterministic across calls, and
    within tolerance of the unsplit kernel (a 256-byte workspace turns the
    split off)."""
    a = _rand(m, k, m + n + k)
    w = _rand(n, k, 3 * m + n, 0.05)
    qa, ra = _quant_both(a, "split A")
    qw, rw = _quant_both(w, "split W")
    big = nb.Workspace(DEV, 64 << 20)
    small = nb.Workspace(DEV, 256)
    d1 = nb.nvfp4_gemm(qa, qw, workspace=big)
    d2 = nb.nvfp4_gemm(qa, qw, workspace=big)
    d0 = nb.nvfp4_gemm(qa, qw, workspace=small)
    torch.cuda.synchronize()
    assert nb.nvfp4_check_status(big) == 0 and nb.nvfp4_check_status(small) == 0
    assert torch.equal(d1, d2)                                   # split order fixed
    ii, jj = np.meshgrid(np.arange(m), np.arange(n), indexing="ij")
    ref, ab = oracle.gemm_ref(ra, rw, ii.ravel(), jj.ravel())
    tol = gemm_tolerance(ref, ab)
    for d in (d1, d0):
        assert np.all(np.abs(bf16_to_f64(d).ravel() - ref) <= tol)


@pytest.mark.parametrize("m", [1, 15, 16, 17, 33, 48, 64])
@pytest.mark.parametrize("n,k", [(2048, 5120), (300, 192), (128, 64), (1000, 1088)])
def test_small_m_swapped_operands(m, n, k):
    """Few rows of A run with W on the MMA's 128-row side and A's rows
    (padded to a multiple of 16) on its N side, split over K when the
    workspace holds the FP32 slices.  Every output against the oracle, with
    and without splits; the split result is the same on every call."""
    qa, ra = _quant_both(_rand(m, k, 11 * m + n + k), f"small-M A {m}x{k}")
    qw, rw = _quant_both(_rand(n, k, 7 * m + 3 * n + k, 0.02), f"small-M W {n}x{k}")
    ii, jj = np.meshgrid(np.arange(m), np.arange(n), indexing="ij")
    ref, ab = oracle.gemm_ref(ra, rw, ii.ravel(), jj.ravel())
    tol = gemm_tolerance(ref, ab)
    big, small = nb.Workspace(DEV, 64 << 20), nb.Workspace(DEV, 256)
    d1 = nb.nvfp4_gemm(qa, qw, workspace=big)
    d2 = nb.nvfp4_gemm(qa, qw, workspace=big)
    d0 = nb.nvfp4_gemm(qa, qw, workspace=small)
    torch.cuda.synchronize()
    assert nb.nvfp4_check_status(big) == 0 and nb.nvfp4_check_status(small) == 0
    assert torch.equal(d1, d2)
    for d in (d1, d0):
        err = np.abs(bf16_to_f64(d).ravel() - ref)
        bad = np.nonzero(err > tol)[0]
        assert bad.size == 0, f"{bad.size} outside tolerance, first (i,j)={ii.ravel()[bad[:4]]},{jj.ravel()[bad[:4]]}"

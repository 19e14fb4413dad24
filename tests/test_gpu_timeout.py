"""Bounded pipeline waits of the GEMM kernels, exercised on the GPU without a
fault or a hang.

Every mbarrier wait in the GEMM pipelines (single-CTA, CTA-pair, swapped
operands, split-K) gives up after a cycle limit.  Cutting that limit to a
few hundred SM cycles (the library's test hook) makes the first wait on a
real TMA copy run out: the launch must record
NVFP4_ERR_TIMEOUT in the status word, stop every role, let its issued copies
and MMAs finish, release TMEM and exit.  Each wait still ends by itself
(copies land, the limit passes), so nothing here can hang.  After the default
limit is restored the same GEMM, on the same workspace, must match the oracle
and report no error: the context and the library are clean.
"""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_block_scaled_22_b200 import binding as nb
from tests.gpu_util import assert_quantized_equal, bf16_to_f64, gemm_tolerance

pytestmark = pytest.mark.gpu
DEV = "cuda"
TIMEOUT = 7            # NVFP4_ERR_TIMEOUT
TINY_LIMIT = 300       # SM cycles: below any TMA round trip


@pytest.fixture(autouse=True)
def _single_cta_and_default_limit():
    nb.lib()
    prev_pairs = nb.nvfp4_set_gemm_pairs(False)     # the CTA-pair kernel only where a test enables it
    yield
    nb.nvfp4_set_wait_limit_cycles(0)                # back to the default bound
    nb.nvfp4_set_gemm_pairs(prev_pairs)
    nb.nvfp4_check_status()


def _rand(rows, cols, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(rows, cols, generator=g) * scale).to(torch.bfloat16)


def _quant(x, what):
    q = nb.nvfp4_quantize(x.to(DEV))
    st, r = oracle.quantize(x)
    assert st == oracle.OK
    assert_quantized_equal(q, r, what)
    return q, r


def _timed_out_then_clean(run, check, ws):
    """run() under the tiny limit must time out; then run() again under the
    default limit must be clean and pass check()."""
    assert nb.nvfp4_check_status(ws) == 0
    nb.nvfp4_set_wait_limit_cycles(TINY_LIMIT)
    run()
    assert nb.nvfp4_check_status(ws) == TIMEOUT
    nb.nvfp4_set_wait_limit_cycles(0)
    out = run()
    assert nb.nvfp4_check_status(ws) == 0
    check(out)


def _full_check(ra, rw, m, n):
    ii, jj = np.meshgrid(np.arange(m), np.arange(n), indexing="ij")
    ref, ab = oracle.gemm_ref(ra, rw, ii.ravel(), jj.ravel())

    def check(d):
        got = bf16_to_f64(d).ravel()
        assert np.all(np.abs(got - ref) <= gemm_tolerance(ref, ab))
    return check


@pytest.mark.parametrize("m,n,k", [(256, 256, 256), (1000, 1024, 1024)])
def test_dense_gemm_timeout_then_clean(m, n, k):
    qa, ra = _quant(_rand(m, k, m + k), "A")
    qw, rw = _quant(_rand(n, k, n + k + 1, 0.02), "W")
    ws = nb.Workspace(DEV, 256)                      # status word only: no split-K
    _timed_out_then_clean(lambda: nb.nvfp4_gemm(qa, qw, workspace=ws), _full_check(ra, rw, m, n), ws)


@pytest.mark.parametrize("m,n,k", [(256, 256, 256), (768, 1280, 1024)])
def test_pair_gemm_timeout_then_clean(m, n, k):
    """The CTA-pair kernel: a timed-out wait in either CTA stops that CTA's
    roles; the other CTA's waits on the pair's barriers then time out in turn
    (each is bounded), every issued copy and MMA drains before the final
    cluster barrier, and TMEM is released by both CTAs."""
    nb.nvfp4_set_gemm_pairs(True)
    qa, ra = _quant(_rand(m, k, m + k + 7), "A")
    qw, rw = _quant(_rand(n, k, n + k + 8, 0.02), "W")
    ws = nb.Workspace(DEV, 256)
    _timed_out_then_clean(lambda: nb.nvfp4_gemm(qa, qw, workspace=ws), _full_check(ra, rw, m, n), ws)


@pytest.mark.parametrize("m", [16, 100])
def test_small_m_gemm_timeout_then_clean(m):
    """m = 16: the swapped-operand kernel with K splits; m = 100: the split-K
    instance of the 128x256 kernel."""
    n, k = 2048, 5120
    qa, ra = _quant(_rand(m, k, 3), "A")
    qw, rw = _quant(_rand(n, k, 4, 0.02), "W")
    ws = nb.Workspace(DEV, 64 << 20)
    _timed_out_then_clean(lambda: nb.nvfp4_gemm(qa, qw, workspace=ws), _full_check(ra, rw, m, n), ws)


def test_grouped_gemm_timeout_then_clean():
    rows, n, k = [5, 130, 0, 128], 256, 512
    offs = np.concatenate([[0], np.cumsum([-(-r // 128) * 128 for r in rows])]).astype(np.int32)
    a = torch.zeros(int(offs[-1]), k, dtype=torch.bfloat16)
    for g, r in enumerate(rows):
        a[offs[g]:offs[g] + r] = _rand(r, k, 10 + g)
    qa, ra = _quant(a, "grouped A")
    w_all = _rand(len(rows) * n, k, 20, 0.02)
    qw, rw = _quant(w_all, "stacked W")              # one tensor scale shared by the groups
    gws = qw.global_scale.repeat(len(rows))
    ws = nb.Workspace(DEV, 256)
    off_d = torch.from_numpy(offs).to(DEV)
    rows_d = torch.tensor(rows, dtype=torch.int32, device=DEV)

    def run():
        out = torch.zeros((a.shape[0], n), dtype=torch.bfloat16, device=DEV)
        return nb.nvfp4_grouped_gemm(off_d, rows_d, qa, qw, gws, n, out=out, workspace=ws)

    def check(d):
        got = bf16_to_f64(d)
        for g, r in enumerate(rows):
            if r == 0:
                continue
            o = int(offs[g])
            ii, jj = np.meshgrid(np.arange(o, o + r), np.arange(n) + g * n, indexing="ij")
            ref, ab = oracle.gemm_ref(ra, rw, ii.ravel(), jj.ravel())
            assert np.all(np.abs(got[o:o + r].ravel() - ref) <= gemm_tolerance(ref, ab)), f"group {g}"

    _timed_out_then_clean(run, check, ws)


def test_mxfp4_gemm_timeout_then_clean():
    m, n, k = 256, 512, 512
    a, w = _rand(m, k, 31), _rand(n, k, 32, 0.02)
    qa, qw = nb.nvfp4_quantize_mx(a.to(DEV)), nb.nvfp4_quantize_mx(w.to(DEV))
    st, ra = oracle.quantize_mx(a)
    st2, rw = oracle.quantize_mx(w)
    assert st == st2 == oracle.OK
    assert np.array_equal(qa.codes.cpu().numpy(), ra.codes)
    assert np.array_equal(qw.scales.cpu().numpy(), rw.scales)
    ws = nb.Workspace(DEV, 256)
    ii, jj = np.meshgrid(np.arange(m), np.arange(n), indexing="ij")
    ref, ab = oracle.gemm_ref_mx(ra, rw, ii.ravel(), jj.ravel())

    def check(d):
        assert np.all(np.abs(bf16_to_f64(d).ravel() - ref) <= gemm_tolerance(ref, ab))

    _timed_out_then_clean(lambda: nb.nvfp4_gemm_mx(qa, qw, workspace=ws), check, ws)

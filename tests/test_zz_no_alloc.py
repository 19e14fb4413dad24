"""nvfp4_quantize_noalloc: the quantize entry point for callers that cannot
allocate device memory (graph capture, allocation-free hot paths, hosts whose
pool owns the device).  Its scratch is a fixed array inside the library and
every call shares it, so the checks below run it twice in a row on different
tensors and compare each result with nvfp4_quantize, which uses a
caller-provided workspace.  Codes, scales and the tensor scale must match
bit for bit (the tolerance the quantize tests use).

The file name sorts last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from nvfp4_block_scaled_22_b200 import binding as nb

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _tensor(rows, cols, seed, scale):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, cols, generator=g) * scale
    x.view(-1)[torch.randint(0, x.numel(), (x.numel() // 300,), generator=g)] *= 40
    return x.to(torch.bfloat16).to(DEV)


def _noalloc(x, layout, global_supplied=False, out=None):
    rows, cols = x.shape
    if out is None:
        out = nb.NVFP4Tensor.empty(rows, cols, layout, DEV)
    t = out.c_struct()
    st = nb.lib().nvfp4_quantize_noalloc(x.data_ptr(), x.stride(0), C.byref(t),
                                         int(global_supplied),
                                         torch.cuda.current_stream().cuda_stream)
    assert st == 0, nb.nvfp4_status_string(st)
    return out


def _same(a: nb.NVFP4Tensor, b: nb.NVFP4Tensor):
    torch.cuda.synchronize()
    assert torch.equal(a.codes, b.codes)
    assert torch.equal(a.scales, b.scales)
    assert np.float32(a.global_scale.item()) == np.float32(b.global_scale.item())


@pytest.mark.parametrize("layout", [nb.SF_SWIZZLED, nb.SF_LINEAR])
def test_two_calls_in_a_row_match_workspace_entry_point(layout):
    first = _tensor(1000, 4096, 1, 1.0)
    second = _tensor(257, 1040, 2, 1e-3)      # different shape and amax
    got1 = _noalloc(first, layout)
    got2 = _noalloc(second, layout)
    ref1 = nb.nvfp4_quantize(first, layout=layout)
    ref2 = nb.nvfp4_quantize(second, layout=layout)
    assert nb.nvfp4_check_status() == 0
    _same(got1, ref1)
    _same(got2, ref2)


def test_supplied_scale_and_in_band_error_reporting():
    x = _tensor(300, 512, 3, 2.0)
    ref = nb.nvfp4_quantize(x)
    out = nb.NVFP4Tensor.empty(300, 512, device=DEV)
    out.global_scale.copy_(ref.global_scale)
    _same(_noalloc(x, nb.SF_SWIZZLED, global_supplied=True, out=out), ref)
    bad = x.clone()
    bad[7, 9] = float("nan")
    err = _noalloc(bad, nb.SF_SWIZZLED)
    torch.cuda.synchronize()
    assert torch.isnan(err.global_scale).item()
    # the shared status word was cleared: the next call is clean again
    _same(_noalloc(x, nb.SF_SWIZZLED), ref)
    assert nb.nvfp4_check_status() == 0

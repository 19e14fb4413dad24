"""CPU checks of the C ABI library: it loads, exports every declared entry
point, and its size arithmetic matches the storage rules.  No kernel runs."""
import os
import re

import pytest

import oracle
from nvfp4_block_scaled_22_b200 import binding
from nvfp4_block_scaled_22_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return binding.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "nvfp4.h")).read()
    return set(re.findall(r"NVFP4_API[^;(]*?\b(nvfp4_\w+)\s*\(", src))


def test_header_declares_binding_symbols():
    assert _declared() == set(binding.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name
    out = os.popen(f"nm -D --defined-only {binding.LIB_PATH}").read()
    exported = set(re.findall(r" T (nvfp4_\w+)", out))
    assert _declared() <= exported


def test_sizes_match_storage_rules(lib):
    for rows, cols in [(1, 16), (128, 256), (130, 80), (4096, 6144), (131072, 1024)]:
        assert binding.nvfp4_codes_bytes(rows, cols) == rows * cols // 2
        for layout in (binding.SF_SWIZZLED, binding.SF_LINEAR):
            assert binding.nvfp4_scales_bytes(rows, cols, layout) == \
                oracle.scales_bytes(rows, cols, layout)
    for op in range(5):
        assert binding.nvfp4_workspace_bytes(op) >= 16


def test_status_strings_and_version(lib):
    assert binding.nvfp4_status_string(0) == "ok"
    for s in range(1, 10):
        assert binding.nvfp4_status_string(s) not in ("", "unknown status")
    assert lib.nvfp4_version() >= 100


def test_host_side_argument_errors_need_no_gpu(lib):
    """Argument validation returns before any CUDA call."""
    t = binding.CTensor(0, 0, 0, 4, 24, 0)
    st = lib.nvfp4_quantize(16, 32, t, 0, 16, 1 << 16, 0)
    assert st == 3                                  # NVFP4_ERR_SHAPE
    t = binding.CTensor(16, 16, 0, 4, 32, 0)         # no global pointer
    assert lib.nvfp4_quantize(16, 32, t, 0, 16, 1 << 16, 0) == 1
    t = binding.CTensor(16, 16, 16, 4, 32, 7)        # bad layout
    assert lib.nvfp4_quantize(16, 32, t, 0, 16, 1 << 16, 0) == 1
    t = binding.CTensor(16, 16, 16, 4, 32, 0)
    assert lib.nvfp4_quantize(8, 32, t, 0, 16, 1 << 16, 0) == 2   # x misaligned
    assert lib.nvfp4_quantize(16, 32, t, 0, 16, 8, 0) == 6        # workspace too small
    t = binding.CTensor(16, 16, 16, 4, 32, 0)
    assert lib.nvfp4_quantize_rht(16, 32, 0x10000, t, 0, 16, 1 << 16, 0) == 1   # mask > 16 bits
    t = binding.CTensor(16, 16, 16, 4, 24, 0)
    assert lib.nvfp4_quantize_rht(16, 32, 0xFFFF, t, 0, 16, 1 << 16, 0) == 3    # cols % 16
    t = binding.CTensor(16, 16, 16, 12, 32, 0)
    assert lib.nvfp4_quantize_t(16, 32, 0, 0, t, 0, 16, 1 << 16, 0) == 3        # x columns % 8
    t = binding.CTensor(16, 16, 16, 16, 32, 0)
    assert lib.nvfp4_quantize_t(16, 32, 2, 0, t, 0, 16, 1 << 16, 0) == 1        # rht flag
    t = binding.CTensor(16, 16, 16, 40, 32, 0)
    tt = binding.CTensor(16, 16, 16, 32, 40, 0)
    assert lib.nvfp4_quantize_2d(16, 32, t, tt, 0, 16, 1 << 16, 0) == 3         # rows % 16 with W^T
    tt = binding.CTensor(16, 16, 16, 32, 48, 0)
    assert lib.nvfp4_quantize_2d(16, 32, t, tt, 0, 16, 1 << 16, 0) == 3         # W^T shape
    t = binding.CTensor(16, 16, 16, 16, 32, 0)
    assert lib.nvfp4_quantize_sr(16, 32, 2, 0, 0, 1, t, 0, 16, 1 << 16, 0) == 1  # transposed flag
    assert lib.nvfp4_quantize_sr(16, 32, 0, 0, 1 << 16, 1, t, 0, 16, 1 << 16, 0) == 1   # mask
    t = binding.CTensor(16, 16, 16, 12, 32, 0)
    assert lib.nvfp4_quantize_sr(16, 32, 1, 0, 0, 1, t, 0, 16, 1 << 16, 0) == 3  # x columns % 8
    t = binding.CTensor(16, 16, 0, 4, 48, 0)
    assert lib.nvfp4_quantize_mx(16, 48, t, 16, 1 << 16, 0) == 3                 # cols % 32
    assert lib.nvfp4_mx_scales_bytes(256, 1024, 1) == 256 * 32
    assert lib.nvfp4_moe_combine(16, 16, 4, 16, 16, 4, 0, 16, 16, 16, 0) == 1    # topk 0
    assert lib.nvfp4_moe_combine(16, 16, 4, 16, 16, 4, 2, 12, 16, 16, 0) == 3    # hidden % 8
    a = binding.CTensor(16, 16, 16, 128, 96, 0)      # K % 64 != 0
    w = binding.CTensor(16, 16, 16, 256, 96, 0)
    assert lib.nvfp4_gemm(a, w, 16, 256, 16, 1 << 16, 0) == 3


def test_attention_argument_errors_and_workspace_size(lib):
    """Host checks of the attention read return before any CUDA call; the
    workspace holds per chunk and query head the 128 outputs, m and l."""
    k = binding.CTensor(16, 16, 16, 1000, 1024, 1)      # 8 KV heads x 128, linear
    ws = 1 << 20
    assert lib.nvfp4_attention_decode(16, 128, 64, k, k, 8, 0.1, 16, 128, 16, ws, 0) != 3
    assert lib.nvfp4_attention_decode(16, 128, 60, k, k, 8, 0.1, 16, 128, 16, ws, 0) == 3  # heads
    assert lib.nvfp4_attention_decode(16, 128, 72, k, k, 8, 0.1, 16, 128, 16, ws, 0) == 3  # group 9
    assert lib.nvfp4_attention_decode(16, 128, 64, k, k, 4, 0.1, 16, 128, 16, ws, 0) == 3  # cols
    sw = binding.CTensor(16, 16, 16, 1000, 1024, 0)      # swizzled scales
    assert lib.nvfp4_attention_decode(16, 128, 64, sw, sw, 8, 0.1, 16, 128, 16, ws, 0) == 3
    v = binding.CTensor(16, 16, 16, 999, 1024, 1)
    assert lib.nvfp4_attention_decode(16, 128, 64, k, v, 8, 0.1, 16, 128, 16, ws, 0) == 3  # rows
    assert lib.nvfp4_attention_decode(18, 128, 64, k, k, 8, 0.1, 16, 128, 16, ws, 0) == 2  # q align
    assert lib.nvfp4_attention_decode(16, 129, 64, k, k, 8, 0.1, 16, 128, 16, ws, 0) == 2  # odd ldq
    assert lib.nvfp4_attention_decode(16, 128, 64, k, k, 8, float("nan"), 16, 128, 16, ws, 0) == 1
    assert lib.nvfp4_attention_decode(16, 128, 64, k, k, 8, 0.1, 16, 128, 16, 300, 0) == 6  # ws
    # 131072 tokens, 8 KV heads: 18 chunks of 7424 tokens; 64 query heads
    need = binding.nvfp4_workspace_bytes(binding.OP_ATTENTION, 131072, 64, 8)
    assert need == 256 + 18 * 64 * 130 * 4
    assert binding.nvfp4_workspace_bytes(binding.OP_ATTENTION, 0, 64, 8) == 256
    # one KV head: up to 148 chunks, never more chunks than 256-token sub-tiles
    assert binding.nvfp4_workspace_bytes(binding.OP_ATTENTION, 1000, 2, 1) == 256 + 4 * 2 * 130 * 4


def test_attention_chunking_matches_the_library(lib):
    """The chunk count the attention parity tolerance assumes is the one
    the library's workspace size implies."""
    from tests.gpu_util import attention_chunking
    for tokens in (1, 255, 256, 257, 1000, 4099, 20000, 131072, 1 << 20):
        for heads_kv in (1, 2, 3, 8, 37, 200):
            heads_q = heads_kv * 2
            ws = binding.nvfp4_workspace_bytes(binding.OP_ATTENTION, tokens, heads_q, heads_kv)
            n_lib = (ws - 256) // (heads_q * 130 * 4)
            assert n_lib == attention_chunking(tokens, heads_kv)[1], (tokens, heads_kv)

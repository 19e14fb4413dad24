"""Pins of the CPU oracle against what the pages and the mathematics fix.

None of these re-types an oracle formula: each checks a value the pages
print, a brute-force search, a closed form, an invariant or an independent
library routine.
"""
import ctypes as C
import math
import os

import numpy as np
import pytest
import torch

import oracle
from tests.golden_io import read_kv, read_lines
from tests.pins.build import build as build_pins


def _grid_from_pages():
    vals = [float(v) for v in read_lines("e2m1_values.txt")]
    assert len(vals) == 16
    return vals


def _e4m3_table():
    """Non-negative finite E4M3 values built from the format's definition:
    bias 7, exponent field 0 subnormal (m/8 * 2^-6), S.1111.111 NaN."""
    vals, codes = [], []
    for e in range(16):
        for m in range(8):
            if e == 15 and m == 7:
                continue
            v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
            vals.append(v)
            codes.append((e << 3) | m)
    return vals, codes


# ------------------------------------------------------------------ formats
def test_e2m1_decode_matches_page_value_list():
    grid = _grid_from_pages()
    for code in range(16):
        got = oracle.e2m1_decode(code)
        assert got == grid[code] and math.copysign(1, got) == math.copysign(1, grid[code])
    # 16 codes, 15 distinct values (+0 and -0 are one value)
    assert len({oracle.e2m1_decode(c) for c in range(16)}) == 15
    assert max(grid) == 6.0


def test_e4m3_decode_definition():
    vals, codes = _e4m3_table()
    assert len(vals) == 127
    for v, c in zip(vals, codes):
        assert oracle.e4m3_decode(c) == v
        assert oracle.e4m3_decode(c | 0x80) == -v
    assert max(vals) == 448.0 and min(v for v in vals if v > 0) == 2.0 ** -9
    assert math.isnan(oracle.e4m3_decode(0x7F)) and math.isnan(oracle.e4m3_decode(0xFF))


@pytest.mark.parametrize("y,code", [
    (0.25, 0x0), (0.2500001, 0x1), (0.75, 0x2), (1.25, 0x2), (1.75, 0x4), (2.5, 0x4),
    (3.5, 0x6), (5.0, 0x6), (5.0000005, 0x7), (6.0, 0x7), (7.0, 0x7), (1e30, 0x7),
    (-0.1, 0x8), (-0.0, 0x8), (0.0, 0x0), (-3.4, 0xD), (0.74, 0x1), (1e-45, 0x0),
])
def test_e2m1_rounding_points(y, code):
    # nearest value, ties to the even code, saturation at 6, sign kept
    assert oracle.e2m1_rne(y) == code


@pytest.mark.parametrize("v,code", [
    (2.0 ** -10, 0x00), (2.0 ** -10 * 1.000001, 0x01), (2.0 ** -9, 0x01), (3 * 2.0 ** -10, 0x02),
    (1.0625, 0x38), (1.1875, 0x3A), (448.0, 0x7E), (463.9, 0x7E), (464.0, 0x7E), (1e9, 0x7E),
    (0.0, 0x00), (2.0 ** -6, 0x08), (7 * 2.0 ** -9, 0x07), (15 * 2.0 ** -10, 0x08),
])
def test_e4m3_rounding_points(v, code):
    assert oracle.e4m3_rne(v) == code


def _sweep(which, vals, codes):
    L = C.CDLL(build_pins())
    L.pins_sweep.restype = C.c_int64
    L.pins_sweep.argtypes = [C.c_int, C.c_void_p, C.c_void_p, C.c_int, C.c_int,
                             C.POINTER(C.c_int64)]
    v = np.ascontiguousarray(vals, np.float64)
    c = np.ascontiguousarray(codes, np.uint8)
    steps = C.c_int64()
    bad = L.pins_sweep(which, v.ctypes.data, c.ctypes.data, len(v), os.cpu_count() or 4,
                       C.byref(steps))
    return bad, steps.value


def test_e2m1_exhaustive_against_brute_force():
    grid = _grid_from_pages()[:8]
    bad, steps = _sweep(0, grid, list(range(8)))
    assert bad == 0
    assert steps == 7          # one step per decision point


def test_e4m3_exhaustive_against_brute_force():
    vals, codes = _e4m3_table()
    bad, steps = _sweep(1, vals, codes)
    assert bad == 0
    assert steps == 126


def test_bf16_rounding_matches_torch():
    g = torch.Generator().manual_seed(7)
    x = torch.cat([torch.randn(100000, generator=g) * 10 ** torch.randint(-40, 38, (100000,), generator=g).float(),
                   torch.tensor([0.0, -0.0, 1.00390625, 1.01171875, 3.0e38, 1e-40, -1e-41])])
    x = x[torch.isfinite(x)]
    ref = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.f32_to_bf16(float(v)) for v in x.numpy()], np.uint16)
    assert np.array_equal(got, ref)


# ------------------------------------------------------------ scale layouts
def test_swizzled_layout_is_a_bijection_onto_padded_buffer():
    for rows, cols in [(128, 256), (130, 80), (1, 16), (256, 64 * 5)]:
        s = cols // 16
        sp = (s + 3) // 4 * 4
        rp = (rows + 127) // 128 * 128
        assert oracle.scales_bytes(rows, cols, oracle.SF_SWIZZLED) == rp * sp
        offs = {oracle.sf_offset(r, c, rows, cols, oracle.SF_SWIZZLED)
                for r in range(rp) for c in range(sp)}
        assert offs == set(range(rp * sp))


def test_swizzled_layout_points():
    # 128x4 tile: row r%32 at 16 B, (r%128)/32 at 4 B, scale column c%4 at
    # 1 B; tiles run along the scale columns first (cols=1024 -> 64 scale
    # columns -> 16 tiles per 128 rows).
    rows, cols = 256, 1024
    pts = {(0, 0): 0, (1, 0): 16, (31, 0): 496, (32, 0): 4, (96, 0): 12, (0, 1): 1,
           (0, 3): 3, (0, 4): 512, (5, 7): 5 * 16 + 512 + 3, (128, 0): 16 * 512,
           (200, 9): (16 + 2) * 512 + 8 * 16 + 2 * 4 + 1}
    for (r, c), off in pts.items():
        assert oracle.sf_offset(r, c, rows, cols, oracle.SF_SWIZZLED) == off


# --------------------------------------------------------------- storage
def test_storage_is_4p5_bits_per_value():
    facts = read_kv("kv_cache_sizes.txt")
    for rows, cols in [(128, 64), (256, 4096), (1024, 128)]:
        n = rows * cols
        for layout in (oracle.SF_SWIZZLED, oracle.SF_LINEAR):
            total = n // 2 + oracle.scales_bytes(rows, cols, layout)
            assert total == n * facts["nvfp4_bytes_per_value"]
            assert total * 8 / n == facts["nvfp4_bits_per_value"]


def test_kv_cache_worked_example():
    f = read_kv("kv_cache_sizes.txt")
    per_token_values = 2 * f["layers"] * f["kv_heads"] * f["head_dim"]
    assert per_token_values == f["values_per_token"]
    # one token of one (layer, K/V) tensor is a [heads, head_dim] row
    rows, cols = 1, f["kv_heads"] * f["head_dim"]
    per_tensor_token = rows * cols // 2 + oracle.scales_bytes(rows, cols, oracle.SF_LINEAR)
    per_token = per_tensor_token * 2 * f["layers"]
    assert per_token == f["nvfp4_bytes_per_token"] == 36 * 1024
    assert per_token_values * f["bf16_bytes_per_value"] == f["bf16_bytes_per_token"]
    assert per_token_values * f["fp8_bytes_per_value"] == f["fp8_bytes_per_token"]
    assert per_token * f["context_tokens"] == f["nvfp4_bytes_per_context"] == int(4.5 * 2 ** 30)
    assert f["bf16_bytes_per_token"] * f["context_tokens"] == f["bf16_bytes_per_context"]
    assert abs(16 / 4.5 - f["nvfp4_vs_fp16_ratio_approx"]) < 0.1
    assert abs(8 / 4.5 - f["nvfp4_vs_fp8_ratio_approx"]) < 0.05


# --------------------------------------------------------------- quantize
def _rand_bf16(rows, cols, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(rows, cols, generator=g) * scale).to(torch.bfloat16)


def _codes_unpacked(q):
    lo = q.codes & 15
    hi = q.codes >> 4
    return np.stack([lo, hi], -1).reshape(q.rows, q.cols)


def _scales_grid(q):
    s = np.zeros((q.rows, q.cols // 16), np.uint8)
    for r in range(q.rows):
        for c in range(q.cols // 16):
            s[r, c] = q.scales[oracle.sf_offset(r, c, q.rows, q.cols, q.layout)]
    return s


def test_global_scale_definition():
    for amax in (1.0, 6.0, 3.14159, 1e-20, 1e20):
        st, g = oracle.global_scale(amax)
        assert st == oracle.OK and g == np.float32(np.float32(2688.0) / np.float32(amax))
    assert oracle.global_scale(0.0) == (oracle.OK, 1.0)
    assert oracle.global_scale(1e-36)[0] == oracle.ERR_RANGE
    assert oracle.global_scale(float("inf"))[0] == oracle.ERR_NONFINITE


def test_nonfinite_input_is_reported():
    x = _rand_bf16(4, 32, 1)
    x[2, 5] = float("nan")
    assert oracle.quantize(x)[0] == oracle.ERR_NONFINITE
    x[2, 5] = float("inf")
    assert oracle.quantize(x)[0] == oracle.ERR_NONFINITE


def test_block_amax_code_is_six():
    """The block amax lands on the FP4 maximum for every block whose scale is
    a normal E4M3 number: RN(amax_b * g / s) lies in (5, 7)."""
    x = _rand_bf16(64, 512, 2)
    x[:, 37] *= 40                       # outlier column squeezes other blocks
    st, q = oracle.quantize(x)
    assert st == oracle.OK
    mags = np.array([abs(oracle.e2m1_decode(c)) for c in range(16)])
    vals = mags[_codes_unpacked(q)].reshape(64, 32, 16)
    s = _scales_grid(q)
    normal = s >= 0x08
    assert normal.sum() > 1000
    assert np.all(vals.max(-1)[normal] == 6.0)


def test_codes_are_nearest_grid_points_of_the_scaled_input():
    """Per element, the code is the nearest grid value to x*e (numpy float32)
    with e = g / s per block: |x*e - value(code)| <= half the local gap."""
    x = _rand_bf16(32, 256, 3, scale=5.0)
    st, q = oracle.quantize(x)
    xs = oracle.bf16_to_f32(oracle.bf16_bits(x))
    s = _scales_grid(q)
    sval = np.array([oracle.e4m3_decode(int(b)) for b in range(256)], np.float32)[s]
    e = np.where(sval > 0, np.float32(q.g) / sval, np.float32(0)).astype(np.float32)
    y = (xs.reshape(32, 16, 16) * e[:, :, None]).reshape(32, 256).astype(np.float32)
    mags = np.array([abs(oracle.e2m1_decode(c)) for c in range(16)])
    v = mags[_codes_unpacked(q)]
    a = np.abs(y)
    gap = np.where(a < 2, 0.5, np.where(a < 4, 1.0, 2.0))
    assert np.all(np.abs(np.minimum(a, 6) - v) <= gap / 2 + 1e-7)


def test_zero_blocks_and_zero_tensor():
    x = _rand_bf16(8, 64, 4)
    x[3, 16:32] = 0.0
    st, q = oracle.quantize(x)
    s = _scales_grid(q)
    assert s[3, 1] == 0
    assert np.all(_codes_unpacked(q)[3, 16:32] == 0)
    y = q.dequantize()
    assert np.all(y[3, 16:32] == 0)          # +0 bit pattern
    z = torch.zeros(8, 64, dtype=torch.bfloat16)
    st, q = oracle.quantize(z)
    assert st == oracle.OK and q.g == 1.0
    assert not q.codes.any() and not q.scales.any()
    assert not q.dequantize().any()


def test_exact_round_trip_of_representable_tensor():
    """X = c * 2^k_b with c on the E2M1 grid, a |c| = 6 in every nonzero block
    and k_max - k_b <= 14: every scale is exact, so the round trip is exact."""
    rng = np.random.default_rng(5)
    rows, cols = 64, 256
    grid = np.array([float(v) for v in read_lines("e2m1_values.txt")], np.float32)
    c = grid[rng.integers(0, 16, (rows, cols // 16, 16))]
    pos = rng.integers(0, 16, (rows, cols // 16))
    sgn = rng.choice([-1.0, 1.0], (rows, cols // 16))
    c[np.arange(rows)[:, None], np.arange(cols // 16)[None, :], pos] = 6.0 * sgn
    kmax = 3
    k = rng.integers(kmax - 14, kmax + 1, (rows, cols // 16))
    k[0, 0] = kmax
    xv = c * np.exp2(k)[:, :, None].astype(np.float32)
    xv[7, 3] = 0.0                                     # an all-zero block
    xv = xv.reshape(rows, cols).astype(np.float32)
    x = torch.from_numpy(xv).to(torch.bfloat16)
    assert torch.equal(x.float(), torch.from_numpy(xv))   # exact in BF16
    for layout in (oracle.SF_SWIZZLED, oracle.SF_LINEAR):
        st, q = oracle.quantize(x, layout)
        assert st == oracle.OK and q.g == np.float32(448 * 2.0 ** -kmax)
        y = q.dequantize()
        assert np.array_equal(y, oracle.bf16_bits(x))     # -0 stays -0


def test_dequantize_error_bound():
    """|x - x_hat| <= d_b (half the widest grid gap, 2, times the block
    factor d_b = s/g) plus BF16 rounding of x_hat."""
    x = _rand_bf16(16, 512, 6, scale=3.0)
    st, q = oracle.quantize(x)
    xs = oracle.bf16_to_f32(oracle.bf16_bits(x)).reshape(16, 32, 16).astype(np.float64)
    xh = oracle.bf16_to_f32(q.dequantize()).reshape(16, 32, 16).astype(np.float64)
    s = _scales_grid(q).astype(np.int64)
    d = np.array([oracle.e4m3_decode(int(b)) for b in range(256)])[s] / float(q.g)
    err = np.abs(xs - xh)
    assert np.all(err <= d[:, :, None] * (1 + 2 ** -7) + np.abs(xh) * 2 ** -8)


# -------------------------------------------------------------------- GEMM
def test_gemm_fp64_equals_integer_exact_sum_tiny():
    for (m, n, k), seed in zip([(1, 1, 64), (3, 5, 64), (8, 8, 128), (7, 2, 128)], range(4)):
        a = _rand_bf16(m, k, 10 + seed)
        w = _rand_bf16(n, k, 20 + seed, scale=0.02)
        _, qa = oracle.quantize(a)
        _, qw = oracle.quantize(w)
        ii, jj = np.meshgrid(np.arange(m), np.arange(n), indexing="ij")
        ref, ab = oracle.gemm_ref(qa, qw, ii.ravel(), jj.ravel())
        for t, (i, j) in enumerate(zip(ii.ravel(), jj.ravel())):
            exact = oracle.dot_exact_i64(qa, qw, int(i), int(j))
            val = exact / 2.0 ** 20 / (float(qa.g) * float(qw.g))
            assert abs(ref[t] - val) <= 1e-12 * ab[t] + 1e-300
            assert ab[t] >= abs(ref[t])


def test_gemm_one_hot_rows_select_weight_columns():
    """A with one 1.0 per row (code 0x2, scale 1.0 = E4M3 0x38, g = 1) gives
    D[i, j] = What[j, p(i)]: pins D = A * W^T (no transposed operand)."""
    m, n, k = 8, 6, 64
    rng = np.random.default_rng(9)
    p = rng.permutation(k)[:m]
    codes = np.zeros((m, k // 2), np.uint8)
    for i in range(m):
        codes[i, p[i] // 2] |= (0x2 << 4) if p[i] % 2 else 0x2
    scales = np.zeros(oracle.scales_bytes(m, k, oracle.SF_LINEAR), np.uint8)
    scales[:] = 0x38
    qa = oracle.Quantized(codes, scales, 1.0, m, k, oracle.SF_LINEAR)
    w = _rand_bf16(n, k, 30)
    _, qw = oracle.quantize(w, oracle.SF_LINEAR)
    ii, jj = np.meshgrid(np.arange(m), np.arange(n), indexing="ij")
    ref, _ = oracle.gemm_ref(qa, qw, ii.ravel(), jj.ravel())
    e2m1 = np.array([oracle.e2m1_decode(c) for c in range(16)])
    e4m3 = np.array([oracle.e4m3_decode(b) for b in range(256)])
    for t, (i, j) in enumerate(zip(ii.ravel(), jj.ravel())):
        kk = p[i]
        byte = qw.codes[j, kk // 2]
        code = (byte >> 4) if kk % 2 else (byte & 15)
        s = e4m3[qw.scales[j * (k // 16) + kk // 16]]
        assert ref[t] == e2m1[code] * s / float(qw.g)

"""Pins of the oracle's MXFP4 (the format the pages compare NVFP4 with:
"NVIDIA shrank GLM-5.2 to 4 bits" section 3, blocks of 32 with a
power-of-two E8M0 scale; KV page "FP4 formats compared", about 4.25 bits
per value)."""
import math

import numpy as np
import torch

import oracle

GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16)


def _rand(rows, cols, seed, outliers=0.01):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols))
    x[rng.random((rows, cols)) < outliers] *= 40
    return _bf16(x)


def _nibbles(q):
    c = np.zeros((q.rows, q.cols), np.uint8)
    c[:, 0::2], c[:, 1::2] = q.codes & 15, q.codes >> 4
    return c


def test_ue8m0_is_a_power_of_two():
    for b in range(255):
        assert oracle.ue8m0_decode(b) == 2.0 ** (b - 127)
    assert math.isnan(oracle.ue8m0_decode(255))


def test_storage_is_4_25_bits_per_value():
    """Codes plus one scale byte per block of 32 (the block size of the
    GLM page's glossary, tests/golden/format_facts.txt): 4.25 bits per value
    (KV page, "FP4 formats compared")."""
    from tests.golden_io import read_kv
    assert read_kv("format_facts.txt")["mxfp4_block_size"] == 32
    rows, cols = 256, 1024
    _, q = oracle.quantize_mx(_rand(rows, cols, 1))
    bits = (q.codes.size + q.scales.size) * 8 / (rows * cols)
    assert bits == 4.25


def test_scale_puts_the_block_max_in_the_top_binade():
    """amax * 2^-X lies in [4, 8) for every block (checked with math.frexp,
    not the oracle's exponent routine), so the block max encodes as 4 or 6."""
    x = _rand(64, 256, 2)
    xf = oracle.bf16_to_f32(oracle.bf16_bits(x)).astype(np.float64)
    _, q = oracle.quantize_mx(x, oracle.SF_LINEAR)
    nib = _nibbles(q)
    for r in range(64):
        for b in range(8):
            amax = np.abs(xf[r, 32 * b:32 * b + 32]).max()
            X = int(q.scales[r * 8 + b]) - 127
            assert 4.0 <= amax * 2.0 ** -X < 8.0
            assert math.frexp(amax)[1] - 3 == X
            top = GRID[nib[r, 32 * b:32 * b + 32] & 7].max()
            assert top in (4.0, 6.0)


def test_codes_are_nearest_grid_points_and_round_trip():
    x = _rand(32, 128, 3)
    xf = oracle.bf16_to_f32(oracle.bf16_bits(x)).astype(np.float64)
    _, q = oracle.quantize_mx(x, oracle.SF_LINEAR)
    nib = _nibbles(q)
    for r in range(32):
        for c in range(128):
            y = min(abs(xf[r, c]) * 2.0 ** -(int(q.scales[r * 4 + c // 32]) - 127), 6.0)
            d = np.abs(GRID - y)
            best = np.flatnonzero(d == d.min())
            k = nib[r, c] & 7
            assert k in best and (len(best) == 1 or k % 2 == 0)      # ties to even code
    # representable values round-trip: c * 2^k with a 6 in every block
    rng = np.random.default_rng(4)
    vals = rng.choice(GRID, (8, 64)) * rng.choice([-1, 1], (8, 64))
    vals[:, ::32] = 6.0
    e = rng.integers(-6, 6, (8, 2)).repeat(32, axis=1)
    xr = _bf16(vals * 2.0 ** e)
    _, qr = oracle.quantize_mx(xr)
    assert np.array_equal(oracle.bf16_to_f32(qr.dequantize()), oracle.bf16_to_f32(oracle.bf16_bits(xr)))


def test_zero_blocks_and_nonfinite():
    x = _rand(4, 64, 5)
    x[1, :32] = 0.0
    st, q = oracle.quantize_mx(x, oracle.SF_LINEAR)
    assert st == oracle.OK and q.scales[1 * 2] == 0 and not np.any(_nibbles(q)[1, :32] & 7)
    x[2, 5] = float("inf")
    assert oracle.quantize_mx(x)[0] == oracle.ERR_NONFINITE


def test_gemm_reference_against_exact_integers():
    a = _rand(6, 128, 6)
    w = _rand(5, 128, 7)
    _, qa = oracle.quantize_mx(a, oracle.SF_LINEAR)
    _, qw = oracle.quantize_mx(w, oracle.SF_LINEAR)
    ii, jj = np.meshgrid(np.arange(6), np.arange(5), indexing="ij")
    ref, ab = oracle.gemm_ref_mx(qa, qw, ii.ravel(), jj.ravel())
    na, nw = _nibbles(qa), _nibbles(qw)
    for t, (i, j) in enumerate(zip(ii.ravel(), jj.ravel())):
        tot = 0
        for c in range(128):
            # 2 * e2m1 is an integer; scales are powers of two
            ia = int(round(2 * GRID[na[i, c] & 7])) * (-1 if na[i, c] & 8 else 1)
            iw = int(round(2 * GRID[nw[j, c] & 7])) * (-1 if nw[j, c] & 8 else 1)
            sa = int(qa.scales[i * 4 + c // 32]) - 127
            sw = int(qw.scales[j * 4 + c // 32]) - 127
            tot += ia * iw * 2 ** (sa + sw + 300)       # shift to keep integers
        assert ref[t] == tot / 4 / 2.0 ** 300
        assert ab[t] >= abs(ref[t])


def test_shared_exponent_closed_form_and_clamps():
    """X = floor(log2 amax) - 2 for every finite amax, computed here from the
    float's own bit pattern (not frexp), then clamped to [-127, 127]; an
    all-zero block takes -127."""
    rng = np.random.default_rng(9)
    bits = rng.integers(1, 0x7F800000, 4000, dtype=np.int64).astype(np.uint32)
    extra = np.array([1, 2, 0x007FFFFF, 0x00800000, 0x40800000, 0x40C00000, 0x407FFFFF,
                      0x7F7FFFFF, 0x3F800000], np.uint32)      # subnormals, 4, 6, <4, max, 1
    for b in np.concatenate([bits, extra]):
        v = float(np.uint32(b).view(np.float32))
        e = int(b) >> 23
        if e == 0:                                    # subnormal: 2^-149 * mantissa
            fl = int(b).bit_length() - 1 - 149
        else:
            fl = e - 127
        want = max(-127, min(127, fl - 2))
        assert oracle.mx_exponent(v) == want, hex(int(b))
    assert oracle.mx_exponent(0.0) == -127
    assert oracle.mx_exponent(6.0) == 0 and oracle.mx_exponent(4.0) == 0
    assert oracle.mx_exponent(3.999) == -1 and oracle.mx_exponent(8.0) == 1


def test_scale_layouts_cover_every_byte_once():
    """Linear: row-major over cols/32 scale columns.  Swizzled: the same
    128x4 tiling as the NVFP4 layout, taken over cols/32 scale columns, so
    each position equals the NVFP4 offset of a tensor with half the columns;
    rows pad to 128 and scale columns to 4, every padded position is hit
    exactly once."""
    for rows, cols in [(1, 32), (130, 96), (256, 1024), (300, 32 * 9)]:
        s = cols // 32
        assert oracle.mx_scales_bytes(rows, cols, oracle.SF_LINEAR) == rows * s
        for r in range(rows):
            for c in range(s):
                assert oracle.mx_sf_offset(r, c, cols, oracle.SF_LINEAR) == r * s + c
        rp, sp = (rows + 127) // 128 * 128, (s + 3) // 4 * 4
        assert oracle.mx_scales_bytes(rows, cols, oracle.SF_SWIZZLED) == rp * sp
        offs = [oracle.mx_sf_offset(r, c, cols, oracle.SF_SWIZZLED) for r in range(rp) for c in range(sp)]
        assert sorted(offs) == list(range(rp * sp))
        for r in range(0, rp, 7):
            for c in range(sp):
                assert (oracle.mx_sf_offset(r, c, cols, oracle.SF_SWIZZLED)
                        == oracle.sf_offset(r, c, rows, cols // 2, oracle.SF_SWIZZLED))


def test_dequantize_is_code_times_power_of_two():
    """Every stored value decodes to sign * grid[code] * 2^(byte - 127),
    rounded to BF16 (exact here: the products are short binary fractions),
    in both scale layouts."""
    x = _rand(130, 96, 10)
    for layout in (oracle.SF_LINEAR, oracle.SF_SWIZZLED):
        _, q = oracle.quantize_mx(x, layout)
        y = oracle.bf16_to_f32(q.dequantize()).astype(np.float64)
        nib = _nibbles(q)
        for r in range(0, 130, 3):
            for c in range(96):
                byte = int(q.scales[oracle.mx_sf_offset(r, c // 32, 96, layout)])
                v = GRID[nib[r, c] & 7] * (-1.0 if nib[r, c] & 8 else 1.0) * 2.0 ** (byte - 127)
                assert y[r, c] == v

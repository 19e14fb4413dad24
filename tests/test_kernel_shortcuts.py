"""The quantize kernels replace two IEEE divisions by cheaper exact
shortcuts; these CPU checks show the shortcuts give the division's result
bit for bit on the inputs the kernels use them for (the GPU parity tests
then check the kernels themselves against the oracle, which divides)."""
import ctypes as C

from tests.pins.build import build as build_pins


def _lib():
    L = C.CDLL(build_pins())
    L.shortcut_div6_table.restype = C.c_int64
    L.shortcut_div6_fma.restype = C.c_int64
    L.shortcut_div6_fma.argtypes = [C.c_uint32, C.c_uint32]
    L.shortcut_sr.restype = C.c_int64
    L.shortcut_sr.argtypes = [C.c_uint32, C.c_uint32, C.c_void_p, C.c_int, C.c_uint32]
    for f in (L.shortcut_rint_shift, L.shortcut_tf32_split):
        f.restype = C.c_int64
        f.argtypes = [C.c_uint32, C.c_uint32, C.c_uint32]
    return L


def test_bf16_amax_over_six_table_every_pattern():
    assert _lib().shortcut_div6_table() == 0


def test_fp32_amax_over_six_fma_correction():
    """Scaling a by 2^k scales every step of the shortcut by 2^k exactly
    while all values stay normal, so one full binade in the middle stands
    for all of them; the binades next to the underflow threshold
    (a >= 1.5 * 2^-124) and the top binade are checked in full too."""
    L = _lib()
    binade = lambda e: ((e + 127) << 23, (e + 128) << 23)
    assert L.shortcut_div6_fma(*binade(0)) == 0
    assert L.shortcut_div6_fma(0x01C00000, binade(-122)[1]) == 0   # 1.5 * 2^-124 .. 2^-121
    assert L.shortcut_div6_fma(*binade(127)) == 0


def test_stochastic_rounding_on_the_bit_pattern():
    """Every 31st binary32 magnitude below 8 with draws at the ends and in
    the middle of the range, every 211th with 64 random draws, and every
    pattern within 2^14 ulps of each grid value and segment boundary."""
    import struct

    import numpy as np
    L = _lib()
    draws = np.array([0, 1, 2, 63, 64, 0x7FFF, 0x8000, 0xFFFE, 0xFFFF], np.uint32)
    assert L.shortcut_sr(0, 0x41000000, draws.ctypes.data, len(draws), 31) == 0
    rnd = np.random.default_rng(5).integers(0, 1 << 16, 64).astype(np.uint32)
    assert L.shortcut_sr(0, 0x41000000, rnd.ctypes.data, len(rnd), 211) == 0
    for v in (0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0):
        b = struct.unpack("<I", struct.pack("<f", v))[0]
        assert L.shortcut_sr(b - (1 << 14), b + (1 << 14), draws.ctypes.data, len(draws), 1) == 0
    assert L.shortcut_sr(0, 1 << 15, draws.ctypes.data, len(draws), 1) == 0   # zero and subnormals


def _bits(x: float) -> int:
    import struct
    return struct.unpack("<I", struct.pack("<f", x))[0]


def test_exp_rint_by_shift():
    """The gated activation's exponential rounds y = RN(x * log2 e) to an
    integer by adding and subtracting 1.5 * 2^23 and reads the integer from
    the sum's bits: equal to rintf for every 5th binary32 x up to 87 (both
    signs), every pattern around the values where y is a half-integer, and
    the clamp ends."""
    L = _lib()
    assert L.shortcut_rint_shift(0, _bits(87.0) + 1, 5) == 0
    for k in range(-125, 126):
        b = _bits((k + 0.5) / 1.4426950408889634)
        assert L.shortcut_rint_shift(max(b - 4096, 0), b + 4096, 1) == 0, k


def test_attention_weight_split_into_three_tf32_parts():
    """p = p1 + p2 + p3 exactly with each part a TF32 value, for every
    binary32 p in [1, 2) and every 7th one from 2^-113 to 1: the three
    tensor-core products of a weight with a restored value sum to the exact
    product."""
    L = _lib()
    assert L.shortcut_tf32_split(_bits(1.0), _bits(2.0), 1) == 0
    assert L.shortcut_tf32_split(_bits(2.0 ** -113), _bits(1.0) + 1, 7) == 0


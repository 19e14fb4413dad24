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

"""ctypes front end of the NVFP4 CPU oracle (test infrastructure only).

All arrays are numpy; BF16 tensors travel as their uint16 bit patterns.
Torch CPU BF16 tensors are accepted wherever a BF16 array is expected.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from .build import LIB, build

__all__ = [
    "SF_SWIZZLED", "SF_LINEAR", "OK", "ERR_SHAPE", "ERR_NONFINITE", "ERR_RANGE",
    "lib", "bf16_bits", "bf16_to_f32", "f32_to_bf16", "e2m1_decode", "e2m1_rne",
    "e4m3_decode", "e4m3_rne", "scales_bytes", "sf_offset", "tensor_amax",
    "global_scale", "quantize", "quantize_with_global", "quantize_parallel", "dequantize",
    "gemm_ref", "gemm_ref_parallel", "tensor_amax_parallel", "host_threads",
    "dot_exact_i64", "Quantized", "rht16", "rht16_inverse", "quantize_rht", "quantize_2d",
    "philox4x32_10", "e2m1_sr", "sr_block_draws", "quantize_sr",
    "ue8m0_decode", "mx_scales_bytes", "mx_sf_offset", "mx_exponent", "quantize_mx",
    "dequantize_mx", "gemm_ref_mx", "QuantizedMX", "moe_combine", "dequantize_fp8",
    "exp_ref", "swiglu", "quantize_swiglu", "attention_decode",
]

SF_SWIZZLED, SF_LINEAR = 0, 1
OK, ERR_SHAPE, ERR_NONFINITE, ERR_RANGE = 0, 3, 4, 5

_lib = None
_p = C.c_void_p
_i64 = C.c_int64


def lib() -> C.CDLL:
    global _lib
    if _lib is None:
        build()
        L = C.CDLL(LIB)
        sig = {
            "nvo_bf16_to_f32": (C.c_float, [C.c_uint16]),
            "nvo_f32_to_bf16": (C.c_uint16, [C.c_float]),
            "nvo_e2m1_decode": (C.c_float, [C.c_uint8]),
            "nvo_e2m1_rne_satfinite": (C.c_uint8, [C.c_float]),
            "nvo_e4m3_decode": (C.c_float, [C.c_uint8]),
            "nvo_e4m3_rne_satfinite": (C.c_uint8, [C.c_float]),
            "nvo_scales_bytes": (_i64, [_i64, _i64, C.c_int]),
            "nvo_codes_bytes": (_i64, [_i64, _i64]),
            "nvo_sf_offset": (_i64, [_i64, _i64, _i64, _i64, C.c_int]),
            "nvo_tensor_amax": (C.c_int, [_p, _i64, _i64, _i64, C.POINTER(C.c_float)]),
            "nvo_global_scale": (C.c_int, [C.c_float, C.POINTER(C.c_float)]),
            "nvo_quantize_with_global": (None, [_p, _i64, _i64, _i64, C.c_float, _p, _p, C.c_int]),
            "nvo_quantize": (C.c_int, [_p, _i64, _i64, _i64, _p, _p, C.c_int, C.POINTER(C.c_float)]),
            "nvo_dequantize": (None, [_p, _p, C.c_int, C.c_float, _i64, _i64, _p, _i64]),
            "nvo_gemm_ref": (None, [_p, _p, C.c_int, C.c_float, _i64, _p, _p, C.c_int, _p,
                                    _i64, _i64, _p, _p, _i64, _p, _p]),
            "nvo_dot_exact_i64": (_i64, [_p, _p, C.c_int, _i64, _p, _p, C.c_int, _i64,
                                         _i64, _i64, _i64]),
            "nvo_rht16": (None, [_p, C.c_uint32, _p]),
            "nvo_rht16_inverse": (None, [_p, C.c_uint32, _p]),
            "nvo_quantize_rht": (C.c_int, [_p, _i64, _i64, _i64, C.c_uint32, _p, _p, C.c_int,
                                           C.c_int, C.POINTER(C.c_float)]),
            "nvo_quantize_2d": (C.c_int, [_p, _i64, _i64, _i64, _p, _p, C.c_int, C.c_int,
                                          C.POINTER(C.c_float)]),
            "nvo_philox4x32_10": (None, [_p, _p, _p]),
            "nvo_ue8m0_decode": (C.c_double, [C.c_uint8]),
            "nvo_moe_combine": (None, [_p, _i64, _p, _p, _i64, _i64, _i64, _p, _i64]),
            "nvo_exp_ref": (C.c_float, [C.c_float]),
            "nvo_attention_decode": (C.c_int, [_p, _i64, _i64, _p, _p, C.c_float, _p, _p, C.c_float,
                                               C.c_int, _i64, _i64, _i64, C.c_double, _i64, _i64,
                                               _p, _p, _p]),
            "nvo_swiglu": (C.c_float, [C.c_float, C.c_float]),
            "nvo_quantize_swiglu": (C.c_int, [_p, _i64, _i64, _i64, _p, _p, C.c_int,
                                              C.POINTER(C.c_float)]),
            "nvo_dequantize_fp8": (None, [_p, _p, C.c_int, C.c_float, _i64, _i64, _p, _i64,
                                          C.POINTER(C.c_float)]),
            "nvo_mx_scales_bytes": (_i64, [_i64, _i64, C.c_int]),
            "nvo_mx_sf_offset": (_i64, [_i64, _i64, _i64, C.c_int]),
            "nvo_mx_exponent": (C.c_int, [C.c_float]),
            "nvo_quantize_mx": (C.c_int, [_p, _i64, _i64, _i64, _p, _p, C.c_int]),
            "nvo_dequantize_mx": (None, [_p, _p, C.c_int, _i64, _i64, _p, _i64]),
            "nvo_gemm_ref_mx": (None, [_p, _p, C.c_int, _i64, _p, _p, C.c_int, _i64, _i64, _p, _p,
                                       _i64, _p, _p]),
            "nvo_e2m1_sr": (C.c_uint8, [C.c_float, C.c_uint32]),
            "nvo_sr_block_draws": (None, [C.c_uint64, _i64, _i64, _i64, _p]),
            "nvo_quantize_sr": (C.c_int, [_p, _i64, _i64, _i64, C.c_int, C.c_uint32, C.c_uint64, _p,
                                          _p, C.c_int, C.c_int, C.POINTER(C.c_float)]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def bf16_bits(x) -> np.ndarray:
    """uint16 bit patterns of a BF16 array (torch CPU tensor or numpy u16)."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch
    assert x.dtype == torch.bfloat16
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(v: float) -> int:
    return int(lib().nvo_f32_to_bf16(float(v)))


def e2m1_decode(code: int) -> float:
    return float(lib().nvo_e2m1_decode(code))


def e2m1_rne(y: float) -> int:
    return int(lib().nvo_e2m1_rne_satfinite(float(np.float32(y))))


def e4m3_decode(b: int) -> float:
    return float(lib().nvo_e4m3_decode(b))


def e4m3_rne(v: float) -> int:
    return int(lib().nvo_e4m3_rne_satfinite(float(np.float32(v))))


def scales_bytes(rows: int, cols: int, layout: int) -> int:
    return int(lib().nvo_scales_bytes(rows, cols, layout))


def sf_offset(r: int, c: int, rows: int, cols: int, layout: int) -> int:
    return int(lib().nvo_sf_offset(r, c, rows, cols, layout))


def tensor_amax(x) -> tuple[int, float]:
    b = bf16_bits(x)
    rows, cols = b.shape
    out = C.c_float()
    st = lib().nvo_tensor_amax(_ptr(b), rows, cols, cols, C.byref(out))
    return st, float(out.value)


def global_scale(amax: float) -> tuple[int, float]:
    out = C.c_float()
    st = lib().nvo_global_scale(float(np.float32(amax)), C.byref(out))
    return st, float(out.value)


class Quantized:
    """Oracle NVFP4 tensor: codes [rows, cols/2] u8, scales (flat u8), g."""

    def __init__(self, codes, scales, g, rows, cols, layout):
        self.codes, self.scales, self.g = codes, scales, np.float32(g)
        self.rows, self.cols, self.layout = rows, cols, layout

    def dequantize(self) -> np.ndarray:
        return dequantize(self.codes, self.scales, self.layout, self.g, self.rows, self.cols)


def quantize_with_global(x, g: float, layout: int = SF_SWIZZLED) -> Quantized:
    b = bf16_bits(x)
    rows, cols = b.shape
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros(scales_bytes(rows, cols, layout), np.uint8)
    lib().nvo_quantize_with_global(_ptr(b), rows, cols, cols, float(np.float32(g)),
                                   _ptr(codes), _ptr(scales), layout)
    return Quantized(codes, scales, g, rows, cols, layout)


def quantize(x, layout: int = SF_SWIZZLED) -> tuple[int, Quantized]:
    """Two-level quantize (amax -> g -> encode).  Returns (status, tensor)."""
    b = bf16_bits(x)
    rows, cols = b.shape
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros(scales_bytes(rows, cols, layout), np.uint8)
    g = C.c_float(0.0)
    st = lib().nvo_quantize(_ptr(b), rows, cols, cols, _ptr(codes), _ptr(scales), layout,
                            C.byref(g))
    return st, Quantized(codes, scales, g.value, rows, cols, layout)


def _row_ranges(rows: int, threads: int) -> list[tuple[int, int]]:
    """Disjoint row ranges starting at multiples of 128: a range of the 128x4
    scale layout then owns one contiguous run of scale bytes, as does a range
    of the row-major layout."""
    per = -(-rows // max(1, threads))
    step = max(128, -(-per // 128) * 128)
    return [(r, min(rows, r + step)) for r in range(0, rows, step)]


def host_threads() -> int:
    """Host cores this process may run on."""
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()


def tensor_amax_parallel(x, threads: int | None = None) -> tuple[int, float]:
    """`tensor_amax` over disjoint row ranges on host threads; the maximum of
    the ranges' exact maxima is the tensor's (a maximum does not depend on
    grouping)."""
    from concurrent.futures import ThreadPoolExecutor
    b = bf16_bits(x)
    rows, cols = b.shape
    ranges = _row_ranges(rows, threads or host_threads())
    L = lib()

    def amax_of(rr):
        out = C.c_float()
        st = L.nvo_tensor_amax(b.ctypes.data + 2 * rr[0] * cols, rr[1] - rr[0], cols, cols,
                               C.byref(out))
        return st, out.value

    amax = 0.0
    with ThreadPoolExecutor(max(1, len(ranges))) as ex:
        for st, a in ex.map(amax_of, ranges):
            if st != OK:
                return st, 0.0
            amax = max(amax, a)
    return OK, amax


def quantize_parallel(x, layout: int = SF_SWIZZLED, threads: int | None = None
                      ) -> tuple[int, Quantized]:
    """`quantize` with its row loops spread over host threads (the C calls
    release the GIL).  The steps are the same calls in the same order of
    definition: the tensor amax is the maximum of the ranges' exact maxima
    (a maximum does not depend on grouping), g follows from it once, and
    every range is encoded by `quantize_with_global` with that g, each
    writing only its own rows' codes and scale bytes.  Bit-identical to
    `quantize` by construction; a CPU test checks it."""
    from concurrent.futures import ThreadPoolExecutor
    b = bf16_bits(x)
    rows, cols = b.shape
    if threads is None:
        threads = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros(scales_bytes(rows, cols, layout), np.uint8)
    if cols % 16 != 0:
        return ERR_SHAPE, Quantized(codes, scales, 0.0, rows, cols, layout)
    ranges = _row_ranges(rows, threads)
    L = lib()

    def amax_of(rr):
        out = C.c_float()
        st = L.nvo_tensor_amax(b.ctypes.data + 2 * rr[0] * cols, rr[1] - rr[0], cols, cols,
                               C.byref(out))
        return st, out.value

    with ThreadPoolExecutor(max(1, len(ranges))) as ex:
        parts = list(ex.map(amax_of, ranges))
        amax = 0.0
        for st, a in parts:
            if st != OK:
                return st, Quantized(codes, scales, 0.0, rows, cols, layout)
            amax = max(amax, a)
        st, g = global_scale(amax)
        if st != OK:
            return st, Quantized(codes, scales, g, rows, cols, layout)

        def encode(rr):
            r0, r1 = rr
            sf0 = scales_bytes(r0, cols, layout)
            L.nvo_quantize_with_global(b.ctypes.data + 2 * r0 * cols, r1 - r0, cols, cols,
                                       float(np.float32(g)), codes.ctypes.data + r0 * (cols // 2),
                                       scales.ctypes.data + sf0, layout)

        list(ex.map(encode, ranges))
    return OK, Quantized(codes, scales, g, rows, cols, layout)


def dequantize(codes, scales, layout, g, rows, cols) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    y = np.zeros((rows, cols), np.uint16)
    lib().nvo_dequantize(_ptr(codes), _ptr(scales), layout, float(np.float32(g)), rows, cols,
                         _ptr(y), cols)
    return y


def gemm_ref(a: Quantized, w: Quantized, i_idx, j_idx, gw=None):
    """Sampled FP64 reference of D = Ahat * What^T at pairs (i_idx, j_idx).

    ``gw`` (per sample) overrides w.g, for per-expert weight scales.
    Returns (ref, abs_sum) float64 arrays."""
    assert a.cols == w.cols
    i_idx = np.ascontiguousarray(i_idx, np.int64)
    j_idx = np.ascontiguousarray(j_idx, np.int64)
    n = len(i_idx)
    if gw is None:
        gw = np.full(n, w.g, np.float32)
    gw = np.ascontiguousarray(gw, np.float32)
    ref = np.zeros(n, np.float64)
    ab = np.zeros(n, np.float64)
    lib().nvo_gemm_ref(_ptr(a.codes), _ptr(a.scales), a.layout, float(a.g), a.rows,
                       _ptr(w.codes), _ptr(w.scales), w.layout, _ptr(gw), w.rows, a.cols,
                       _ptr(i_idx), _ptr(j_idx), n, _ptr(ref), _ptr(ab))
    return ref, ab


def gemm_ref_parallel(a: Quantized, w: Quantized, i_idx, j_idx, threads: int | None = None):
    """`gemm_ref` with the sampled outputs split over host threads (each
    output is computed by the same C routine, independently)."""
    from concurrent.futures import ThreadPoolExecutor
    i_idx = np.ascontiguousarray(i_idx, np.int64)
    j_idx = np.ascontiguousarray(j_idx, np.int64)
    n = len(i_idx)
    t = max(1, min(threads or host_threads(), n))
    bounds = [(n * q) // t for q in range(t + 1)]
    with ThreadPoolExecutor(t) as ex:
        parts = list(ex.map(lambda q: gemm_ref(a, w, i_idx[bounds[q]:bounds[q + 1]],
                                               j_idx[bounds[q]:bounds[q + 1]]), range(t)))
    return (np.concatenate([p[0] for p in parts]) if parts else np.zeros(0),
            np.concatenate([p[1] for p in parts]) if parts else np.zeros(0))


def dot_exact_i64(a: Quantized, w: Quantized, i: int, j: int) -> int:
    return int(lib().nvo_dot_exact_i64(_ptr(a.codes), _ptr(a.scales), a.layout, a.rows,
                                       _ptr(w.codes), _ptr(w.scales), w.layout, w.rows,
                                       a.cols, i, j))


def rht16(x, sign_mask: int) -> np.ndarray:
    """Random Hadamard transform of one 16-value block (float32)."""
    x = np.ascontiguousarray(x, np.float32)
    y = np.zeros(16, np.float32)
    lib().nvo_rht16(_ptr(x), sign_mask, _ptr(y))
    return y


def rht16_inverse(y, sign_mask: int) -> np.ndarray:
    y = np.ascontiguousarray(y, np.float32)
    x = np.zeros(16, np.float32)
    lib().nvo_rht16_inverse(_ptr(y), sign_mask, _ptr(x))
    return x


def quantize_rht(x, sign_mask: int, layout: int = SF_SWIZZLED, g=None) -> tuple[int, Quantized]:
    """Quantize the random-Hadamard-transformed tensor (g given = supplied)."""
    b = bf16_bits(x)
    rows, cols = b.shape
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros(scales_bytes(rows, cols, layout), np.uint8)
    gv = C.c_float(0.0 if g is None else float(np.float32(g)))
    st = lib().nvo_quantize_rht(_ptr(b), rows, cols, cols, sign_mask, _ptr(codes), _ptr(scales),
                                layout, 0 if g is None else 1, C.byref(gv))
    return st, Quantized(codes, scales, gv.value, rows, cols, layout)


def quantize_2d(x, layout: int = SF_SWIZZLED, g=None) -> tuple[int, Quantized]:
    """Quantize with one scale per 16x16 block (g given = supplied)."""
    b = bf16_bits(x)
    rows, cols = b.shape
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros(scales_bytes(rows, cols, layout), np.uint8)
    gv = C.c_float(0.0 if g is None else float(np.float32(g)))
    st = lib().nvo_quantize_2d(_ptr(b), rows, cols, cols, _ptr(codes), _ptr(scales), layout,
                               0 if g is None else 1, C.byref(gv))
    return st, Quantized(codes, scales, gv.value, rows, cols, layout)


def philox4x32_10(ctr, key) -> list[int]:
    c = np.ascontiguousarray(ctr, np.uint32)
    k = np.ascontiguousarray(key, np.uint32)
    out = np.zeros(4, np.uint32)
    lib().nvo_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return [int(v) for v in out]


def e2m1_sr(y: float, u16: int) -> int:
    return int(lib().nvo_e2m1_sr(float(np.float32(y)), u16))


def sr_block_draws(seed: int, r: int, b: int, cols: int) -> np.ndarray:
    u = np.zeros(16, np.uint32)
    lib().nvo_sr_block_draws(seed, r, b, cols, _ptr(u))
    return u


def quantize_sr(x, seed: int, layout: int = SF_SWIZZLED, sign_mask=None, g=None):
    """Quantize with stochastically rounded codes (optionally after the
    Hadamard transform).  Returns (status, tensor)."""
    b = bf16_bits(x)
    rows, cols = b.shape
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros(scales_bytes(rows, cols, layout), np.uint8)
    gv = C.c_float(0.0 if g is None else float(np.float32(g)))
    st = lib().nvo_quantize_sr(_ptr(b), rows, cols, cols, 0 if sign_mask is None else 1,
                               sign_mask or 0, seed, _ptr(codes), _ptr(scales), layout,
                               0 if g is None else 1, C.byref(gv))
    return st, Quantized(codes, scales, gv.value, rows, cols, layout)


def ue8m0_decode(b: int) -> float:
    return float(lib().nvo_ue8m0_decode(b))


def mx_scales_bytes(rows: int, cols: int, layout: int) -> int:
    return int(lib().nvo_mx_scales_bytes(rows, cols, layout))


def mx_sf_offset(r: int, c: int, cols: int, layout: int) -> int:
    return int(lib().nvo_mx_sf_offset(r, c, cols, layout))


def mx_exponent(amax: float) -> int:
    return int(lib().nvo_mx_exponent(float(np.float32(amax))))


class QuantizedMX:
    """Oracle MXFP4 tensor: codes [rows, cols/2] u8, UE8M0 scales (flat u8)."""

    def __init__(self, codes, scales, rows, cols, layout):
        self.codes, self.scales = codes, scales
        self.rows, self.cols, self.layout = rows, cols, layout

    def dequantize(self) -> np.ndarray:
        return dequantize_mx(self.codes, self.scales, self.layout, self.rows, self.cols)


def quantize_mx(x, layout: int = SF_SWIZZLED) -> tuple[int, QuantizedMX]:
    b = bf16_bits(x)
    rows, cols = b.shape
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros(mx_scales_bytes(rows, cols, layout), np.uint8)
    st = lib().nvo_quantize_mx(_ptr(b), rows, cols, cols, _ptr(codes), _ptr(scales), layout)
    return st, QuantizedMX(codes, scales, rows, cols, layout)


def dequantize_mx(codes, scales, layout, rows, cols) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    y = np.zeros((rows, cols), np.uint16)
    lib().nvo_dequantize_mx(_ptr(codes), _ptr(scales), layout, rows, cols, _ptr(y), cols)
    return y


def gemm_ref_mx(a: QuantizedMX, w: QuantizedMX, i_idx, j_idx):
    assert a.cols == w.cols
    i_idx = np.ascontiguousarray(i_idx, np.int64)
    j_idx = np.ascontiguousarray(j_idx, np.int64)
    n = len(i_idx)
    ref = np.zeros(n, np.float64)
    ab = np.zeros(n, np.float64)
    lib().nvo_gemm_ref_mx(_ptr(a.codes), _ptr(a.scales), a.layout, a.rows, _ptr(w.codes),
                          _ptr(w.scales), w.layout, w.rows, a.cols, _ptr(i_idx), _ptr(j_idx), n,
                          _ptr(ref), _ptr(ab))
    return ref, ab


def moe_combine(out, slots, weights) -> np.ndarray:
    """y[t] = bf16(sum_k w[t,k] * out[slots[t,k]]) (FMA chain in k order)."""
    o = bf16_bits(out)
    sl = np.ascontiguousarray(np.asarray(slots), np.int32)
    w = np.ascontiguousarray(np.asarray(weights), np.float32)
    tokens, topk = sl.shape
    hidden = o.shape[1]
    y = np.zeros((tokens, hidden), np.uint16)
    lib().nvo_moe_combine(_ptr(o), hidden, _ptr(sl), _ptr(w), tokens, topk, hidden, _ptr(y), hidden)
    return y


def dequantize_fp8(q: Quantized) -> tuple[np.ndarray, float]:
    """NVFP4 -> E4M3 bytes and the per-tensor dequant factor RN(8 / g)."""
    y = np.zeros((q.rows, q.cols), np.uint8)
    sc = C.c_float()
    lib().nvo_dequantize_fp8(_ptr(np.ascontiguousarray(q.codes)), _ptr(np.ascontiguousarray(q.scales)),
                             q.layout, float(q.g), q.rows, q.cols, _ptr(y), q.cols, C.byref(sc))
    return y, float(sc.value)


def exp_ref(x: float) -> float:
    return float(lib().nvo_exp_ref(float(np.float32(x))))


def swiglu(g: float, u: float) -> float:
    return float(lib().nvo_swiglu(float(np.float32(g)), float(np.float32(u))))


def quantize_swiglu(gu, layout: int = SF_SWIZZLED) -> tuple[int, Quantized]:
    """NVFP4 of h = silu(gate) * up for gu = [gate | up] (BF16, rows x 2I)."""
    b = bf16_bits(gu)
    rows, two_i = b.shape
    inter = two_i // 2
    codes = np.zeros((rows, inter // 2), np.uint8)
    scales = np.zeros(scales_bytes(rows, inter, layout), np.uint8)
    g = C.c_float()
    st = lib().nvo_quantize_swiglu(_ptr(b), rows, inter, two_i, _ptr(codes), _ptr(scales), layout,
                                   C.byref(g))
    return st, Quantized(codes, scales, g.value, rows, inter, layout)


if os.environ.get("NVFP4_ORACLE_EAGER_BUILD"):
    lib()


def attention_decode(q, k: Quantized, v: Quantized, heads_kv: int, scale: float,
                     heads=None):
    """One decode step of grouped-query attention over NVFP4 K and V
    [tokens x heads_kv * head_dim] in FP64 on the exact restored values.
    q: BF16 [heads_q x head_dim].  `heads` = (begin, end) limits the query
    heads computed (default all).  Returns (status, o, abs_o, score_abs):
    o and abs_o [end - begin x head_dim] float64, score_abs [end - begin]."""
    qb = bf16_bits(q)
    heads_q, head_dim = qb.shape
    assert k.layout == v.layout and k.rows == v.rows and k.cols == v.cols
    h0, h1 = (0, heads_q) if heads is None else heads
    n = max(h1 - h0, 0)
    o = np.zeros((n, head_dim), np.float64)
    ao = np.zeros((n, head_dim), np.float64)
    sa = np.zeros(max(n, 1), np.float64)
    kc, ks = np.ascontiguousarray(k.codes), np.ascontiguousarray(k.scales)
    vc, vs = np.ascontiguousarray(v.codes), np.ascontiguousarray(v.scales)
    st = lib().nvo_attention_decode(_ptr(qb), head_dim, heads_q, _ptr(kc), _ptr(ks), float(np.float32(k.g)),
                                    _ptr(vc), _ptr(vs), float(np.float32(v.g)), k.layout, k.rows,
                                    heads_kv, head_dim, float(scale), h0, h1, _ptr(o), _ptr(ao), _ptr(sa))
    return st, o, ao, sa[:n]

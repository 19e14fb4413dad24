"""Thin ctypes binding of libnvfp4.so (the C ABI in include/nvfp4.h).

Argument marshalling only: every step of the NVFP4 path runs in the CUDA
kernels of libnvfp4.so.  PyTorch supplies device memory and streams.  There
is no CPU fallback -- loading fails loudly if the library is missing.

Function names follow the C ABI (``nvfp4_quantize`` ...), taking torch
tensors instead of raw pointers.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
# The in-tree build; NVFP4_LIBRARY may name another build of the same C ABI
# (for example one compiled with a different pipeline geometry).
LIB_PATH = os.environ.get("NVFP4_LIBRARY") or os.path.join(HERE, "libnvfp4.so")

SF_SWIZZLED = 0
SF_LINEAR = 1

OP_QUANTIZE, OP_DEQUANTIZE, OP_GEMM, OP_GROUPED_GEMM, OP_QUANTIZE_GATHER, OP_ATTENTION = range(6)

STATUS_NAMES = {
    0: "NVFP4_OK", 1: "NVFP4_ERR_INVALID_ARG", 2: "NVFP4_ERR_ALIGNMENT", 3: "NVFP4_ERR_SHAPE",
    4: "NVFP4_ERR_NONFINITE", 5: "NVFP4_ERR_RANGE", 6: "NVFP4_ERR_WORKSPACE",
    7: "NVFP4_ERR_TIMEOUT", 8: "NVFP4_ERR_UNSUPPORTED_DEVICE", 9: "NVFP4_ERR_CUDA",
}

# Symbols the header declares; the library must export every one.
EXPORTED = (
    "nvfp4_codes_bytes", "nvfp4_scales_bytes", "nvfp4_workspace_bytes", "nvfp4_quantize",
    "nvfp4_global_scale", "nvfp4_quantize_gather", "nvfp4_dequantize", "nvfp4_gemm",
    "nvfp4_grouped_gemm", "nvfp4_grouped_gemm_out_scale", "nvfp4_check_status",
    "nvfp4_status_string", "nvfp4_version",
    "nvfp4_launch_count", "nvfp4_set_wait_limit_cycles", "nvfp4_set_gemm_pairs",
    "nvfp4_quantize_noalloc", "nvfp4_quantize_rht", "nvfp4_quantize_t", "nvfp4_quantize_2d",
    "nvfp4_quantize_sr", "nvfp4_mx_scales_bytes", "nvfp4_quantize_mx", "nvfp4_dequantize_mx",
    "nvfp4_gemm_mx", "nvfp4_moe_combine", "nvfp4_dequantize_fp8", "nvfp4_quantize_swiglu",
    "nvfp4_attention_decode", "nvfp4_gather_rows",
)


class NVFP4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


class CTensor(C.Structure):
    """Mirror of ``nvfp4_tensor``."""
    _fields_ = [("codes", C.c_void_p), ("scales", C.c_void_p), ("global_", C.c_void_p),
                ("rows", C.c_int64), ("cols", C.c_int64), ("sf_layout", C.c_int32)]


_lib = None


def lib() -> C.CDLL:
    """Load libnvfp4.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libnvfp4.so not built at {LIB_PATH}; run "
                              "python -m nvfp4_block_scaled_22_b200.build")
        L = C.CDLL(LIB_PATH)
        i64, i32, vp, sz = C.c_int64, C.c_int32, C.c_void_p, C.c_size_t
        T = C.POINTER(CTensor)
        sig = {
            "nvfp4_codes_bytes": (sz, [i64, i64]),
            "nvfp4_scales_bytes": (sz, [i64, i64, i32]),
            "nvfp4_workspace_bytes": (sz, [i32, i64, i64, i64, i32]),
            "nvfp4_quantize": (C.c_int, [vp, i64, T, i32, vp, sz, vp]),
            "nvfp4_global_scale": (C.c_int, [vp, i64, i64, i64, vp, vp, sz, vp]),
            "nvfp4_quantize_gather": (C.c_int, [vp, i64, i64, vp, T, i32, vp, sz, vp]),
            "nvfp4_dequantize": (C.c_int, [T, vp, i64, vp]),
            "nvfp4_gemm": (C.c_int, [T, T, vp, i64, vp, sz, vp]),
            "nvfp4_grouped_gemm": (C.c_int, [i32, vp, vp, T, T, vp, i64, vp, i64, vp, sz, vp]),
            "nvfp4_grouped_gemm_out_scale": (C.c_int, [i32, vp, vp, T, T, vp, i64, vp, i64, vp, vp,
                                                       sz, vp]),
            "nvfp4_check_status": (C.c_int, [vp, vp]),
            "nvfp4_status_string": (C.c_char_p, [C.c_int]),
            "nvfp4_version": (i32, []),
            "nvfp4_launch_count": (i64, []),
            "nvfp4_gather_rows": (C.c_int, [T, vp, T, vp, sz, vp]),
            "nvfp4_set_wait_limit_cycles": (C.c_longlong, [C.c_longlong]),
            "nvfp4_set_gemm_pairs": (i32, [i32]),
            "nvfp4_quantize_noalloc": (C.c_int, [vp, i64, T, i32, vp]),
            "nvfp4_quantize_rht": (C.c_int, [vp, i64, C.c_uint32, T, i32, vp, sz, vp]),
            "nvfp4_quantize_t": (C.c_int, [vp, i64, i32, C.c_uint32, T, i32, vp, sz, vp]),
            "nvfp4_quantize_2d": (C.c_int, [vp, i64, T, T, i32, vp, sz, vp]),
            "nvfp4_quantize_sr": (C.c_int, [vp, i64, i32, i32, C.c_uint32, C.c_uint64, T, i32, vp,
                                            sz, vp]),
            "nvfp4_mx_scales_bytes": (sz, [i64, i64, i32]),
            "nvfp4_quantize_mx": (C.c_int, [vp, i64, T, vp, sz, vp]),
            "nvfp4_dequantize_mx": (C.c_int, [T, vp, i64, vp]),
            "nvfp4_gemm_mx": (C.c_int, [T, T, vp, i64, vp, sz, vp]),
            "nvfp4_moe_combine": (C.c_int, [vp, i64, i64, vp, vp, i64, i32, i64, vp, i64, vp]),
            "nvfp4_dequantize_fp8": (C.c_int, [T, vp, i64, vp, vp]),
            "nvfp4_quantize_swiglu": (C.c_int, [vp, i64, T, vp, sz, vp]),
            "nvfp4_attention_decode": (C.c_int, [vp, i64, i32, T, T, i32, C.c_float, vp, i64, vp, sz,
                                                 vp]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(st: int, where: str):
    if st != 0:
        raise NVFP4Error(st, where)


def _ptr(t) -> int:
    return 0 if t is None else t.data_ptr()


# ------------------------------------------------------------------ sizes
def nvfp4_codes_bytes(rows: int, cols: int) -> int:
    return int(lib().nvfp4_codes_bytes(rows, cols))


def nvfp4_scales_bytes(rows: int, cols: int, layout: int = SF_SWIZZLED) -> int:
    return int(lib().nvfp4_scales_bytes(rows, cols, layout))


def nvfp4_workspace_bytes(op: int, a=0, b=0, c=0, groups=0) -> int:
    return int(lib().nvfp4_workspace_bytes(op, a, b, c, groups))


# ---------------------------------------------------------- tensor types
class NVFP4Tensor:
    """Device NVFP4 tensor: packed codes, block scales and the tensor scale.

    ``codes`` uint8 [rows, cols/2], ``scales`` uint8 [scales_bytes],
    ``global_scale`` float32 [1]; all on one CUDA device."""

    def __init__(self, codes, scales, global_scale, rows, cols, layout):
        self.codes, self.scales, self.global_scale = codes, scales, global_scale
        self.rows, self.cols, self.layout = rows, cols, layout

    @classmethod
    def empty(cls, rows: int, cols: int, layout: int = SF_SWIZZLED, device="cuda",
              global_scale=None):
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=device)
        scales = torch.empty(nvfp4_scales_bytes(rows, cols, layout), dtype=torch.uint8,
                             device=device)
        if global_scale is None:
            global_scale = torch.zeros(1, dtype=torch.float32, device=device)
        return cls(codes, scales, global_scale, rows, cols, layout)

    def c_struct(self) -> CTensor:
        return CTensor(_ptr(self.codes), _ptr(self.scales), _ptr(self.global_scale),
                       self.rows, self.cols, self.layout)

    def nbytes(self) -> int:
        return self.codes.numel() + self.scales.numel()


class MXFP4Tensor(NVFP4Tensor):
    """Device MXFP4 tensor: packed codes and UE8M0 scales (one per 32
    values); no tensor scale."""

    @classmethod
    def empty(cls, rows: int, cols: int, layout: int = SF_SWIZZLED, device="cuda"):
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=device)
        scales = torch.empty(lib().nvfp4_mx_scales_bytes(rows, cols, layout), dtype=torch.uint8,
                             device=device)
        return cls(codes, scales, None, rows, cols, layout)


class Workspace:
    """Zero-initialised device workspace (status word + scratch)."""

    def __init__(self, device="cuda", nbytes: int | None = None):
        if nbytes is None:
            # room for the split-K slices of small-M GEMMs (a smaller
            # workspace only turns the split off)
            nbytes = max(max(nvfp4_workspace_bytes(op) for op in range(5)), 32 << 20)
        self.buf = torch.zeros(nbytes, dtype=torch.uint8, device=device)

    @property
    def ptr(self) -> int:
        return self.buf.data_ptr()

    @property
    def nbytes(self) -> int:
        return self.buf.numel()


_default_ws: dict[int, Workspace] = {}


def default_workspace(device=None) -> Workspace:
    dev = torch.device(device or "cuda")
    idx = dev.index if dev.index is not None else torch.cuda.current_device()
    if idx not in _default_ws:
        _default_ws[idx] = Workspace(torch.device("cuda", idx))
    return _default_ws[idx]


# ------------------------------------------------------------ operations
def nvfp4_quantize(x: torch.Tensor, out: NVFP4Tensor | None = None, layout: int = SF_SWIZZLED,
                   global_supplied: bool = False, workspace: Workspace | None = None,
                   stream=None) -> NVFP4Tensor:
    """Two-level NVFP4 quantization of a 2-D BF16 CUDA tensor (row pitch
    x.stride(0)).  With ``global_supplied`` the tensor scale already in
    ``out.global_scale`` is used."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, cols = x.shape
    if out is None:
        out = NVFP4Tensor.empty(rows, cols, layout, x.device)
    ws = workspace or default_workspace(x.device)
    t = out.c_struct()
    _check(lib().nvfp4_quantize(x.data_ptr(), x.stride(0), C.byref(t), int(global_supplied),
                                ws.ptr, ws.nbytes, _stream(stream)), "nvfp4_quantize")
    return out


def nvfp4_quantize_rht(x: torch.Tensor, sign_mask: int, out: NVFP4Tensor | None = None,
                       layout: int = SF_SWIZZLED, global_supplied: bool = False,
                       workspace: Workspace | None = None, stream=None) -> NVFP4Tensor:
    """Quantize after the 16x16 random Hadamard transform of every block
    (``sign_mask`` bit j negates value j of each block before the transform)."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, cols = x.shape
    if out is None:
        out = NVFP4Tensor.empty(rows, cols, layout, x.device)
    ws = workspace or default_workspace(x.device)
    t = out.c_struct()
    _check(lib().nvfp4_quantize_rht(x.data_ptr(), x.stride(0), sign_mask, C.byref(t),
                                    int(global_supplied), ws.ptr, ws.nbytes, _stream(stream)),
           "nvfp4_quantize_rht")
    return out


def nvfp4_quantize_t(x: torch.Tensor, out: NVFP4Tensor | None = None, layout: int = SF_SWIZZLED,
                     sign_mask: int | None = None, global_supplied: bool = False,
                     workspace: Workspace | None = None, stream=None) -> NVFP4Tensor:
    """NVFP4 of x^T from a row-major BF16 x (x.shape = (R, C) gives a C x R
    tensor).  With ``sign_mask`` the blocks are Hadamard-transformed first."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows_x, cols_x = x.shape
    if out is None:
        out = NVFP4Tensor.empty(cols_x, rows_x, layout, x.device)
    ws = workspace or default_workspace(x.device)
    t = out.c_struct()
    rht = 0 if sign_mask is None else 1
    _check(lib().nvfp4_quantize_t(x.data_ptr(), x.stride(0), rht, sign_mask or 0, C.byref(t),
                                  int(global_supplied), ws.ptr, ws.nbytes, _stream(stream)),
           "nvfp4_quantize_t")
    return out


def nvfp4_quantize_2d(w: torch.Tensor, out: NVFP4Tensor | None = None,
                      out_t: NVFP4Tensor | None = None, transposed: bool = False,
                      layout: int = SF_SWIZZLED, global_supplied: bool = False,
                      workspace: Workspace | None = None, stream=None):
    """16x16-block quantization of a BF16 weight; with ``transposed`` (or an
    ``out_t``) also returns W^T's NVFP4 tensor holding the same values."""
    assert w.dtype == torch.bfloat16 and w.dim() == 2 and w.stride(1) == 1
    rows, cols = w.shape
    if out is None:
        out = NVFP4Tensor.empty(rows, cols, layout, w.device)
    if out_t is None and transposed:
        out_t = NVFP4Tensor.empty(cols, rows, layout, w.device)
    ws = workspace or default_workspace(w.device)
    t = out.c_struct()
    tt = out_t.c_struct() if out_t is not None else None
    _check(lib().nvfp4_quantize_2d(w.data_ptr(), w.stride(0), C.byref(t),
                                   C.byref(tt) if tt is not None else None, int(global_supplied),
                                   ws.ptr, ws.nbytes, _stream(stream)), "nvfp4_quantize_2d")
    return (out, out_t) if out_t is not None else out


def nvfp4_quantize_sr(x: torch.Tensor, seed: int, out: NVFP4Tensor | None = None,
                      transposed: bool = False, sign_mask: int | None = None,
                      layout: int = SF_SWIZZLED, global_supplied: bool = False,
                      workspace: Workspace | None = None, stream=None) -> NVFP4Tensor:
    """Quantize with stochastically rounded codes (Philox draws keyed by
    ``seed``); ``transposed`` gives NVFP4 of x^T, ``sign_mask`` applies the
    Hadamard transform first."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, cols = x.shape
    if out is None:
        out = (NVFP4Tensor.empty(cols, rows, layout, x.device) if transposed
               else NVFP4Tensor.empty(rows, cols, layout, x.device))
    ws = workspace or default_workspace(x.device)
    t = out.c_struct()
    _check(lib().nvfp4_quantize_sr(x.data_ptr(), x.stride(0), int(transposed),
                                   0 if sign_mask is None else 1, sign_mask or 0, seed, C.byref(t),
                                   int(global_supplied), ws.ptr, ws.nbytes, _stream(stream)),
           "nvfp4_quantize_sr")
    return out


def nvfp4_quantize_mx(x: torch.Tensor, out: MXFP4Tensor | None = None, layout: int = SF_SWIZZLED,
                      workspace: Workspace | None = None, stream=None) -> MXFP4Tensor:
    """MXFP4 quantization (block 32, UE8M0 scales) of a 2-D BF16 tensor."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, cols = x.shape
    if out is None:
        out = MXFP4Tensor.empty(rows, cols, layout, x.device)
    ws = workspace or default_workspace(x.device)
    t = out.c_struct()
    _check(lib().nvfp4_quantize_mx(x.data_ptr(), x.stride(0), C.byref(t), ws.ptr, ws.nbytes,
                                   _stream(stream)), "nvfp4_quantize_mx")
    return out


def nvfp4_dequantize_mx(t: MXFP4Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty((t.rows, t.cols), dtype=torch.bfloat16, device=t.codes.device)
    ct = t.c_struct()
    _check(lib().nvfp4_dequantize_mx(C.byref(ct), out.data_ptr(), out.stride(0), _stream(stream)),
           "nvfp4_dequantize_mx")
    return out


def nvfp4_gemm_mx(a: MXFP4Tensor, w: MXFP4Tensor, out: torch.Tensor | None = None,
                  workspace: Workspace | None = None, stream=None) -> torch.Tensor:
    """D = A_hat * W_hat^T for MXFP4 operands (BF16 out)."""
    if out is None:
        out = torch.empty((a.rows, w.rows), dtype=torch.bfloat16, device=a.codes.device)
    ws = workspace or default_workspace(a.codes.device)
    ta, tw = a.c_struct(), w.c_struct()
    _check(lib().nvfp4_gemm_mx(C.byref(ta), C.byref(tw), out.data_ptr(), out.stride(0), ws.ptr,
                               ws.nbytes, _stream(stream)), "nvfp4_gemm_mx")
    return out


def nvfp4_moe_combine(expert_out: torch.Tensor, slots: torch.Tensor, weights: torch.Tensor,
                      out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y[t] = bf16(sum_k weights[t,k] * expert_out[slots[t,k]])."""
    assert expert_out.dtype == torch.bfloat16 and expert_out.stride(1) == 1
    assert slots.dtype == torch.int32 and weights.dtype == torch.float32
    tokens, topk = slots.shape
    hidden = expert_out.shape[1]
    if out is None:
        out = torch.empty((tokens, hidden), dtype=torch.bfloat16, device=expert_out.device)
    _check(lib().nvfp4_moe_combine(expert_out.data_ptr(), expert_out.stride(0), expert_out.shape[0],
                                   slots.contiguous().data_ptr(), weights.contiguous().data_ptr(),
                                   tokens, topk, hidden, out.data_ptr(), out.stride(0),
                                   _stream(stream)), "nvfp4_moe_combine")
    return out


def nvfp4_dequantize_fp8(t: NVFP4Tensor, out: torch.Tensor | None = None, scale: torch.Tensor | None = None,
                         stream=None):
    """NVFP4 -> E4M3 bytes (uint8) and the per-tensor factor RN(8/g)."""
    if out is None:
        out = torch.empty((t.rows, t.cols), dtype=torch.uint8, device=t.codes.device)
    if scale is None:
        scale = torch.zeros(1, dtype=torch.float32, device=t.codes.device)
    ct = t.c_struct()
    _check(lib().nvfp4_dequantize_fp8(C.byref(ct), out.data_ptr(), out.stride(0), scale.data_ptr(),
                                      _stream(stream)), "nvfp4_dequantize_fp8")
    return out, scale


def nvfp4_attention_decode(q: torch.Tensor, k: NVFP4Tensor, v: NVFP4Tensor, heads_kv: int,
                           scale: float | None = None, out: torch.Tensor | None = None,
                           workspace: Workspace | None = None, stream=None) -> torch.Tensor:
    """One decode step of grouped-query attention read straight from an
    NVFP4 KV cache: q BF16 [heads_q x 128]; k, v NVFP4 [tokens x heads_kv *
    128] in the linear scale layout.  Returns BF16 [heads_q x 128].  The
    softmax scale defaults to 1 / sqrt(128)."""
    assert q.dtype == torch.bfloat16 and q.dim() == 2 and q.stride(1) == 1
    heads_q = q.shape[0]
    if scale is None:
        scale = 128 ** -0.5
    if out is None:
        out = torch.empty((heads_q, 128), dtype=torch.bfloat16, device=q.device)
    need = nvfp4_workspace_bytes(OP_ATTENTION, k.rows, heads_q, heads_kv)
    ws = workspace or default_workspace(q.device)
    if ws.nbytes < need:
        ws = Workspace(q.device, need)
    tk, tv = k.c_struct(), v.c_struct()
    _check(lib().nvfp4_attention_decode(q.data_ptr(), q.stride(0), heads_q, C.byref(tk), C.byref(tv),
                                        heads_kv, float(scale), out.data_ptr(), out.stride(0), ws.ptr,
                                        ws.nbytes, _stream(stream)), "nvfp4_attention_decode")
    return out


def nvfp4_quantize_swiglu(gate_up: torch.Tensor, out: NVFP4Tensor | None = None,
                          layout: int = SF_SWIZZLED, workspace: Workspace | None = None,
                          stream=None) -> NVFP4Tensor:
    """NVFP4 of silu(gate) * up for gate_up = [gate | up] (BF16, rows x 2I)."""
    assert gate_up.dtype == torch.bfloat16 and gate_up.dim() == 2 and gate_up.stride(1) == 1
    rows, two_i = gate_up.shape
    if out is None:
        out = NVFP4Tensor.empty(rows, two_i // 2, layout, gate_up.device)
    ws = workspace or default_workspace(gate_up.device)
    t = out.c_struct()
    _check(lib().nvfp4_quantize_swiglu(gate_up.data_ptr(), gate_up.stride(0), C.byref(t), ws.ptr,
                                       ws.nbytes, _stream(stream)), "nvfp4_quantize_swiglu")
    return out


def nvfp4_gather_rows(src: NVFP4Tensor, gather: torch.Tensor, out: NVFP4Tensor | None = None,
                      layout: int = SF_SWIZZLED, workspace: Workspace | None = None,
                      stream=None) -> NVFP4Tensor:
    """Out row r = source row gather[r] (codes and scales), -1 = zero row;
    the tensor scale is copied.  gather: int32 CUDA tensor."""
    assert gather.dtype == torch.int32 and gather.is_cuda
    if out is None:
        out = NVFP4Tensor.empty(gather.numel(), src.cols, layout, src.codes.device)
    ws = workspace or default_workspace(src.codes.device)
    cs, co = src.c_struct(), out.c_struct()
    _check(lib().nvfp4_gather_rows(C.byref(cs), gather.data_ptr(), C.byref(co), ws.ptr, ws.nbytes,
                                   _stream(stream)), "nvfp4_gather_rows")
    return out


def nvfp4_global_scale(x: torch.Tensor, out: torch.Tensor | None = None,
                       workspace: Workspace | None = None, stream=None) -> torch.Tensor:
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    if out is None:
        out = torch.zeros(1, dtype=torch.float32, device=x.device)
    ws = workspace or default_workspace(x.device)
    _check(lib().nvfp4_global_scale(x.data_ptr(), x.stride(0), x.shape[0], x.shape[1],
                                    out.data_ptr(), ws.ptr, ws.nbytes, _stream(stream)),
           "nvfp4_global_scale")
    return out


def nvfp4_quantize_gather(x: torch.Tensor, gather: torch.Tensor, out: NVFP4Tensor | None = None,
                          layout: int = SF_SWIZZLED, global_supplied: bool = False,
                          workspace: Workspace | None = None, stream=None) -> NVFP4Tensor:
    """Quantize rows x[gather[r]] (gather int32 CUDA, -1 = zero row)."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    assert gather.dtype == torch.int32 and gather.is_contiguous()
    rows, cols = gather.numel(), x.shape[1]
    if out is None:
        out = NVFP4Tensor.empty(rows, cols, layout, x.device)
    ws = workspace or default_workspace(x.device)
    t = out.c_struct()
    _check(lib().nvfp4_quantize_gather(x.data_ptr(), x.stride(0), x.shape[0], gather.data_ptr(),
                                       C.byref(t), int(global_supplied), ws.ptr, ws.nbytes,
                                       _stream(stream)), "nvfp4_quantize_gather")
    return out


def nvfp4_dequantize(t: NVFP4Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty((t.rows, t.cols), dtype=torch.bfloat16, device=t.codes.device)
    ct = t.c_struct()
    _check(lib().nvfp4_dequantize(C.byref(ct), out.data_ptr(), out.stride(0), _stream(stream)),
           "nvfp4_dequantize")
    return out


def nvfp4_gemm(a: NVFP4Tensor, w: NVFP4Tensor, out: torch.Tensor | None = None,
               workspace: Workspace | None = None, stream=None) -> torch.Tensor:
    """D = A * W^T on the FP4 tensor cores, BF16 [a.rows, w.rows]."""
    if out is None:
        out = torch.empty((a.rows, w.rows), dtype=torch.bfloat16, device=a.codes.device)
    ws = workspace or default_workspace(a.codes.device)
    ca, cw = a.c_struct(), w.c_struct()
    _check(lib().nvfp4_gemm(C.byref(ca), C.byref(cw), out.data_ptr(), out.stride(0), ws.ptr,
                            ws.nbytes, _stream(stream)), "nvfp4_gemm")
    return out


def nvfp4_grouped_gemm(slot_offsets: torch.Tensor, group_rows: torch.Tensor, a: NVFP4Tensor,
                       w: NVFP4Tensor, w_globals: torch.Tensor, n: int,
                       out: torch.Tensor | None = None, workspace: Workspace | None = None,
                       stream=None) -> torch.Tensor:
    """Grouped D_g = A_g * W_g^T over expert slots (see nvfp4_grouped_gemm in
    the header).  slot_offsets/group_rows int32 CUDA, w_globals float32 CUDA."""
    groups = group_rows.numel()
    if out is None:
        out = torch.empty((a.rows, n), dtype=torch.bfloat16, device=a.codes.device)
    ws = workspace or default_workspace(a.codes.device)
    ca, cw = a.c_struct(), w.c_struct()
    _check(lib().nvfp4_grouped_gemm(groups, slot_offsets.data_ptr(), group_rows.data_ptr(),
                                    C.byref(ca), C.byref(cw), w_globals.data_ptr(), n,
                                    out.data_ptr(), out.stride(0), ws.ptr, ws.nbytes,
                                    _stream(stream)), "nvfp4_grouped_gemm")
    return out


def nvfp4_grouped_gemm_out_scale(slot_offsets: torch.Tensor, group_rows: torch.Tensor,
                                 a: NVFP4Tensor, w: NVFP4Tensor, w_globals: torch.Tensor, n: int,
                                 out: torch.Tensor | None = None,
                                 out_global: torch.Tensor | None = None,
                                 workspace: Workspace | None = None, stream=None):
    """nvfp4_grouped_gemm that also writes the NVFP4 tensor scale of its BF16
    output over the real rows into out_global (float32 CUDA, one element).
    Returns (out, out_global)."""
    groups = group_rows.numel()
    if out is None:
        out = torch.empty((a.rows, n), dtype=torch.bfloat16, device=a.codes.device)
    if out_global is None:
        out_global = torch.empty(1, dtype=torch.float32, device=a.codes.device)
    ws = workspace or default_workspace(a.codes.device)
    ca, cw = a.c_struct(), w.c_struct()
    _check(lib().nvfp4_grouped_gemm_out_scale(groups, slot_offsets.data_ptr(), group_rows.data_ptr(),
                                              C.byref(ca), C.byref(cw), w_globals.data_ptr(), n,
                                              out.data_ptr(), out.stride(0), out_global.data_ptr(),
                                              ws.ptr, ws.nbytes, _stream(stream)),
           "nvfp4_grouped_gemm_out_scale")
    return out, out_global


def nvfp4_check_status(workspace: Workspace | None = None, stream=None) -> int:
    """Synchronise, return and clear the workspace status word (0 = OK)."""
    ws = workspace or default_workspace()
    return int(lib().nvfp4_check_status(ws.ptr, _stream(stream)))


def nvfp4_status_string(status: int) -> str:
    return lib().nvfp4_status_string(status).decode()


def nvfp4_launch_count() -> int:
    return int(lib().nvfp4_launch_count())


def nvfp4_set_wait_limit_cycles(cycles: int) -> int:
    return int(lib().nvfp4_set_wait_limit_cycles(cycles))


def nvfp4_set_gemm_pairs(enable: bool) -> bool:
    return bool(lib().nvfp4_set_gemm_pairs(int(enable)))

"""Helpers shared by the GPU parity tests (test infrastructure)."""
import numpy as np
import torch

import oracle
from nvfp4_block_scaled_22_b200 import binding as nb


def to_host_quantized(t: nb.NVFP4Tensor) -> oracle.Quantized:
    """Copy a device NVFP4 tensor into the oracle's container."""
    return oracle.Quantized(t.codes.cpu().numpy(), t.scales.cpu().numpy(),
                            float(t.global_scale.cpu()[0]), t.rows, t.cols, t.layout)


def assert_quantized_equal(gpu: nb.NVFP4Tensor, ref: oracle.Quantized, what=""):
    h = to_host_quantized(gpu)
    assert np.float32(h.g) == np.float32(ref.g), f"{what}: g {h.g!r} != {ref.g!r}"
    if not np.array_equal(h.scales, ref.scales):
        bad = np.nonzero(h.scales != ref.scales)[0]
        raise AssertionError(f"{what}: {bad.size} scale bytes differ, first at {bad[:8]}: "
                             f"gpu {h.scales[bad[:8]]} ref {ref.scales[bad[:8]]}")
    if not np.array_equal(h.codes, ref.codes):
        bad = np.argwhere(h.codes != ref.codes)
        raise AssertionError(f"{what}: {len(bad)} code bytes differ, first at {bad[:4].tolist()}: "
                             f"gpu {h.codes[tuple(bad[:4].T)]} ref {ref.codes[tuple(bad[:4].T)]}")


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """Spacing of BF16 numbers at |v| (8 significant bits)."""
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126)
    return np.exp2(e - 7)


def gemm_tolerance(ref: np.ndarray, abs_sum: np.ndarray) -> np.ndarray:
    """Allowed |D - ref|: 1e-3 * sum_k |a_ik w_jk| (FP32 accumulation on the
    tensor cores) plus half a BF16 ulp of the result (output rounding)."""
    return 1e-3 * abs_sum + 0.5 * bf16_ulp(ref) + 1e-30


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def attention_chunking(tokens: int, heads_kv: int):
    """Tokens per chunk and chunk count of the attention read (about one CTA
    per SM of 148 over the KV heads, whole 256-token sub-tiles); the
    tolerance of the attention parity tests depends on it."""
    subs = -(-tokens // 256)
    want = max(1, min(subs, 148 // heads_kv))
    chunk = -(-subs // want) * 256
    return chunk, (-(-tokens // chunk) if tokens > 0 else 0)


def tile_samples(m, n, rng, tm=128, tn=256):
    """Outputs that touch every tm x tn output tile: per tile one random
    interior output, its last row at a random column, its last column at a
    random row, and its last (row, column) corner.  Any fault tied to a
    tile index, a CTA's wave or a ragged edge lands on at least one."""
    mt, nt = -(-m // tm), -(-n // tn)
    ti, tj = np.meshgrid(np.arange(mt), np.arange(nt), indexing="ij")
    ti, tj = ti.ravel(), tj.ravel()
    r0, c0 = ti * tm, tj * tn
    rl = np.minimum(r0 + tm, m) - 1                   # last row / column of the tile
    cl = np.minimum(c0 + tn, n) - 1
    ri = r0 + (rng.random(ti.size) * (rl - r0 + 1)).astype(np.int64)
    ci = c0 + (rng.random(tj.size) * (cl - c0 + 1)).astype(np.int64)
    return np.concatenate([ri, rl, ri, rl]), np.concatenate([ci, ci, cl, cl])

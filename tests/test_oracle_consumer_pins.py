"""Pins of the oracle's consumer steps: the MoE per-token combine ("NVIDIA
shrank GLM-5.2 to 4 bits", section 2: 8 of 256 experts per token) and the
NVFP4 -> FP8 conversion of the KV cache before attention ("FP4 KV-cache
quantization": current implementations dequantize to FP8)."""
import numpy as np
import torch

import oracle
from nvfp4_block_scaled_22_b200 import inputs


def _bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16)


def test_combine_one_hot_and_exact_sums():
    rng = np.random.default_rng(1)
    out = _bf16(rng.standard_normal((40, 64)))
    of = oracle.bf16_to_f32(oracle.bf16_bits(out))
    # weight 1 on one slot, 0 elsewhere: the selected row, bit for bit
    slots = rng.integers(0, 40, (10, 8)).astype(np.int32)
    w = np.zeros((10, 8), np.float32)
    w[:, 3] = 1.0
    y = oracle.moe_combine(out, slots, w)
    assert np.array_equal(y, oracle.bf16_bits(out)[slots[:, 3]])
    # small integers times powers of two: every partial sum exact
    ints = _bf16(rng.integers(-20, 21, (16, 32)))
    sl = rng.integers(0, 16, (6, 8)).astype(np.int32)
    ww = (2.0 ** -rng.integers(0, 4, (6, 8))).astype(np.float32)
    got = oracle.bf16_to_f32(oracle.moe_combine(ints, sl, ww)).astype(np.float64)
    vi = oracle.bf16_to_f32(oracle.bf16_bits(ints)).astype(np.float64)
    exact = np.einsum("tk,tkc->tc", ww.astype(np.float64), vi[sl])
    bf = oracle.bf16_to_f32(oracle.bf16_bits(_bf16(exact))).astype(np.float64)
    assert np.array_equal(got, bf)
    # a -1 slot contributes nothing
    sl2 = sl.copy()
    sl2[:, 7] = -1
    ww2 = ww.copy()
    ww2[:, 7] = 0.0
    assert np.array_equal(oracle.moe_combine(ints, sl2, ww), oracle.moe_combine(ints, sl, ww2))


def test_routing_weights_and_slots():
    r = inputs.MoeRouting()
    assert np.allclose(r.combine_weights.sum(1).numpy(), 1.0, atol=1e-6)
    assert torch.equal(r.gather[r.token_slots.view(-1).long()].long(),
                       torch.arange(r.tokens).repeat_interleave(r.topk))


def test_fp8_conversion_values():
    """Every (code, scale) pair: fp8 * RN(8/g) is within half an E4M3 step of
    the NVFP4 value, and exactly equal whenever e2m1 * s / 8 fits in E4M3."""
    e4m3 = np.array([oracle.e4m3_decode(b) for b in range(256)])
    e2m1 = np.array([oracle.e2m1_decode(c) for c in range(16)])
    rows, cols = 127, 256                       # row r uses scale code r + 1 (finite ones)
    codes = np.zeros((rows, cols // 2), np.uint8)
    cvals = np.tile(np.arange(16, dtype=np.uint8), cols // 16)
    codes[:] = (cvals[0::2] | (cvals[1::2] << 4))[None, :]
    scales = np.zeros(oracle.scales_bytes(rows, cols, oracle.SF_LINEAR), np.uint8)
    scales[:] = np.repeat(np.arange(1, 128, dtype=np.uint8), cols // 16)[: scales.size]
    scales[scales == 0x7F] = 0x7E
    g = np.float32(3.0)
    q = oracle.Quantized(codes, scales, g, rows, cols, oracle.SF_LINEAR)
    y, fs = oracle.dequantize_fp8(q)
    assert fs == np.float32(8.0) / g
    for r in range(rows):
        s = e4m3[scales[r * (cols // 16)]]
        for c in range(16):
            exact = e2m1[c] * s / 8.0
            got = e4m3[y[r, c]]
            finite = np.abs(e4m3[np.isfinite(e4m3)])
            if abs(exact) in set(finite):
                assert got == exact or (exact == 0 and got == 0)
            else:
                # E4M3 spacing: 2^(e-3) in binade e >= -6, 2^-9 for subnormals
                e = max(np.floor(np.log2(abs(exact))), -6)
                assert abs(got - exact) <= 2.0 ** (e - 3) / 2
            assert got == 0 or np.sign(got) == np.sign(exact)

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


def test_exp_against_libm_and_its_constants():
    """The fixed-order exp stays within 2 ulp of the correctly rounded value
    on a dense sweep, and its ln 2 split is exact: L_hi + L_lo = ln 2 to the
    precision of the sum."""
    import math
    xs = np.float32(np.linspace(-87, 87, 200001))
    worst = 0.0
    for x in xs[::7]:
        got = np.float32(oracle.exp_ref(float(x)))
        ref = math.exp(float(x))
        ulp = np.spacing(np.float32(ref))
        worst = max(worst, abs(float(got) - ref) / float(ulp))
    assert worst <= 2.0
    assert 0.693145751953125 * 65536 == 45426
    assert abs(0.693145751953125 + float(np.float32(math.log(2) - 0.693145751953125)) - math.log(2)) < 1e-13


def test_silu_closed_forms():
    assert oracle.swiglu(0.0, 1.0) == 0.0
    for g in (20.0, 50.0, 87.5):
        assert oracle.swiglu(g, 1.0) == np.float32(g)           # sigmoid rounds to 1
    for g in (-100.0, -90.0):
        assert abs(oracle.swiglu(g, 1.0)) < 1e-35               # silu(-large) -> -0
    rng = np.random.default_rng(3)
    for g in rng.standard_normal(200) * 4:
        g = float(np.float32(g))
        ref = g / (1 + np.exp(-g))
        assert abs(oracle.swiglu(g, 1.0) - ref) <= 4 * np.spacing(np.float32(abs(ref))) + 1e-45


def test_quantize_swiglu_reduces_to_plain_quantize():
    """gate >= 20 makes silu(gate) = gate exactly; with up a power of two the
    product is exact, so quantize_swiglu([gate | up]) = quantize(gate * up)."""
    rng = np.random.default_rng(4)
    gate = 20.0 + np.abs(rng.standard_normal((40, 64))) * 50
    up = 2.0 ** rng.integers(-3, 4, (40, 64))
    gu = _bf16(np.concatenate([gate, up], axis=1))
    gf = oracle.bf16_to_f32(oracle.bf16_bits(gu))
    prod = _bf16(gf[:, :64].astype(np.float64) * gf[:, 64:])
    assert np.array_equal(oracle.bf16_to_f32(oracle.bf16_bits(prod)), gf[:, :64] * gf[:, 64:])
    st, qs = oracle.quantize_swiglu(gu)
    st2, qp = oracle.quantize(prod)
    assert st == st2 == oracle.OK and np.float32(qs.g) == np.float32(qp.g)
    assert np.array_equal(qs.codes, qp.codes) and np.array_equal(qs.scales, qp.scales)
    zero = _bf16(np.concatenate([gate, np.zeros_like(up)], axis=1))
    st, qz = oracle.quantize_swiglu(zero)
    assert st == oracle.OK and qz.g == 1.0 and not qz.scales.any()

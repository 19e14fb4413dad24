"""Pins of the oracle's stochastic rounding ("NVFP4: how NVIDIA pre-trained
a 12B model on 10T tokens", section "Four stabilisation devices": gradients
are rounded stochastically -- a value 0.7 of the way to the next grid point
goes up with probability 0.7) and of the counter-based generator behind it
(Philox4x32-10, pinned by its published known-answer vectors)."""
import math

import numpy as np
import torch

import oracle
from tests.golden_io import read_lines

GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_philox_known_answers():
    for ln in read_lines("philox4x32_10_kat.txt"):
        w = [int(t, 16) for t in ln.split()]
        assert oracle.philox4x32_10(w[0:4], w[4:6]) == w[6:10]


def test_grid_values_never_move():
    for k, v in enumerate(GRID):
        for u in (0, 1, 12345, 65535):
            assert oracle.e2m1_sr(v, u) == k
            assert oracle.e2m1_sr(-v, u) == (k | 8)
    for u in (0, 65535):
        assert oracle.e2m1_sr(7.0, u) == 7 and oracle.e2m1_sr(-1e30, u) == 15


def _prob_up(v):
    """Fraction of the 65536 draws that round v up, by enumeration."""
    codes = np.array([oracle.e2m1_sr(v, u) for u in range(0, 65536, 1)])
    lo = max(k for k, g in enumerate(GRID) if g <= abs(v))
    assert set(np.unique(codes & 7)) <= {lo, lo + 1}
    return float(np.mean((codes & 7) == lo + 1)), lo


def test_page_example_probability():
    """The page's 0.7 example on the grid segment [2, 3]: 2.7 goes to 3 with
    probability 0.7 (exactly ceil(0.7 * 2^16) / 2^16 with 16-bit draws)."""
    v = float(np.float32(2.7))
    p, lo = _prob_up(v)
    frac = (v - 2.0) / 1.0
    assert GRID[lo] == 2.0 and p == math.ceil(frac * 65536) / 65536
    assert abs(p - 0.7) < 1e-4


def test_unbiased_in_expectation_on_every_segment():
    rng = np.random.default_rng(1)
    for lo_i in range(7):
        a, b = GRID[lo_i], GRID[lo_i + 1]
        for _ in range(3):
            v = float(np.float32(a + (b - a) * rng.random()))
            p, lo = _prob_up(v)
            frac = (v - a) / (b - a)
            assert p == math.ceil(frac * 65536) / 65536
            mean = a + p * (b - a)
            assert abs(mean - v) <= (b - a) / 65536


def test_block_draws_are_the_documented_philox_words():
    seed, r, b, cols = 0x0123456789ABCDEF, 5, 3, 64
    u = oracle.sr_block_draws(seed, r, b, cols)
    n = r * (cols // 16) + b
    for j in range(2):
        w = oracle.philox4x32_10([n & 0xFFFFFFFF, n >> 32, j, 0], [seed & 0xFFFFFFFF, seed >> 32])
        for i in range(4):
            assert u[8 * j + 2 * i] == (w[i] & 0xFFFF) and u[8 * j + 2 * i + 1] == (w[i] >> 16)


def _bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16)


def test_quantize_sr_shares_scales_and_picks_a_neighbour():
    rng = np.random.default_rng(2)
    x = _bf16(rng.standard_normal((40, 96)) * 3)
    st, qr = oracle.quantize(x, oracle.SF_LINEAR)
    st2, qs = oracle.quantize_sr(x, 77, oracle.SF_LINEAR)
    assert st == st2 == oracle.OK
    assert np.float32(qr.g) == np.float32(qs.g) and np.array_equal(qr.scales, qs.scales)
    xf = oracle.bf16_to_f32(oracle.bf16_bits(x))
    e2m1 = np.array([oracle.e2m1_decode(c) for c in range(16)])
    nib = np.zeros((40, 96), np.uint8)
    nib[:, 0::2], nib[:, 1::2] = qs.codes & 15, qs.codes >> 4
    g = np.float32(qs.g)
    for r in range(40):
        for c in range(96):
            s = qs.scales[r * 6 + c // 16]
            e = np.float32(0) if s == 0 else np.float32(g / np.float32(oracle.e4m3_decode(int(s))))
            y = float(np.float32(xf[r, c]) * e)
            got = abs(e2m1[nib[r, c]])
            below = max(v for v in GRID if v <= min(abs(y), 6.0))
            above = min((v for v in GRID if v >= min(abs(y), 6.0)), default=6.0)
            assert got in (below, above)


def test_quantize_sr_averages_to_the_value():
    """Dequantized SR tensors over many seeds average to x * e / g times the
    block factor, i.e. to the unrounded value, within the sampling error."""
    rng = np.random.default_rng(3)
    x = _bf16(rng.standard_normal((4, 32)))
    xf = oracle.bf16_to_f32(oracle.bf16_bits(x)).astype(np.float64)
    acc = np.zeros_like(xf)
    n = 400
    for seed in range(n):
        st, q = oracle.quantize_sr(x, seed, oracle.SF_LINEAR)
        acc += oracle.bf16_to_f32(q.dequantize())
    err = np.abs(acc / n - xf)
    _, qr = oracle.quantize(x, oracle.SF_LINEAR)
    step = np.abs(oracle.bf16_to_f32(qr.dequantize()) - xf).max() * 2 + 1e-6
    assert err.max() < 0.25 * step


def test_quantize_sr_with_rht_matches_rht_scales():
    rng = np.random.default_rng(4)
    x = _bf16(rng.standard_normal((20, 64)))
    st, qh = oracle.quantize_rht(x, 0x5A5A)
    st2, qs = oracle.quantize_sr(x, 9, sign_mask=0x5A5A)
    assert st == st2 == oracle.OK
    assert np.float32(qh.g) == np.float32(qs.g) and np.array_equal(qh.scales, qs.scales)

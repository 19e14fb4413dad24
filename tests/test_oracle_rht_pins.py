"""Pins of the oracle's random Hadamard transform and of quantization after
it ("NVFP4: how NVIDIA pre-trained a 12B model on 10T tokens", section
"Four stabilisation devices": a 16x16 Hadamard matrix and a random +-1 sign
vector applied to the Wgrad inputs before they are quantized).

The Hadamard matrix here is built independently of the oracle, as the
Kronecker power of the 2x2 matrix [[1, 1], [1, -1]] (Sylvester's
construction), so a wrong butterfly stride, a dropped stage, a wrong sign
bit or a wrong normalisation in the oracle fails these checks.
"""
import numpy as np
import pytest
import torch

import oracle

H2 = np.array([[1.0, 1.0], [1.0, -1.0]])
H16 = np.kron(np.kron(np.kron(H2, H2), H2), H2)


def _signs(mask):
    return np.array([-1.0 if (mask >> j) & 1 else 1.0 for j in range(16)])


def _rht_f64(x, mask):
    return 0.25 * H16 @ (_signs(mask) * np.asarray(x, np.float64))


def test_sylvester_matrix_is_orthogonal():
    assert np.array_equal(H16 @ H16.T, 16 * np.eye(16))
    assert np.array_equal(H16, H16.T)


def test_unit_vectors_give_the_hadamard_columns():
    """rht16(e_k, 0) = column k of H16 / 4, for every k: the one-hot closed form."""
    for k in range(16):
        e = np.zeros(16, np.float32)
        e[k] = 1.0
        assert np.array_equal(oracle.rht16(e, 0), 0.25 * H16[:, k])


def test_sign_bit_j_negates_input_j():
    rng = np.random.default_rng(3)
    for mask in [0x0001, 0x8000, 0xA5A5, 0xFFFF, 0x1234]:
        x = rng.integers(-64, 65, 16).astype(np.float32)
        # integer inputs: every partial sum is exact in FP32
        assert np.array_equal(oracle.rht16(x, mask), _rht_f64(x, mask))


def test_random_inputs_within_fp32_butterfly_bound():
    """Four rounded add/sub stages and an exact quarter: each output is within
    4 * 2^-24 * (sum |x|) / 4 of the exact transform."""
    rng = np.random.default_rng(4)
    for t in range(200):
        mask = int(rng.integers(0, 1 << 16))
        x = (rng.standard_normal(16) * 10.0 ** rng.integers(-3, 4)).astype(np.float32)
        got = oracle.rht16(x, mask).astype(np.float64)
        exact = _rht_f64(x, mask)
        bound = 4 * 2.0 ** -24 * np.abs(x.astype(np.float64)).sum() / 4 * 1.0001
        assert np.all(np.abs(got - exact) <= bound)


def test_norm_preserved_and_inverse_recovers():
    rng = np.random.default_rng(5)
    for t in range(50):
        mask = int(rng.integers(0, 1 << 16))
        x = rng.integers(-1000, 1001, 16).astype(np.float32)
        y = oracle.rht16(x, mask)
        assert float(np.dot(y.astype(np.float64), y)) == pytest.approx(float(np.dot(x.astype(np.float64), x)),
                                                                   rel=1e-12)
        assert np.array_equal(oracle.rht16_inverse(y, mask), x)


def test_shared_transform_keeps_dot_products():
    """Both GEMM operands transformed with the same signs along the
    contraction axis: a . w is unchanged (the transform is orthogonal)."""
    rng = np.random.default_rng(6)
    mask = 0x6B1D
    a = rng.integers(-50, 51, 16).astype(np.float32)
    w = rng.integers(-50, 51, 16).astype(np.float32)
    ya, yw = oracle.rht16(a, mask), oracle.rht16(w, mask)
    assert float(np.dot(ya.astype(np.float64), yw)) == float(np.dot(a.astype(np.float64), w))


def _bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16)


def test_quantize_rht_equals_plain_quantize_of_the_transformed_tensor():
    """Choose the transformed tensor y first (multiples of 4 of small
    integers, exact in BF16), set x = inverse transform of y (small integers,
    exact in BF16): quantize_rht(x) must equal quantize(y) bit for bit."""
    rng = np.random.default_rng(7)
    rows, cols = 130, 96
    for mask in [0, 0x0F0F, 0xC3A5]:
        y = 4.0 * rng.integers(-8, 9, (rows, cols))
        y[5, :16] = 0.0                                     # an all-zero block
        s = _signs(mask)
        x = np.empty_like(y)
        for r in range(rows):
            for b in range(cols // 16):
                x[r, b * 16:(b + 1) * 16] = s * (0.25 * H16 @ y[r, b * 16:(b + 1) * 16])
        assert np.array_equal(x, np.round(x)) and np.abs(x).max() <= 256
        for layout in (oracle.SF_SWIZZLED, oracle.SF_LINEAR):
            st1, q1 = oracle.quantize_rht(_bf16(x), mask, layout)
            st2, q2 = oracle.quantize(_bf16(y), layout)
            assert st1 == st2 == oracle.OK
            assert np.float32(q1.g) == np.float32(q2.g)
            assert np.array_equal(q1.codes, q2.codes)
            assert np.array_equal(q1.scales, q2.scales)


def test_quantize_rht_supplied_global_and_errors():
    rng = np.random.default_rng(8)
    x = _bf16(rng.standard_normal((20, 64)))
    st, q = oracle.quantize_rht(x, 0x1357)
    assert st == oracle.OK
    st2, q2 = oracle.quantize_rht(x, 0x1357, g=q.g)
    assert st2 == oracle.OK and np.array_equal(q.codes, q2.codes) and np.array_equal(q.scales, q2.scales)
    bad = x.clone()
    bad[3, 17] = float("inf")
    assert oracle.quantize_rht(bad, 0x1357)[0] == oracle.ERR_NONFINITE
    zero = torch.zeros((4, 32), dtype=torch.bfloat16)
    st, qz = oracle.quantize_rht(zero, 0xFFFF)
    assert st == oracle.OK and qz.g == 1.0 and not qz.scales.any()
    # all signs flipped: -0 inputs.  IEEE sums keep -0 only in output 0 of
    # each block (-0 + -0 = -0 at every stage; any difference is +0), so the
    # low nibble of byte 0 of each 8-byte block holds the negative zero code
    assert np.all(qz.codes[:, [0, 8]] == 0x08)
    assert not np.any(np.delete(qz.codes, [0, 8], axis=1))

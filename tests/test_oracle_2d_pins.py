"""Pins of the oracle's 2D (16x16 block) weight quantization ("NVFP4: how
NVIDIA pre-trained a 12B model on 10T tokens", section "Four stabilisation
devices": weights use 16x16 blocks so that W and its transpose are
quantized the same way).

Each check ties the 2D quantizer to the already pinned 1D one or to a
property the pages state: rows that repeat inside every 16-row group reduce
it to the 1D quantizer; the transposed tensor quantizes to the transposed
codes with the same block scales; every 2D scale is the largest of the 1D
scales of its 16 rows (E4M3 rounding is monotone); every code is the 1D
encode of its value under the block's scale.
"""
import numpy as np
import torch

import oracle


def _bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16)


def _rand(rows, cols, seed, outliers=0.01):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols))
    m = rng.random((rows, cols)) < outliers
    x[m] *= 40
    return _bf16(x)


def _scale_matrix(q):
    """[rows x cols/16] E4M3 codes of a quantized tensor."""
    s = np.zeros((q.rows, q.cols // 16), np.uint8)
    for r in range(q.rows):
        for b in range(q.cols // 16):
            s[r, b] = q.scales[oracle.sf_offset(r, b, q.rows, q.cols, q.layout)]
    return s


def _nibbles(q):
    c = np.zeros((q.rows, q.cols), np.uint8)
    c[:, 0::2] = q.codes & 15
    c[:, 1::2] = q.codes >> 4
    return c


def test_repeated_rows_reduce_to_1d():
    base = _rand(5, 96, 1)
    x = torch.repeat_interleave(base, 16, dim=0)          # 80 rows, groups of 16 equal rows
    for layout in (oracle.SF_SWIZZLED, oracle.SF_LINEAR):
        st2, q2 = oracle.quantize_2d(x, layout)
        st1, q1 = oracle.quantize(x, layout)
        assert st1 == st2 == oracle.OK
        assert np.float32(q1.g) == np.float32(q2.g)
        assert np.array_equal(q1.codes, q2.codes) and np.array_equal(q1.scales, q2.scales)


def test_transpose_has_transposed_codes_and_the_same_block_scales():
    x = _rand(96, 160, 2)
    st, q = oracle.quantize_2d(x, oracle.SF_LINEAR)
    st_t, qt = oracle.quantize_2d(x.t().contiguous(), oracle.SF_LINEAR)
    assert st == st_t == oracle.OK and np.float32(q.g) == np.float32(qt.g)
    assert np.array_equal(_nibbles(qt), _nibbles(q).T)
    s, st_ = _scale_matrix(q), _scale_matrix(qt)
    for r in range(96):
        for c in range(160):
            assert s[r, c // 16] == st_[c, r // 16]


def test_block_scale_is_max_of_row_scales_and_codes_follow_it():
    x = _rand(50, 64, 3)                                  # partial last group (2 rows)
    x[16:32, 16:32] = 0.0                                 # one all-zero 16x16 block
    st, q2 = oracle.quantize_2d(x, oracle.SF_LINEAR)
    _, q1 = oracle.quantize(x, oracle.SF_LINEAR)
    assert np.float32(q1.g) == np.float32(q2.g)
    s1, s2 = _scale_matrix(q1), _scale_matrix(q2)
    for a in range(0, 50, 16):
        grp = s1[a:a + 16]
        assert np.all(s2[a:a + 16] == grp.max(axis=0))
    assert np.all(s2[16:32, 1] == 0) and not np.any(_nibbles(q2)[16:32, 16:32] & 7)
    # codes: the 1D encode of each value under its block's scale
    xf = oracle.bf16_to_f32(oracle.bf16_bits(x))
    g = np.float32(q2.g)
    nib = _nibbles(q2)
    for r in range(50):
        for c in range(64):
            sc = s2[r, c // 16]
            e = np.float32(0) if sc == 0 else np.float32(g / np.float32(oracle.e4m3_decode(int(sc))))
            assert nib[r, c] == oracle.e2m1_rne(np.float32(xf[r, c]) * e)


def test_supplied_scale_and_errors():
    x = _rand(32, 32, 4)
    st, q = oracle.quantize_2d(x)
    st2, q2 = oracle.quantize_2d(x, g=q.g)
    assert st == st2 == oracle.OK and np.array_equal(q.codes, q2.codes)
    bad = x.clone()
    bad[1, 1] = float("nan")
    assert oracle.quantize_2d(bad)[0] == oracle.ERR_NONFINITE

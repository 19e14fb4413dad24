"""Pins of the oracle's attention read over an NVFP4 KV cache ("FP4 KV-cache
quantization": every decode step re-reads the cache, whose FP4 values are
restored before the attention arithmetic).

The K and V values are restored here with this file's own E2M1 and E4M3
tables, and the reference softmax is numpy's, so a wrong head mapping, a
wrong scale position, a dropped token or a missing normalisation in the
oracle fails one of these checks."""
import math

import numpy as np
import torch

import oracle

GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _e4m3(b):
    s, e, m = b >> 7, (b >> 3) & 15, b & 7
    if e == 15 and m == 7:
        return math.nan
    v = (m / 8) * 2.0 ** -6 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
    return -v if s else v


def _restore(q):
    """Exact values of a linear-layout NVFP4 tensor, decoded independently."""
    nib = np.zeros((q.rows, q.cols), np.int64)
    nib[:, 0::2], nib[:, 1::2] = q.codes & 15, q.codes >> 4
    mag = GRID[nib & 7] * np.where(nib & 8, -1.0, 1.0)
    sc = np.array([_e4m3(int(b)) for b in q.scales], np.float64).reshape(q.rows, q.cols // 16)
    return mag * np.repeat(sc, 16, axis=1) / np.float64(np.float32(q.g))


def _bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16)


def _kv(tokens, heads_kv, head_dim, seed, layout=oracle.SF_LINEAR):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((tokens, heads_kv * head_dim))
    v = rng.standard_normal((tokens, heads_kv * head_dim)) + 0.5
    st1, qk = oracle.quantize(_bf16(k), layout)
    st2, qv = oracle.quantize(_bf16(v), layout)
    assert st1 == st2 == oracle.OK
    return qk, qv


def _numpy_attention(q, qk, qv, heads_kv, scale):
    qf = oracle.bf16_to_f32(oracle.bf16_bits(q)).astype(np.float64)
    heads_q, d = qf.shape
    K, V = _restore(qk), _restore(qv)
    out = np.zeros((heads_q, d))
    for h in range(heads_q):
        c0 = (h // (heads_q // heads_kv)) * d
        s = scale * (K[:, c0:c0 + d] @ qf[h])
        p = np.exp(s - s.max())
        out[h] = p @ V[:, c0:c0 + d] / p.sum()
    return out


def test_brute_force_on_small_caches_both_layouts():
    rng = np.random.default_rng(1)
    for tokens, heads_kv, group, d in [(37, 2, 3, 32), (1, 1, 1, 16), (130, 3, 2, 48)]:
        q = _bf16(rng.standard_normal((heads_kv * group, d)))
        scale = 1.0 / math.sqrt(d)
        outs = []
        for layout in (oracle.SF_LINEAR, oracle.SF_SWIZZLED):
            qk, qv = _kv(tokens, heads_kv, d, 2 + tokens, layout)
            st, o, ao, sa = oracle.attention_decode(q, qk, qv, heads_kv, scale)
            assert st == oracle.OK
            outs.append(o)
            if layout == oracle.SF_LINEAR:
                ref = _numpy_attention(q, qk, qv, heads_kv, scale)
                assert np.all(np.abs(o - ref) <= 1e-12 * ao)
                assert np.all(ao >= np.abs(o) * (1 - 1e-12))
        assert np.array_equal(outs[0], outs[1])


def test_zero_query_gives_the_mean_value_row():
    qk, qv = _kv(257, 4, 32, 5)
    q = _bf16(np.zeros((8, 32)))
    st, o, ao, sa = oracle.attention_decode(q, qk, qv, 4, 0.125)
    V = _restore(qv)
    for h in range(8):
        c0 = (h // 2) * 32
        assert np.allclose(o[h], V[:, c0:c0 + 32].mean(axis=0), rtol=0, atol=1e-13)
    assert not sa.any()


def test_a_dominant_token_returns_its_value_row():
    tokens, heads_kv, d = 300, 2, 32
    rng = np.random.default_rng(6)
    k = rng.uniform(-1, 1, (tokens, heads_kv * d))
    star = {0: 123, 1: 299}                         # the dominant token per KV head
    for hk, t in star.items():
        k[t, hk * d + 5] = 100.0
    _, qk = oracle.quantize(_bf16(k), oracle.SF_LINEAR)
    _, qv = _kv(tokens, heads_kv, d, 7)
    q = np.zeros((4, d))
    q[:, 5] = 1.0
    st, o, _, _ = oracle.attention_decode(_bf16(q), qk, qv, heads_kv, 1000.0)
    V = _restore(qv)
    for h in range(4):
        hk = h // 2
        assert np.array_equal(o[h], V[star[hk], hk * d:(hk + 1) * d])


def test_token_order_does_not_matter():
    qk, qv = _kv(96, 2, 32, 8)
    rng = np.random.default_rng(9)
    q = _bf16(rng.standard_normal((4, 32)))
    perm = rng.permutation(96)
    sf_cols = qk.cols // 16

    def permuted(t):
        return oracle.Quantized(t.codes[perm].copy(), t.scales.reshape(-1, sf_cols)[perm].ravel().copy(),
                                t.g, t.rows, t.cols, t.layout)

    _, o1, ao, _ = oracle.attention_decode(q, qk, qv, 2, 0.2)
    _, o2, _, _ = oracle.attention_decode(q, permuted(qk), permuted(qv), 2, 0.2)
    assert np.all(np.abs(o1 - o2) <= 1e-13 * ao)


def test_head_range_and_score_bound():
    qk, qv = _kv(50, 2, 32, 10)
    rng = np.random.default_rng(11)
    q = _bf16(rng.standard_normal((6, 32)))
    _, o_all, ao_all, sa_all = oracle.attention_decode(q, qk, qv, 2, 0.3)
    _, o_part, _, sa_part = oracle.attention_decode(q, qk, qv, 2, 0.3, heads=(2, 5))
    assert np.array_equal(o_part, o_all[2:5]) and np.array_equal(sa_part, sa_all[2:5])
    K = _restore(qk)
    qf = oracle.bf16_to_f32(oracle.bf16_bits(q)).astype(np.float64)
    for h in range(6):
        c0 = (h // 3) * 32
        want = 0.3 * np.abs(K[:, c0:c0 + 32] * qf[h]).sum(axis=1).max()
        assert abs(sa_all[h] - want) <= 1e-12 * want


def test_empty_cache_and_bad_shapes():
    qk, qv = _kv(0, 2, 32, 12)
    q = _bf16(np.ones((4, 32)))
    st, o, ao, _ = oracle.attention_decode(q, qk, qv, 2, 0.1)
    assert st == oracle.OK and not o.any() and not ao.any()
    qk, qv = _kv(8, 2, 32, 13)
    assert oracle.attention_decode(_bf16(np.ones((3, 32))), qk, qv, 2, 0.1)[0] == oracle.ERR_SHAPE

"""GPU parity of the decode attention read over an NVFP4 KV cache against
the oracle's FP64 attention on the exact restored values.

Tolerance, derived from the kernel's FP32 arithmetic (u = 2^-24):
  * scores (log2 units): exact products of BF16 operands summed in FP32
    over eight 16-term tensor-core steps, then one multiply by
    RN(RN(scale * log2 e) / g_K): allowed 68u * log2(e) * score_abs,
    score_abs = max_t |scale| sum_d |q_d k_td| (more than the eight steps
    lose even if each step's internal sum is off by 2 ulp of each of its 16
    products);
  * weights: exp2 of (score - running max), the subtraction (at most
    2u * log2(e) * score_abs) and exp2 itself (2 ulp), and the rescales of
    the chunk merge (2 ulp): relative error eps <= 72u * score_abs + 8u
    (ln 2 * log2 e = 1);
  * a weighted mean with weights perturbed by eps moves by at most
    2 eps * sum_t p_t |v_t| / sum_t p_t (the oracle's abs_o); the FP32 sums
    add n u * abs_o to numerator and denominator, n = twice the tensor-core
    steps of an accumulator chain (each step adds 8 exact products -- the
    restored V values times the three exact TF32 parts of a weight -- to
    the accumulator and is off by at most 2 ulp of the sum of its terms'
    magnitudes, as for the scores; 4 k-steps x 3 weight parts = 12 steps per
    256 tokens of a chunk) + rescales + reduction levels + chunks (the
    weight sums run as plain FP32 additions, fewer per chain); two final
    divisions 2u.
The bound below is twice that, plus half a BF16 ulp for the output rounding.
Where the FP64 result lies farther than the FP32 bound from a BF16 rounding
midpoint, the BF16 output must equal its correct rounding exactly; that
holds for most elements and checks the FP32 result much more tightly than
the BF16 spacing."""
import math

import numpy as np
import pytest
import torch

import oracle
from nvfp4_block_scaled_22_b200 import binding as nb
from nvfp4_block_scaled_22_b200 import inputs
from tests.gpu_util import assert_quantized_equal, attention_chunking, bf16_to_f64, bf16_ulp

pytestmark = pytest.mark.gpu
DEV = "cuda"
U = 2.0 ** -24


@pytest.fixture(scope="module", autouse=True)
def _lib():
    nb.lib()
    yield
    assert nb.nvfp4_check_status() == 0


def _fp32_bound(abs_o, score_abs, tokens, heads_kv):
    chunk, n_chunks = attention_chunking(max(tokens, 1), heads_kv)
    eps = 72 * U * score_abs[:, None] + 8 * U
    n = 2 * 12 * chunk / 256 + 2 * chunk / 256 + 8 + n_chunks + 8
    return 2 * (2 * eps + 2 * n * U + 2 * U) * abs_o


def _check(o_gpu, o_ref, abs_o, bound, what=""):
    got = bf16_to_f64(o_gpu)
    err = np.abs(got - o_ref)
    lim = bound + 0.5 * bf16_ulp(o_ref) + 1e-30
    if not np.all(err <= lim):
        i = np.unravel_index(np.argmax(err - lim), err.shape)
        raise AssertionError(f"{what}: |o - ref| {err[i]:.3e} > {lim[i]:.3e} at {i}: "
                             f"gpu {got[i]!r} ref {o_ref[i]!r}")
    # the BF16 neighbours of the FP64 result and their midpoint
    bits = o_ref.astype(np.float32).view(np.uint32) & np.uint32(0xFFFF0000)
    lo = bits.view(np.float32).astype(np.float64)
    hi = (bits + np.uint32(0x10000)).view(np.float32).astype(np.float64)
    mid = 0.5 * (lo + hi)
    nearest = np.where(np.abs(o_ref) < np.abs(mid), lo, hi)
    clear = np.abs(np.abs(o_ref) - np.abs(mid)) > bound + np.abs(o_ref) * 2.0 ** -23
    assert np.array_equal(got[clear], nearest[clear]), f"{what}: BF16 rounding differs"
    assert np.all((got[~clear] == lo[~clear]) | (got[~clear] == hi[~clear]))
    return clear.mean()


def _quantize_kv(x):
    """NVFP4 (linear scale layout) on the GPU, compared with the oracle's."""
    q = nb.nvfp4_quantize(x.to(DEV), layout=nb.SF_LINEAR)
    st, r = oracle.quantize(x, oracle.SF_LINEAR)
    assert st == oracle.OK
    assert_quantized_equal(q, r, "KV")
    return q, r


def _bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16)


def _run(q, k, v, heads_kv, scale, heads=None, what=""):
    qk, rk = _quantize_kv(k)
    qv, rv = _quantize_kv(v)
    o = nb.nvfp4_attention_decode(q.to(DEV), qk, qv, heads_kv, scale)
    torch.cuda.synchronize()
    assert nb.nvfp4_check_status() == 0
    st, o_ref, abs_o, score_abs = oracle.attention_decode(q, rk, rv, heads_kv, scale, heads)
    assert st == oracle.OK
    sel = slice(None) if heads is None else slice(*heads)
    bound = _fp32_bound(abs_o, score_abs, k.shape[0], heads_kv)
    return _check(o[sel], o_ref, abs_o, bound, what)


@pytest.mark.parametrize("tokens,heads_kv,group", [(1, 1, 1), (37, 2, 3), (300, 3, 5),
                                                    (1000, 8, 8), (4099, 4, 8)])
def test_small_caches_against_oracle(tokens, heads_kv, group):
    """Ragged sub-tiles and chunks, groups below 8 (idle head slots), one
    token, several chunks per KV head."""
    rng = np.random.default_rng(tokens * 31 + heads_kv)
    k = _bf16(rng.standard_normal((tokens, heads_kv * 128)))
    v = _bf16(rng.standard_normal((tokens, heads_kv * 128)) + 0.25)
    q = _bf16(rng.standard_normal((heads_kv * group, 128)))
    frac = _run(q, k, v, heads_kv, 1.0 / math.sqrt(128), what=f"T={tokens}")
    assert frac > 0.5


def test_zero_query_averages_every_chunk():
    """q = 0: every token weighs the same and o is the mean value row.  V
    carries a ramp over the tokens, so a dropped or doubled chunk or
    sub-tile moves the mean far outside the bound."""
    tokens, heads_kv = 5000, 2
    rng = np.random.default_rng(5)
    ramp = np.linspace(-4.0, 4.0, tokens)[:, None]
    v = _bf16(rng.standard_normal((tokens, heads_kv * 128)) * 0.1 + ramp)
    k = _bf16(rng.standard_normal((tokens, heads_kv * 128)))
    q = _bf16(np.zeros((heads_kv * 4, 128)))
    _run(q, k, v, heads_kv, 0.088, what="zero query")


def test_dominant_tokens_in_the_last_chunk():
    """Peaked weights: for the first query head of each group one token in
    the ragged last sub-tile dominates, so every earlier chunk must be
    rescaled down by the running maximum."""
    tokens, heads_kv, group = 20000, 8, 8
    rng = np.random.default_rng(6)
    qn = rng.standard_normal((heads_kv * group, 128))
    kn = rng.standard_normal((tokens, heads_kv * 128))
    for j in range(heads_kv):
        t = tokens - 1 - 7 * j
        kn[t, j * 128:(j + 1) * 128] = 3.0 * np.sign(qn[j * group])
    v = _bf16(rng.standard_normal((tokens, heads_kv * 128)))
    _run(_bf16(qn), _bf16(kn), v, heads_kv, 1.0, heads=(0, 2 * group), what="dominant")


def test_empty_cache_writes_zeros():
    k = nb.NVFP4Tensor.empty(0, 1024, nb.SF_LINEAR, DEV)
    k.global_scale.fill_(1.0)
    q = torch.ones((64, 128), dtype=torch.bfloat16, device=DEV)
    o = nb.nvfp4_attention_decode(q, k, k, 8)
    torch.cuda.synchronize()
    assert not o.float().abs().sum().item()


def test_full_kv_layer_sampled_heads():
    """One layer of the KV workload: 131072 tokens x 8 KV heads x 128 with
    its outlier channels, 64 query heads; the oracle computes four query
    heads from different KV heads."""
    tokens = inputs.KV_TOKENS
    k = inputs.kv_tensor(0, 0).view(tokens, -1)
    v = inputs.kv_tensor(0, 1).view(tokens, -1)
    q = inputs.kv_query(0)
    qk, rk = _quantize_kv(k)
    qv, rv = _quantize_kv(v)
    o = nb.nvfp4_attention_decode(q.to(DEV), qk, qv, inputs.KV_HEADS)
    torch.cuda.synchronize()
    for h in (0, 21, 42, 63):
        st, o_ref, abs_o, score_abs = oracle.attention_decode(q, rk, rv, inputs.KV_HEADS,
                                                              1.0 / math.sqrt(128), (h, h + 1))
        bound = _fp32_bound(abs_o, score_abs, tokens, inputs.KV_HEADS)
        _check(o[h:h + 1], o_ref, abs_o, bound, f"head {h}")
    # the same call twice gives the same bits (fixed chunking and order)
    o2 = nb.nvfp4_attention_decode(q.to(DEV), qk, qv, inputs.KV_HEADS)
    assert torch.equal(o.view(torch.int16), o2.view(torch.int16))

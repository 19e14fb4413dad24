"""Seeded synthetic inputs for the five NVFP4 workloads.

This module only draws numbers.  It holds none of the quantization or GEMM
arithmetic, so both the CUDA path and the CPU oracle can take their inputs
from here without sharing any of the method.

Workloads (shapes and value mixes stand in for the pages' models, none of
which ships weights here):

* ``tiny``      -- W4A4 linear, A 128x256 and W 256x256, N(0,1), 0.5% of the
  entries x30, one all-zero 16-block per row.
* ``sweep``     -- standalone quantize of n in {2^20, 2^24, 2^28} values as
  [n/4096, 4096]: N(0,1), 0.1% x50, 1% replaced by c*2^k with c a nonzero
  E2M1 grid value and k in [-4, 4].
* ``ffn``       -- dense FFN linear of a 12B hybrid model: W 20480x5120
  N(0, 0.02^2); A Mx5120 N(0,1) with 1% of the K columns x20 (M in
  {16, 512, 8192}).
* ``moe``       -- 256 experts, top-8 routing of 4096 tokens (router logits
  N(0,1)), hidden 6144, expert intermediate 2048.
* ``kv``        -- KV cache, 32 layers x {K,V} x [131072 tokens x 8 heads x
  128], N(0,1) with 5 of the 1024 (head, dim) channels x10.
* ``wgrad``     -- weight-gradient GEMM inputs of the same FFN linear, laid
  out with the token axis contiguous (the contraction axis of the Wgrad
  GEMM): dY^T 20480 x M with N(0,1) * 2^-10 entries and 0.1% x50, X^T
  5120 x M (the ffn activation, transposed); plus the random 16-bit sign
  mask of the Hadamard transform applied to both before quantization.

Every draw is keyed by ``seed_for(workload, stream)``; a tensor drawn on a
given device type is the same on every call.  CPU and CUDA generators give
different numbers, so a test feeds the oracle the very tensor the GPU saw.
"""
from __future__ import annotations

import math

import torch

SEED_BASE = 0x4E5646
WORKLOADS = ("tiny", "sweep", "ffn", "moe", "kv", "wgrad")

# The seven nonzero E2M1 magnitudes, used only to plant "exactly
# representable" inputs in the sweep workload (the format's value list is
# given in the NVFP4 pre-training page, section "E2M1 format and two-level
# scaling").
_GRID_NONZERO = (0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)

FFN_N, FFN_K = 20480, 5120
FFN_M = (16, 512, 8192)
MOE_TOKENS, MOE_EXPERTS, MOE_TOPK = 4096, 256, 8
MOE_HIDDEN, MOE_INTER = 6144, 2048
MOE_ROW_ALIGN = 128
KV_LAYERS, KV_HEADS, KV_HEAD_DIM, KV_TOKENS = 32, 8, 128, 131072


def seed_for(workload: str, stream: int = 0) -> int:
    """Seed of one draw: base + workload index (1..5) + 1000 * stream."""
    return SEED_BASE + 1 + WORKLOADS.index(workload) + 1000 * stream


def _gen(workload: str, stream: int, device) -> torch.Generator:
    g = torch.Generator(device=torch.device(device).type)
    g.manual_seed(seed_for(workload, stream))
    return g


def _randn(shape, g, device, std: float = 1.0) -> torch.Tensor:
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x


def _pick(n: int, k: int, g, device, replace: bool) -> torch.Tensor:
    """k indices in [0, n): without replacement when cheap, else uniform."""
    if not replace:
        return torch.randperm(n, generator=g, device=device)[:k]
    return torch.randint(0, n, (k,), generator=g, device=device)


# --------------------------------------------------------------------------
# tiny: W4A4 linear
# --------------------------------------------------------------------------
def tiny_operand(which: str, device="cpu") -> torch.Tensor:
    """A (128x256, stream 0) or W (256x256, stream 1) of the tiny linear."""
    rows = {"A": 128, "W": 256}[which]
    cols = 256
    stream = {"A": 0, "W": 1}[which]
    g = _gen("tiny", stream, device)
    x = _randn((rows, cols), g, device)
    flat = x.view(-1)
    k = round(0.005 * flat.numel())
    idx = _pick(flat.numel(), k, g, device, replace=False)
    flat[idx] *= 30.0
    zero_blk = torch.randint(0, cols // 16, (rows,), generator=g, device=device)
    cols_idx = zero_blk[:, None] * 16 + torch.arange(16, device=device)[None, :]
    x.scatter_(1, cols_idx, 0.0)
    return x.to(torch.bfloat16)


# --------------------------------------------------------------------------
# sweep: standalone quantize
# --------------------------------------------------------------------------
SWEEP_SIZES = (1 << 20, 1 << 24, 1 << 28)
SWEEP_COLS = 4096


def sweep_tensor(n: int, device="cpu", cols: int = SWEEP_COLS) -> torch.Tensor:
    """[n/cols, cols] BF16: N(0,1), 0.1% x50, 1% exact grid values c*2^k."""
    assert n % cols == 0
    g = _gen("sweep", int(round(math.log2(n))), device)
    x = _randn((n,), g, device)
    big = n > (1 << 22)
    k_out = round(0.001 * n)
    idx = _pick(n, k_out, g, device, replace=big)
    x[idx] *= 50.0
    k_grid = round(0.01 * n)
    idx = _pick(n, k_grid, g, device, replace=big)
    grid = torch.tensor(_GRID_NONZERO, device=device)
    c = grid[torch.randint(0, 7, (k_grid,), generator=g, device=device)]
    sign = torch.randint(0, 2, (k_grid,), generator=g, device=device) * 2 - 1
    e = torch.randint(-4, 5, (k_grid,), generator=g, device=device)
    x[idx] = c * sign * torch.exp2(e.to(torch.float32))
    return x.view(n // cols, cols).to(torch.bfloat16)


# --------------------------------------------------------------------------
# ffn: dense W4A4 linear of a 12B hybrid model
# --------------------------------------------------------------------------
def ffn_weight(device="cpu", n: int = FFN_N, k: int = FFN_K) -> torch.Tensor:
    g = _gen("ffn", 0, device)
    return _randn((n, k), g, device, std=0.02).to(torch.bfloat16)


def ffn_outlier_columns(k: int = FFN_K) -> torch.Tensor:
    """The 1% of K columns (51 of 5120) that carry x20 outliers."""
    g = _gen("ffn", 1, "cpu")
    return torch.randperm(k, generator=g)[: round(0.01 * k)]


def ffn_activation(m: int, device="cpu", k: int = FFN_K) -> torch.Tensor:
    g = _gen("ffn", 2 + m, device)
    x = _randn((m, k), g, device)
    cols = ffn_outlier_columns(k).to(device)
    x[:, cols] *= 20.0
    return x.to(torch.bfloat16)


# --------------------------------------------------------------------------
# moe: 256-expert top-8 routing and expert weights
# --------------------------------------------------------------------------
class MoeRouting:
    """Routing of ``tokens`` tokens onto ``experts`` experts, top-``topk``.

    ``rows[e]`` is how many (token, expert) pairs land on expert e.  Pairs
    are laid out expert by expert; each expert's slot is padded up to a
    multiple of ``align`` rows.  ``slot_offsets`` (experts+1 entries) gives
    the padded start of each slot, ``gather`` (one entry per padded row) the
    source token of each row or -1 for a padding row.
    """

    def __init__(self, tokens=MOE_TOKENS, experts=MOE_EXPERTS, topk=MOE_TOPK,
                 align=MOE_ROW_ALIGN):
        g = _gen("moe", 0, "cpu")
        logits = torch.randn((tokens, experts), generator=g)
        probs = torch.softmax(logits.double(), dim=-1)
        # top-k by probability; ties (measure zero for continuous logits)
        # go to the lower expert index because sort is stable.
        order = torch.sort(-probs, dim=-1, stable=True).indices[:, :topk]
        self.topk_ids = order.to(torch.int32)
        self.topk_weights = torch.gather(probs, 1, order).float()
        self.tokens, self.experts, self.topk, self.align = tokens, experts, topk, align
        flat_e = self.topk_ids.reshape(-1).long()
        flat_t = torch.arange(tokens).repeat_interleave(topk)
        key = flat_e * tokens + flat_t          # expert-major, token order
        perm = torch.argsort(key)
        self.rows = torch.bincount(flat_e, minlength=experts).to(torch.int32)
        padded = ((self.rows + align - 1) // align) * align
        self.slot_offsets = torch.zeros(experts + 1, dtype=torch.int32)
        self.slot_offsets[1:] = torch.cumsum(padded, 0).to(torch.int32)
        total = int(self.slot_offsets[-1])
        self.gather = torch.full((total,), -1, dtype=torch.int32)
        src_tokens = flat_t[perm]
        starts = torch.zeros(experts + 1, dtype=torch.int64)
        starts[1:] = torch.cumsum(self.rows.long(), 0)
        for e in range(experts):
            a, b = int(starts[e]), int(starts[e + 1])
            o = int(self.slot_offsets[e])
            self.gather[o:o + (b - a)] = src_tokens[a:b].to(torch.int32)
        self.padded_rows = total
        self.real_rows = int(self.rows.sum())
        # row of (token t, choice k) in the padded expert-major layout
        slot_of_pair = torch.empty(tokens * topk, dtype=torch.int64)
        flat_e_sorted = flat_e[perm]
        pos = torch.arange(tokens * topk) - starts[flat_e_sorted]
        slot_of_pair[perm] = self.slot_offsets.long()[flat_e_sorted] + pos
        self.token_slots = slot_of_pair.view(tokens, topk).to(torch.int32)
        # combine weights: the selected probabilities, renormalized to sum 1
        w = self.topk_weights.double()
        self.combine_weights = (w / w.sum(dim=1, keepdim=True)).float()


def moe_activation(device="cpu", tokens=MOE_TOKENS, hidden=MOE_HIDDEN) -> torch.Tensor:
    g = _gen("moe", 1, device)
    return _randn((tokens, hidden), g, device).to(torch.bfloat16)


def moe_expert_weight(which: str, expert: int, device="cpu",
                      hidden=MOE_HIDDEN, inter=MOE_INTER) -> torch.Tensor:
    """W_up[e] (inter x hidden) or W_down[e] (hidden x inter), N(0, 0.02^2).

    Each expert has its own stream, so one expert can be drawn alone."""
    shape = {"up": (inter, hidden), "down": (hidden, inter)}[which]
    stream = {"up": 2, "down": 2 + MOE_EXPERTS}[which] + expert
    g = _gen("moe", stream, device)
    return _randn(shape, g, device, std=0.02).to(torch.bfloat16)


def moe_expert_weights(which: str, device="cpu", experts=MOE_EXPERTS,
                       hidden=MOE_HIDDEN, inter=MOE_INTER) -> torch.Tensor:
    """All experts stacked: [experts * rows_e, cols_e] BF16."""
    return torch.cat([moe_expert_weight(which, e, device, hidden, inter)
                      for e in range(experts)], 0)


# --------------------------------------------------------------------------
# kv: NVFP4 KV cache
# --------------------------------------------------------------------------
def kv_outlier_channels(layer: int, kv: int) -> torch.Tensor:
    """5 of the 1024 (head, dim) channels of one tensor (0.5%, rounded)."""
    g = _gen("kv", 1 + 2 * layer + kv, "cpu")
    return torch.randperm(KV_HEADS * KV_HEAD_DIM, generator=g)[:5]


def kv_tensor(layer: int, kv: int, device="cpu", tokens: int = KV_TOKENS) -> torch.Tensor:
    """[tokens, heads, head_dim] BF16 for layer ``layer``, K (kv=0) or V (1)."""
    g = _gen("kv", 100 + 2 * layer + kv, device)
    x = _randn((tokens, KV_HEADS * KV_HEAD_DIM), g, device)
    x[:, kv_outlier_channels(layer, kv).to(device)] *= 10.0
    return x.view(tokens, KV_HEADS, KV_HEAD_DIM).to(torch.bfloat16)


KV_QUERY_HEADS = 64        # grouped-query attention: 8 query heads per KV head


def kv_query(layer: int, device="cpu", heads_q: int = KV_QUERY_HEADS) -> torch.Tensor:
    """Query of one decode step for layer ``layer``: BF16 [heads_q x head_dim], N(0,1)."""
    g = _gen("kv", 1000 + layer, device)
    return _randn((heads_q, KV_HEAD_DIM), g, device).to(torch.bfloat16)


# --------------------------------------------------------------------------
# wgrad: inputs of the weight-gradient GEMM dW = dY^T X of the FFN linear
# --------------------------------------------------------------------------
WGRAD_M = 8192


def rht_sign_mask(stream: int = 0) -> int:
    """The random +-1 sign vector of the 16x16 Hadamard transform as a
    16-bit mask (bit j set = value j of a block negated), one per draw."""
    g = _gen("wgrad", 100 + stream, "cpu")
    return int(torch.randint(0, 1 << 16, (1,), generator=g).item())


def wgrad_grad_output_t(m: int = WGRAD_M, device="cpu", n: int = FFN_N) -> torch.Tensor:
    """dY^T [n x m] BF16: N(0,1) * 2^-10, 0.1% of the entries x50."""
    g = _gen("wgrad", 1 + m, device)
    x = _randn((n * m,), g, device) * 2.0 ** -10
    idx = _pick(n * m, round(0.001 * n * m), g, device, replace=n * m > (1 << 22))
    x[idx] *= 50.0
    return x.view(n, m).to(torch.bfloat16)


def wgrad_activation_t(m: int = WGRAD_M, device="cpu", k: int = FFN_K) -> torch.Tensor:
    """X^T [k x m] BF16: the ffn activation of m tokens, transposed."""
    return ffn_activation(m, device, k).t().contiguous()

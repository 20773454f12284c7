"""Seeded synthetic routing inputs for MoE layout / dispatch / combine.

This module only makes inputs: BF16 activations, group-limited top-k routing
(DeepSeek-V3 style gating, as the DeepEP pages name it: "top-4 groups, top-8
experts" in the normal-kernel settings of the DeepEP README mirrors), optional
Zipf expert skew, gradient rows and stand-in expert outputs.  It computes none
of the layout, quantisation or combine arithmetic; both the CUDA path and the
CPU oracle consume what it returns.

Draw order from one ``numpy.random.Generator(PCG64(seed))``:
x (standard normal fp32) -> logits fp32 [N, E] -> hot-row choice -> Zipf
permutation -> grad.  Expert outputs come from a second generator seeded with
``(seed, 1)`` so that drawing them never shifts the routing.

Routing rule (the pages give only "top-4 groups, top-8 experts"; the details
below are this library's reading):
  score   = sigmoid(logit + bias_e)            (bias_e = 0 without skew)
  group   = max score over the group's experts
  keep the top ``topk_group`` groups, then the top ``k`` experts inside them;
  ordering is by descending score, a lower index wins a tie; slots are filled
  in descending score order; weights = selected scores / their sum.
Zipf skew: rank_e = permutation(E) + 1, bias_e = -0.3 * s * ln(rank_e).
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np

ZIPF_BETA = 0.3


@dataclass(frozen=True)
class Workload:
    """Shape and routing recipe of one synthetic MoE layer invocation."""

    name: str
    num_tokens: int          # N
    hidden: int              # H
    num_experts: int         # E
    num_ranks: int           # R, logical expert-parallel ranks (E % R == 0)
    topk: int                # k
    num_groups: int = 1      # G (1 = no group limit)
    topk_group: int = 1      # groups kept per token
    padded: bool = False     # receive buffers padded to the max tokens per expert
    fp8: bool = True         # FP8 e4m3 dispatch (False: BF16 rows)
    hot_row_frac: float = 0.0   # fraction of rows scaled x100 before BF16 rounding
    zipf_s: float = 0.0      # 0 = no skew
    with_grad: bool = False  # also draw combine-backward grad rows [N, H]
    description: str = ""


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny", 128, 256, 16, 4, 4, num_groups=4, topk_group=2,
                 description="128 tok, H=256, 16 experts in 4 groups, top-2 groups / top-4, 4 ranks"),
        Workload("decode", 128, 7168, 256, 32, 8, padded=True,
                 description="128 tok, H=7168, plain top-8 of 256, 32 ranks, padded receive buffers"),
        Workload("prefill", 4096, 7168, 256, 64, 8, num_groups=8, topk_group=4,
                 hot_row_frac=0.01,
                 description="4096 tok, H=7168, 256 experts in 8 groups, top-4 groups / top-8, 64 ranks, 1% rows x100"),
        Workload("skewed", 16384, 7168, 256, 64, 8, num_groups=8, topk_group=4,
                 zipf_s=1.1,
                 description="16384 tok, H=7168, group-limited top-8 with Zipf(1.1) expert skew, 64 ranks"),
        Workload("bf16", 8192, 7168, 256, 64, 8, fp8=False, zipf_s=1.2, with_grad=True,
                 description="8192 tok, H=7168, plain top-8 with Zipf(1.2) skew, BF16 dispatch + combine-backward"),
    ]
}
WORKLOAD_ORDER = ["tiny", "decode", "prefill", "skewed", "bf16"]


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to BF16 (nearest, ties to even); returns the uint16 bit patterns.

    Inputs are finite by construction (normal draws), so no NaN handling is needed.
    """
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen BF16 bit patterns to fp32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _sigmoid32(z: np.ndarray) -> np.ndarray:
    return (1.0 / (1.0 + np.exp(-z.astype(np.float64)))).astype(np.float32)


def route(scores: np.ndarray, k: int, num_groups: int, topk_group: int):
    """Group-limited top-k selection over fp32 scores [N, E].

    Returns (topk_idx int32 [N, k], topk_w fp32 [N, k]).
    """
    n, e = scores.shape
    masked = scores.astype(np.float32, copy=True)
    if num_groups > 1:
        per = e // num_groups
        gscore = masked.reshape(n, num_groups, per).max(axis=2)
        gorder = np.argsort(-gscore, axis=1, kind="stable")
        keep = np.zeros((n, num_groups), dtype=bool)
        np.put_along_axis(keep, gorder[:, :topk_group], True, axis=1)
        masked = np.where(np.repeat(keep, per, axis=1), masked, -np.inf).astype(np.float32)
    order = np.argsort(-masked, axis=1, kind="stable")[:, :k]
    sel = np.take_along_axis(scores.astype(np.float32), order, axis=1).astype(np.float64)
    w = (sel / sel.sum(axis=1, keepdims=True)).astype(np.float32)
    return order.astype(np.int32), w


@dataclass
class Inputs:
    """One drawn workload: host arrays, BF16 kept as uint16 bit patterns."""

    workload: Workload
    seed: int
    x: np.ndarray               # uint16 [N, H]
    topk_idx: np.ndarray        # int32 [N, k]
    topk_w: np.ndarray          # fp32 [N, k]
    scores: np.ndarray          # fp32 [N, E] (biased sigmoid scores used for routing)
    hot_rows: np.ndarray        # int64 indices of rows scaled x100
    zipf_rank: Optional[np.ndarray] = None
    grad: Optional[np.ndarray] = None   # uint16 [N, H]
    extra: dict = field(default_factory=dict)


def make_inputs(name_or_wl, seed: int = 0, num_tokens: Optional[int] = None) -> Inputs:
    """Draw the inputs of a named workload (optionally with a different token count)."""
    wl = WORKLOADS[name_or_wl] if isinstance(name_or_wl, str) else name_or_wl
    n = wl.num_tokens if num_tokens is None else int(num_tokens)
    h, e = wl.hidden, wl.num_experts
    g = np.random.Generator(np.random.PCG64(seed))
    x32 = g.standard_normal((n, h), dtype=np.float32)
    logits = g.standard_normal((n, e), dtype=np.float32)
    hot = np.zeros(0, dtype=np.int64)
    if wl.hot_row_frac > 0 and n > 0:
        nhot = int(np.ceil(wl.hot_row_frac * n))
        hot = np.sort(g.choice(n, size=nhot, replace=False))
        x32[hot] *= np.float32(100.0)
    zrank = None
    if wl.zipf_s > 0:
        zrank = g.permutation(e) + 1
        bias = (-ZIPF_BETA * wl.zipf_s * np.log(zrank.astype(np.float64))).astype(np.float32)
        logits = (logits + bias[None, :]).astype(np.float32)
    grad = None
    if wl.with_grad:
        grad = f32_to_bf16_bits(g.standard_normal((n, h), dtype=np.float32))
    scores = _sigmoid32(logits)
    idx, w = route(scores, wl.topk, wl.num_groups, wl.topk_group)
    return Inputs(wl, seed, f32_to_bf16_bits(x32), idx, w, scores, hot, zrank, grad)


def expert_outputs(num_rows: int, hidden: int, seed: int = 0, chunk_rows: int = 4096) -> np.ndarray:
    """Stand-in expert outputs y ~ N(0, 1) as BF16 bits [num_rows, hidden].

    Drawn in row chunks so that large receive buffers do not need an fp32 copy.
    """
    g = np.random.Generator(np.random.PCG64([seed, 1]))
    out = np.empty((num_rows, hidden), dtype=np.uint16)
    for r0 in range(0, num_rows, chunk_rows):
        r1 = min(num_rows, r0 + chunk_rows)
        out[r0:r1] = f32_to_bf16_bits(g.standard_normal((r1 - r0, hidden), dtype=np.float32))
    return out


def algorithmic_bytes(wl: Workload, num_tokens: Optional[int] = None) -> dict:
    """Bytes each kernel must move at minimum (reads + writes), per launch.

    dispatch FP8  = 2NH (x) + 4Nk (dst_pos) + NkH (e4m3 rows) + 4Nk*H/128 (fp32 scales)
    dispatch BF16 = 2NH + 4Nk + 2NkH
    combine       = 2NkH (expert outputs) + 8Nk (dst_pos + weights) + 2NH (out)
    layout        = 4Nk (ids) + 8Nk (dst_pos + recv_src) + N*R (is_token_in_rank)
    """
    n = wl.num_tokens if num_tokens is None else num_tokens
    h, k, r = wl.hidden, wl.topk, wl.num_ranks
    return {
        "layout": 4 * n * k + 8 * n * k + n * r,
        "dispatch_fp8": 2 * n * h + 4 * n * k + n * k * h + 4 * n * k * (h // 128),
        "dispatch_bf16": 2 * n * h + 4 * n * k + 2 * n * k * h,
        "combine": 2 * n * k * h + 8 * n * k + 2 * n * h,
    }

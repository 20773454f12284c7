"""Pure-Python brute force for tiny layouts (test infrastructure only).

A second, deliberately different statement of the stable layout: for every
expert, list the (token, slot) pairs routed to it, sort them, and number them.
Quadratic and slow; use on inputs of a few hundred pairs.  It shares nothing
with oracle.c and is used to pin it.
"""

from __future__ import annotations


def layout(topk_idx, num_experts: int, num_ranks: int, capacity: int = 0):
    """Returns a dict with the same fields as the oracle's layout (Python lists)."""
    n = len(topk_idx)
    k = len(topk_idx[0]) if n else 0
    E, R = num_experts, num_ranks
    per = E // R
    pairs = {e: sorted((t, j) for t in range(n) for j in range(k) if topk_idx[t][j] == e)
             for e in range(E)}
    counts = [len(pairs[e]) for e in range(E)]
    offset = [sum(counts[:e]) for e in range(E + 1)]
    rows = E * capacity if capacity > 0 else n * k
    dst = [[-1] * k for _ in range(n)]
    src = [-1] * rows
    overflow = False
    for e in range(E):
        for slot, (t, j) in enumerate(pairs[e]):
            if capacity > 0:
                if slot >= capacity:
                    overflow = True
                    continue
                row = e * capacity + slot
            else:
                row = offset[e] + slot
            dst[t][j] = row
            src[row] = t * k + j
    in_rank = [[int(any(0 <= topk_idx[t][j] < E and topk_idx[t][j] // per == r for j in range(k)))
                for r in range(R)] for t in range(n)]
    bad = any(not (-1 <= topk_idx[t][j] < E) for t in range(n) for j in range(k))
    return {
        "tokens_per_expert": counts,
        "tokens_per_rank": [sum(in_rank[t][r] for t in range(n)) for r in range(R)],
        "is_token_in_rank": in_rank,
        "expert_offset": offset,
        "max_count": max(counts) if counts else 0,
        "dst_pos": dst,
        "recv_src": src,
        "range_error": bad,
        "capacity_error": overflow,
    }


def rank_layout(topk_idx, num_experts: int, num_ranks: int, capacity: int = 0):
    """Per-rank layout, brute force: for each rank, the sorted list of tokens that
    reach it; a token's copy for rank r is attributed to its first slot on r."""
    n = len(topk_idx)
    k = len(topk_idx[0]) if n else 0
    E, R = num_experts, num_ranks
    per = E // R

    def rank_of(e):
        return e // per if 0 <= e < E else None

    tokens = {r: sorted({t for t in range(n) for j in range(k) if rank_of(topk_idx[t][j]) == r})
              for r in range(R)}
    counts = [len(tokens[r]) for r in range(R)]
    offset = [sum(counts[:r]) for r in range(R + 1)]
    rows = R * capacity if capacity > 0 else n * k
    dst = [[-1] * k for _ in range(n)]
    src = [-1] * rows
    overflow = False
    for r in range(R):
        for slot, t in enumerate(tokens[r]):
            j = min(j for j in range(k) if rank_of(topk_idx[t][j]) == r)
            if capacity > 0:
                if slot >= capacity:
                    overflow = True
                    continue
                row = r * capacity + slot
            else:
                row = offset[r] + slot
            dst[t][j] = row
            src[row] = t
    return {"tokens_per_rank": counts, "rank_offset": offset, "max_count": max(counts) if counts else 0,
            "rank_dst": dst, "recv_token": src, "capacity_error": overflow}

"""Pins for the oracle's layout: brute force on tiny inputs, invariants on every workload."""

import numpy as np
import pytest

from combine_get_layout_02_b200 import workloads as W
from oracle import brute


def _random_idx(rng, n, k, E, p_mask=0.1, p_bad=0.0, distinct=True):
    if distinct and k <= E:
        idx = np.stack([rng.permutation(E)[:k] for _ in range(n)]).astype(np.int32) if n else np.zeros((0, k), np.int32)
    else:
        idx = rng.integers(0, E, (n, k)).astype(np.int32)
    idx[rng.random((n, k)) < p_mask] = -1
    if p_bad:
        bad = rng.random((n, k)) < p_bad
        idx[bad] = rng.choice([-7, -2, E, E + 5], bad.sum())
    return idx


def _compare_to_brute(oracle_mod, idx, E, R, cap):
    L = oracle_mod.get_layout(idx, E, R, cap)
    B = brute.layout(idx.tolist(), E, R, cap)
    assert L.tokens_per_expert.tolist() == B["tokens_per_expert"]
    assert L.tokens_per_rank.tolist() == B["tokens_per_rank"]
    assert L.is_token_in_rank.tolist() == B["is_token_in_rank"]
    assert L.expert_offset.tolist() == B["expert_offset"]
    assert L.max_count == B["max_count"]
    assert L.dst_pos.tolist() == B["dst_pos"]
    assert L.recv_src.tolist() == B["recv_src"]
    assert bool(L.flags & oracle_mod.FLAG_RANGE) == B["range_error"]
    assert bool(L.flags & oracle_mod.FLAG_CAPACITY) == B["capacity_error"]


@pytest.mark.parametrize("seed", range(12))
def test_brute_force_compact(oracle_mod, seed):
    rng = np.random.default_rng(seed)
    E = int(rng.choice([4, 6, 8, 12]))
    R = int(rng.choice([r for r in (1, 2, 3, 4, 6) if E % r == 0]))
    k = int(rng.integers(1, min(E, 6) + 1))
    n = int(rng.integers(0, 40))
    _compare_to_brute(oracle_mod, _random_idx(rng, n, k, E), E, R, 0)


@pytest.mark.parametrize("seed", range(8))
def test_brute_force_padded_with_overflow(oracle_mod, seed):
    rng = np.random.default_rng(100 + seed)
    E, R, k, n = 8, 4, 3, 30
    idx = _random_idx(rng, n, k, E)
    cap = int(rng.integers(1, 14))
    _compare_to_brute(oracle_mod, idx, E, R, cap)


@pytest.mark.parametrize("seed", range(6))
def test_brute_force_duplicates_and_bad_ids(oracle_mod, seed):
    rng = np.random.default_rng(200 + seed)
    E, R, k, n = 6, 3, 4, 25
    idx = _random_idx(rng, n, k, E, p_mask=0.15, p_bad=0.1, distinct=False)
    _compare_to_brute(oracle_mod, idx, E, R, 0)
    _compare_to_brute(oracle_mod, idx, E, R, 5)


def check_invariants(L, idx, E, R, cap):
    n, k = idx.shape
    valid = (idx >= 0) & (idx < E)
    m = int(valid.sum())
    assert L.tokens_per_expert.sum() == m
    assert np.array_equal(L.tokens_per_expert, np.bincount(idx[valid], minlength=E))
    assert L.expert_offset[0] == 0 and L.expert_offset[-1] == m
    assert np.all(np.diff(L.expert_offset) == L.tokens_per_expert)
    assert L.max_count == L.tokens_per_expert.max(initial=0)
    used = L.dst_pos[L.dst_pos >= 0]
    assert len(np.unique(used)) == used.size                       # injective
    if cap == 0:
        assert np.array_equal(np.sort(used), np.arange(m))          # bijection onto [0, M)
    else:
        e_of = idx[L.dst_pos >= 0]
        assert np.all(used // cap == e_of)                           # row inside its expert's block
    tk = np.nonzero(L.dst_pos >= 0)
    assert np.all(L.recv_src[L.dst_pos[tk]] == tk[0] * k + tk[1])   # inverse map
    assert (L.recv_src >= 0).sum() == used.size
    for e in range(E):                                              # ascending token order per expert
        rows = np.sort(used[(idx[L.dst_pos >= 0] == e)])
        src = L.recv_src[rows]
        assert np.all(np.diff(src) > 0)
    per = E // R
    ranks = np.where(valid, idx // per, -1)
    itr = np.zeros((n, R), np.uint8)
    for r in range(R):
        itr[:, r] = (ranks == r).any(axis=1)
    assert np.array_equal(L.is_token_in_rank, itr)
    assert np.array_equal(L.tokens_per_rank, itr.sum(axis=0))
    n_routed = int(valid.any(axis=1).sum())
    assert n_routed <= L.tokens_per_rank.sum() <= n_routed * min(k, R)


@pytest.mark.parametrize("name", W.WORKLOAD_ORDER)
def test_invariants_on_workloads(oracle_mod, name):
    inp = W.make_inputs(name, 0)
    wl = inp.workload
    L = oracle_mod.get_layout(inp.topk_idx, wl.num_experts, wl.num_ranks, 0)
    check_invariants(L, inp.topk_idx, wl.num_experts, wl.num_ranks, 0)
    assert L.flags == 0
    if wl.padded:
        cap = L.max_count
        P = oracle_mod.get_layout(inp.topk_idx, wl.num_experts, wl.num_ranks, cap)
        check_invariants(P, inp.topk_idx, wl.num_experts, wl.num_ranks, cap)
        assert P.flags == 0
        # padded and compact layouts agree on each copy's slot inside its expert
        e = inp.topk_idx
        assert np.array_equal(P.dst_pos - e * cap, L.dst_pos - L.expert_offset[e])


def test_masked_tokens_and_empty(oracle_mod):
    idx = np.full((5, 4), -1, np.int32)
    L = oracle_mod.get_layout(idx, 8, 2)
    assert L.tokens_per_expert.sum() == 0 and np.all(L.dst_pos == -1) and np.all(L.recv_src == -1)
    assert L.tokens_per_rank.sum() == 0 and L.max_count == 0 and L.flags == 0
    L0 = oracle_mod.get_layout(np.zeros((0, 8), np.int32), 256, 64)
    assert L0.expert_offset.sum() == 0 and L0.recv_src.size == 0


def test_capacity_overflow_drops_late_tokens(oracle_mod):
    # all 6 tokens route to expert 1; capacity 4 keeps tokens 0..3 in order
    idx = np.array([[1, 0]] * 6, np.int32)
    L = oracle_mod.get_layout(idx, 4, 2, capacity=4)
    assert L.flags & oracle_mod.FLAG_CAPACITY
    assert L.dst_pos[:, 0].tolist() == [4, 5, 6, 7, -1, -1]
    assert L.dst_pos[:, 1].tolist() == [0, 1, 2, 3, -1, -1]
    assert L.tokens_per_expert.tolist() == [6, 6, 0, 0] and L.max_count == 6


def _compare_rank_to_brute(oracle_mod, idx, E, R, cap):
    L = oracle_mod.get_rank_layout(idx, E, R, cap)
    B = brute.rank_layout(idx.tolist(), E, R, cap)
    assert L.tokens_per_rank.tolist() == B["tokens_per_rank"]
    assert L.rank_offset.tolist() == B["rank_offset"]
    assert L.max_count == B["max_count"]
    assert L.rank_dst.tolist() == B["rank_dst"]
    assert L.recv_token.tolist() == B["recv_token"]
    assert bool(L.flags & oracle_mod.FLAG_CAPACITY) == B["capacity_error"]


@pytest.mark.parametrize("seed", range(10))
def test_rank_layout_brute_force(oracle_mod, seed):
    rng = np.random.default_rng(300 + seed)
    E = int(rng.choice([4, 8, 12, 16]))
    R = int(rng.choice([r for r in (1, 2, 4) if E % r == 0]))
    k = int(rng.integers(1, 6))
    n = int(rng.integers(0, 40))
    idx = _random_idx(rng, n, k, E, distinct=bool(seed % 2), p_bad=0.05 if seed % 3 == 0 else 0.0)
    _compare_rank_to_brute(oracle_mod, idx, E, R, 0)
    _compare_rank_to_brute(oracle_mod, idx, E, R, int(rng.integers(1, 12)))


@pytest.mark.parametrize("name", W.WORKLOAD_ORDER)
def test_rank_layout_invariants(oracle_mod, name):
    inp = W.make_inputs(name, 0)
    wl = inp.workload
    E, R = wl.num_experts, wl.num_ranks
    L = oracle_mod.get_layout(inp.topk_idx, E, R)
    RL = oracle_mod.get_rank_layout(inp.topk_idx, E, R)
    # same distinct-token counts as the expert layout's rank sets
    assert np.array_equal(RL.tokens_per_rank, L.tokens_per_rank)
    rows = int(RL.tokens_per_rank.sum())
    used = RL.rank_dst[RL.rank_dst >= 0]
    assert np.array_equal(np.sort(used), np.arange(rows))                 # bijection onto [0, rows)
    tk = np.nonzero(RL.rank_dst >= 0)
    assert np.all(RL.recv_token[RL.rank_dst[tk]] == tk[0])
    per = E // R
    ranks = inp.topk_idx // per
    for t in range(0, wl.num_tokens, max(1, wl.num_tokens // 200)):   # one copy per distinct rank
        kept = RL.rank_dst[t] >= 0
        assert sorted(ranks[t][kept].tolist()) == sorted(set(ranks[t].tolist()))
    for r in range(R):                                                     # ascending tokens per rank
        seg = RL.recv_token[RL.rank_offset[r]:RL.rank_offset[r + 1]]
        assert np.all(np.diff(seg) > 0) and np.all((ranks[seg] == r).any(axis=1))
    assert np.all(RL.recv_token[rows:] == -1)


# Property-based pin: hypothesis draws tiny shapes and id tables (duplicates,
# masked and out-of-range ids, compact or padded with any capacity) and the
# oracle must equal the brute force exactly, for expert and for rank keys.
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st


@st.composite
def _tables(draw):
    E = draw(st.sampled_from([1, 2, 4, 6, 8, 12]))
    R = draw(st.sampled_from([r for r in (1, 2, 3, 4, 6, 12) if r <= E and E % r == 0]))
    k = draw(st.integers(1, 5))
    n = draw(st.integers(0, 24))
    ids = draw(st.lists(st.lists(st.integers(-3, E + 2), min_size=k, max_size=k), min_size=n, max_size=n))
    cap = draw(st.integers(0, 6))
    idx = np.array(ids, dtype=np.int32).reshape(n, k)
    return idx, E, R, cap


@settings(max_examples=150, deadline=None, suppress_health_check=[HealthCheck.function_scoped_fixture])
@given(_tables())
def test_layout_equals_brute_force_property(oracle_mod, table):
    idx, E, R, cap = table
    _compare_to_brute(oracle_mod, idx, E, R, cap)


@settings(max_examples=150, deadline=None, suppress_health_check=[HealthCheck.function_scoped_fixture])
@given(_tables())
def test_rank_layout_equals_brute_force_property(oracle_mod, table):
    idx, E, R, cap = table
    L = oracle_mod.get_rank_layout(idx, E, R, cap)
    B = brute.rank_layout(idx.tolist(), E, R, cap)
    assert L.tokens_per_rank.tolist() == B["tokens_per_rank"]
    assert L.rank_offset.tolist() == B["rank_offset"]
    assert L.max_count == B["max_count"]
    assert L.rank_dst.tolist() == B["rank_dst"]
    assert L.recv_token.tolist() == B["recv_token"]
    assert bool(L.flags & oracle_mod.FLAG_CAPACITY) == B["capacity_error"]

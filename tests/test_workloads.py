"""Pins for the seeded routing-input generator (group-limited top-k, Zipf skew)."""

import numpy as np
import pytest

from combine_get_layout_02_b200 import workloads as W


def _brute_route(scores, k, G, topk_group):
    """Per token, in plain Python: rank groups by (max score desc, index asc),
    keep the first topk_group, then rank their experts the same way."""
    n, E = scores.shape
    per = E // G
    idx = []
    for t in range(n):
        s = [float(v) for v in scores[t]]
        groups = sorted(range(G), key=lambda g: (-max(s[g * per:(g + 1) * per]), g))[:topk_group]
        cand = [e for g in groups for e in range(g * per, (g + 1) * per)]
        idx.append(sorted(cand, key=lambda e: (-s[e], e))[:k])
    return np.array(idx, np.int32)


@pytest.mark.parametrize("name", W.WORKLOAD_ORDER)
def test_routing_matches_brute_force_on_a_slice(name):
    inp = W.make_inputs(name, 0, num_tokens=64)
    wl = inp.workload
    ref = _brute_route(inp.scores, wl.topk, wl.num_groups, wl.topk_group)
    assert np.array_equal(inp.topk_idx, ref)


def test_routing_brute_force_with_ties():
    rng = np.random.default_rng(1)
    scores = rng.choice(np.array([0.1, 0.5, 0.5, 0.9], np.float32), (50, 16)).astype(np.float32)
    idx, w = W.route(scores, 4, 4, 2)
    assert np.array_equal(idx, _brute_route(scores, 4, 4, 2))


@pytest.mark.parametrize("name", W.WORKLOAD_ORDER)
def test_routing_invariants(name):
    inp = W.make_inputs(name, 0)
    wl = inp.workload
    n, k = inp.topk_idx.shape
    assert (n, k) == (wl.num_tokens, wl.topk)
    assert inp.x.shape == (wl.num_tokens, wl.hidden) and inp.x.dtype == np.uint16
    srt = np.sort(inp.topk_idx, axis=1)
    assert np.all(np.diff(srt, axis=1) > 0)                       # k distinct experts
    assert inp.topk_idx.min() >= 0 and inp.topk_idx.max() < wl.num_experts
    if wl.num_groups > 1:
        per = wl.num_experts // wl.num_groups
        assert np.all(np.array([len(set(r)) for r in (inp.topk_idx // per)]) <= wl.topk_group)
    sel = np.take_along_axis(inp.scores, inp.topk_idx, axis=1)
    assert np.all(np.diff(sel, axis=1) <= 0)                      # slots in descending score
    ws = inp.topk_w.astype(np.float32).sum(axis=1, dtype=np.float32)
    assert np.all(np.abs(ws - 1) <= 4 * np.finfo(np.float32).eps)  # sum to 1 within 4 ulp
    ratio = inp.topk_w / sel
    assert np.allclose(ratio, ratio[:, :1], rtol=1e-6)             # weights proportional to scores


@pytest.mark.parametrize("name,lo,hi", [("skewed", 8, 13), ("bf16", 8, 13)])
def test_zipf_skew_hottest_about_ten_times_mean(name, lo, hi):
    inp = W.make_inputs(name, 0)
    cnt = np.bincount(inp.topk_idx.ravel(), minlength=inp.workload.num_experts)
    assert lo <= cnt.max() / cnt.mean() <= hi
    # popularity decreases with Zipf rank on average
    order = np.argsort(inp.zipf_rank)
    assert cnt[order[:16]].mean() > 3 * cnt[order[-16:]].mean()


def test_prefill_hot_rows():
    inp = W.make_inputs("prefill", 0)
    assert len(inp.hot_rows) == 41 == int(np.ceil(0.01 * 4096))
    amax = np.abs(W.bf16_bits_to_f32(inp.x)).max(axis=1)
    cold = np.setdiff1d(np.arange(4096), inp.hot_rows)
    assert amax[inp.hot_rows].min() > 100 and amax[cold].max() < 10


def test_seeded_and_reproducible():
    a = W.make_inputs("tiny", 5)
    b = W.make_inputs("tiny", 5)
    c = W.make_inputs("tiny", 6)
    assert np.array_equal(a.x, b.x) and np.array_equal(a.topk_idx, b.topk_idx)
    assert not np.array_equal(a.x, c.x)
    y1 = W.expert_outputs(100, 256, 0, chunk_rows=7)
    y2 = W.expert_outputs(100, 256, 0)
    assert y1.shape == (100, 256) and np.array_equal(y1, y2)   # chunking does not change the draws
    v = W.bf16_bits_to_f32(W.expert_outputs(4096, 256, 0))
    assert abs(v.mean()) < 0.01 and abs(v.std() - 1) < 0.01


def test_bf16_helpers_match_torch():
    import torch

    v = np.random.default_rng(0).standard_normal(100_000).astype(np.float32) * 50
    ref = torch.from_numpy(v).to(torch.bfloat16)
    assert np.array_equal(W.f32_to_bf16_bits(v), ref.view(torch.int16).numpy().view(np.uint16))
    assert np.array_equal(W.bf16_bits_to_f32(W.f32_to_bf16_bits(v)), ref.float().numpy())


def test_algorithmic_bytes_target_config():
    b = W.algorithmic_bytes(W.WORKLOADS["prefill"])
    assert b["dispatch_fp8"] == 301_072_384
    assert b["combine"] == 528_744_448

"""GPU layout (cgl_get_layout) against the oracle, bit for bit, through the C ABI."""

import numpy as np
import pytest
import torch

import combine_get_layout_02_b200 as cgl
from combine_get_layout_02_b200 import workloads as W

from helpers import dev, i32

pytestmark = pytest.mark.gpu


def run_both(oracle_mod, idx, E, R, cap=0):
    st = cgl.new_status(dev())
    lay = cgl.get_layout(i32(idx), E, R, cap, status=st)
    torch.cuda.synchronize()
    ref = oracle_mod.get_layout(idx, E, R, cap)
    got = {f: getattr(lay, f).cpu().numpy() for f in
           ("tokens_per_expert", "tokens_per_rank", "is_token_in_rank", "expert_offset", "dst_pos", "recv_src")}
    for f, g in got.items():
        r = getattr(ref, f)
        assert g.shape == r.shape, f
        assert np.array_equal(g, r), f"{f} differs at {np.argwhere(g != r)[:5].tolist()}"
    assert int(lay.max_count.item()) == ref.max_count
    bits = int(st.item())
    assert bool(bits & (1 << cgl.ERANGE)) == bool(ref.flags & oracle_mod.FLAG_RANGE)
    assert bool(bits & (1 << cgl.ECAPACITY)) == bool(ref.flags & oracle_mod.FLAG_CAPACITY)
    return lay, ref


@pytest.mark.parametrize("name", W.WORKLOAD_ORDER)
def test_layout_full_size_workloads(oracle_mod, name):
    inp = W.make_inputs(name, 0)
    wl = inp.workload
    lay, ref = run_both(oracle_mod, inp.topk_idx, wl.num_experts, wl.num_ranks, 0)
    if wl.padded:
        run_both(oracle_mod, inp.topk_idx, wl.num_experts, wl.num_ranks, int(lay.max_count.item()))


@pytest.mark.parametrize("seed", range(10))
def test_layout_random_ragged(oracle_mod, seed):
    rng = np.random.default_rng(seed)
    E = int(rng.choice([8, 16, 64, 256, 1024]))
    R = int(rng.choice([r for r in (1, 2, 4, 8, 32, 64, E) if E % r == 0]))
    k = int(rng.choice([1, 2, 3, 4, 6, 8, 13, 32]))
    n = int(rng.choice([1, 7, 255, 256, 257, 1000, 3333]))
    if k <= E:
        idx = np.argsort(rng.random((n, E)), axis=1)[:, :k].astype(np.int32)
    else:
        idx = rng.integers(0, E, (n, k)).astype(np.int32)
    idx[rng.random((n, k)) < 0.05] = -1
    run_both(oracle_mod, idx, E, R, 0)


@pytest.mark.parametrize("n,k", [(4096, 8), (4097, 8), (8192, 8), (8193, 8), (5462, 6), (43, 6)])
def test_layout_block_size_boundaries(oracle_mod, n, k):
    """Token counts on both sides of a change of block size (32 -> 64 -> 128
    tokens per block at k = 8 once the grid would pass 128 blocks), padded too."""
    rng = np.random.default_rng(n * 31 + k)
    E, R = 256, 64
    idx = np.argsort(rng.random((n, E)), axis=1)[:, :k].astype(np.int32)
    idx[rng.random((n, k)) < 0.03] = -1
    lay, _ = run_both(oracle_mod, idx, E, R, 0)
    run_both(oracle_mod, idx, E, R, max(1, int(lay.max_count.item()) - 3))   # a few copies over capacity


@pytest.mark.parametrize("n,k,E,R", [(33, 8, 256, 64), (64, 8, 256, 32), (100, 8, 256, 64), (200, 8, 256, 64),
                                     (256, 8, 256, 64), (170, 3, 64, 8), (96, 6, 96, 12), (130, 4, 16, 4)])
def test_layout_cluster_sizes(oracle_mod, n, k, E, R):
    """Batches of 2 to 8 one-chunk blocks (the thread-block-cluster path): duplicates
    inside tokens, masked and bad ids, compact and padded with overflow."""
    rng = np.random.default_rng(n * 7 + k)
    idx = rng.integers(0, E, (n, k)).astype(np.int32)
    idx[rng.random((n, k)) < 0.05] = -1
    idx[rng.random((n, k)) < 0.01] = E
    lay, _ = run_both(oracle_mod, idx, E, R, 0)
    mc = int(lay.max_count.item())
    run_both(oracle_mod, idx, E, R, max(1, mc - 2))
    run_both(oracle_mod, idx, E, R, mc + 1)


def test_layout_duplicates_bad_ids_and_overflow(oracle_mod):
    rng = np.random.default_rng(42)
    n, k, E, R = 700, 8, 16, 4
    idx = rng.integers(0, E, (n, k)).astype(np.int32)          # duplicates within tokens
    bad = rng.random((n, k)) < 0.02
    idx[bad] = rng.choice([-5, -2, E, E + 100], bad.sum())
    idx[rng.random((n, k)) < 0.05] = -1
    run_both(oracle_mod, idx, E, R, 0)
    run_both(oracle_mod, idx, E, R, 300)      # padded, no overflow
    run_both(oracle_mod, idx, E, R, 200)      # padded, some experts overflow


def test_layout_skewed_hot_expert(oracle_mod):
    # one expert takes every token: the worst case for same-expert contention
    n, k, E, R = 5000, 4, 64, 8
    rng = np.random.default_rng(1)
    idx = np.stack([np.concatenate([[3], rng.permutation(np.delete(np.arange(E), 3))[:k - 1]])
                    for _ in range(n)]).astype(np.int32)
    run_both(oracle_mod, idx, E, R, 0)


def test_layout_empty_and_all_masked(oracle_mod):
    run_both(oracle_mod, np.zeros((0, 8), np.int32), 256, 64, 0)
    run_both(oracle_mod, np.zeros((0, 8), np.int32), 256, 64, 4)
    run_both(oracle_mod, np.full((300, 8), -1, np.int32), 256, 64, 0)


def test_layout_max_sizes(oracle_mod):
    rng = np.random.default_rng(9)
    n, k, E = 2048, 32, 1024
    idx = np.argsort(rng.random((n, E)), axis=1)[:, :k].astype(np.int32)
    run_both(oracle_mod, idx, E, 1024, 0)
    run_both(oracle_mod, idx, E, 1, 0)


def test_layout_repeated_calls_reuse_workspace(oracle_mod):
    inp = W.make_inputs("prefill", 3)
    wl = inp.workload
    ws = torch.full((cgl.layout_workspace_bytes(4096, 8, 256, 64),), 0x5A, dtype=torch.uint8, device=dev())
    idx = i32(inp.topk_idx)
    a = cgl.get_layout(idx, 256, 64, workspace=ws)
    b = cgl.get_layout(idx, 256, 64, workspace=ws)
    assert torch.equal(a.dst_pos, b.dst_pos)
    ref = oracle_mod.get_layout(inp.topk_idx, 256, 64)
    assert np.array_equal(b.dst_pos.cpu().numpy(), ref.dst_pos)


def test_layout_two_kernel_path_many_blocks(oracle_mod):
    # more than 256 blocks of 256 tokens: the layout runs as two kernels
    rng = np.random.default_rng(11)
    n, k, E, R = 70000, 2, 64, 16
    idx = np.argsort(rng.random((n, E)), axis=1)[:, :k].astype(np.int32)
    idx[rng.random((n, k)) < 0.03] = -1
    run_both(oracle_mod, idx, E, R, 0)
    run_both(oracle_mod, idx, E, R, 2400)


def test_layout_two_kernel_path_large_shared_memory_with_duplicates(oracle_mod):
    # E = 1024, k = 32 needs more than 48 KiB of shared memory per block: two kernels;
    # repeated experts inside tokens take the in-order walk
    rng = np.random.default_rng(12)
    n, k, E, R = 900, 32, 1024, 128
    idx = rng.integers(0, E, (n, k)).astype(np.int32)
    idx[:, 5] = idx[:, 3]                      # every token repeats one expert
    run_both(oracle_mod, idx, E, R, 0)
    run_both(oracle_mod, idx, E, R, 64)


@pytest.mark.parametrize("name", ["prefill", "skewed"])
def test_layout_graph_replays_with_changing_ids(oracle_mod, name):
    # one captured launch, replayed with different ids: every replay must see its
    # own blocks' counts (the inter-block exchange is tagged per launch on the device)
    wl = W.WORKLOADS[name]
    E, R = wl.num_experts, wl.num_ranks
    ids = [W.make_inputs(name, seed).topk_idx for seed in (1, 2, 3)]
    idx = i32(ids[0])
    ws = torch.empty(cgl.layout_workspace_bytes(wl.num_tokens, wl.topk, E, R), dtype=torch.uint8, device=dev())
    lay = cgl.get_layout(idx, E, R, workspace=ws)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        cgl.get_layout(idx, E, R, workspace=ws, out=lay)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        cgl.get_layout(idx, E, R, workspace=ws, out=lay)
    for a in (ids[1], ids[2], ids[0], ids[1]):
        idx.copy_(torch.from_numpy(a))
        g.replay()
        torch.cuda.synchronize()
        ref = oracle_mod.get_layout(a, E, R)
        assert np.array_equal(lay.dst_pos.cpu().numpy(), ref.dst_pos)
        assert np.array_equal(lay.expert_offset.cpu().numpy(), ref.expert_offset)
        assert np.array_equal(lay.recv_src.cpu().numpy(), ref.recv_src)
        assert np.array_equal(lay.tokens_per_rank.cpu().numpy(), ref.tokens_per_rank)
    del g


def test_layout_replicated_counts_with_unaligned_ids(oracle_mod):
    """Ids that start 4 bytes past a 16-byte boundary: the replicated-count
    layout reads them one by one instead of as int4."""
    rng = np.random.default_rng(21)
    n, k, E, R = 3000, 8, 256, 64
    a = np.argsort(rng.random((n, E)), axis=1)[:, :k].astype(np.int32)
    a[rng.random((n, k)) < 0.04] = -1
    buf = torch.empty(n * k + 1, dtype=torch.int32, device=dev())
    idx = buf[1:].view(n, k)
    assert idx.data_ptr() % 16 == 4
    idx.copy_(torch.from_numpy(a))
    st = cgl.new_status(dev())
    lay = cgl.get_layout(idx, E, R, status=st)
    torch.cuda.synchronize()
    ref = oracle_mod.get_layout(a, E, R)
    for f in ("tokens_per_expert", "tokens_per_rank", "is_token_in_rank", "expert_offset", "dst_pos", "recv_src"):
        assert np.array_equal(getattr(lay, f).cpu().numpy(), getattr(ref, f)), f
    assert st.item() == 0


@pytest.mark.parametrize("n,k,E,R", [(200, 8, 256, 256), (250, 4, 512, 256)])
def test_layout_cluster_path_many_ranks(oracle_mod, n, k, E, R):
    """More tokens than SMs, and more ranks than 32 per block of the
    replicated-count layout: these small batches take the thread-block-cluster
    layout instead."""
    rng = np.random.default_rng(n + R)
    idx = rng.integers(0, E, (n, k)).astype(np.int32)
    idx[rng.random((n, k)) < 0.05] = -1
    lay, _ = run_both(oracle_mod, idx, E, R, 0)
    run_both(oracle_mod, idx, E, R, max(1, int(lay.max_count.item()) - 1))


@pytest.mark.parametrize("n,k,E,R,cap", [(4000, 8, 256, 64, 0), (4096, 8, 1024, 1024, 0), (1000, 32, 256, 64, 0),
                                         (3001, 6, 96, 8, 0), (4096, 8, 256, 64, -1), (2049, 4, 64, 64, 0)])
def test_layout_replicated_counts_wide_blocks(oracle_mod, n, k, E, R, cap):
    """Batches of 4097 to 32768 (token, slot) pairs take the replicated-count
    layout with 1024-thread blocks: ragged last blocks, many designated ranks
    per block, top-32, a top-k that is not a multiple of 4 (scalar id loads)
    and padded receive rows, at and below the largest per-expert count."""
    rng = np.random.default_rng(n * 7 + k)
    if k <= E:
        idx = np.argsort(rng.random((n, E)), axis=1)[:, :k].astype(np.int32)
    else:
        idx = rng.integers(0, E, (n, k)).astype(np.int32)
    idx[rng.random((n, k)) < 0.03] = -1
    assert 4096 < n * k <= 32768
    lay, ref = run_both(oracle_mod, idx, E, R, 0)
    if cap < 0:
        run_both(oracle_mod, idx, E, R, int(lay.max_count.item()))
        run_both(oracle_mod, idx, E, R, max(1, int(lay.max_count.item()) - 2))

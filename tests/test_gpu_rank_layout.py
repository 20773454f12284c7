"""Per-rank (deduplicated) layout on the GPU against the oracle, bit for bit, and the
dedup dispatch / combine built on it (the copy kernels with rank_dst as dst_pos)."""

import numpy as np
import pytest
import torch

import combine_get_layout_02_b200 as cgl
from combine_get_layout_02_b200 import workloads as W

from helpers import COMBINE_TOL, bits, dev, f32, i32, max_rel_err, to_bf16

pytestmark = pytest.mark.gpu


def run_both(oracle_mod, idx, E, R, cap=0):
    st = cgl.new_status(dev())
    rl = cgl.get_rank_layout(i32(idx), E, R, cap, status=st)
    torch.cuda.synchronize()
    ref = oracle_mod.get_rank_layout(idx, E, R, cap)
    for f in ("tokens_per_rank", "rank_offset", "rank_dst", "recv_token"):
        g, r = getattr(rl, f).cpu().numpy(), getattr(ref, f)
        assert g.shape == r.shape and np.array_equal(g, r), f"{f} differs at {np.argwhere(g != r)[:5].tolist()}"
    assert int(rl.max_count.item()) == ref.max_count
    bitsv = int(st.item())
    assert bool(bitsv & (1 << cgl.ERANGE)) == bool(ref.flags & oracle_mod.FLAG_RANGE)
    assert bool(bitsv & (1 << cgl.ECAPACITY)) == bool(ref.flags & oracle_mod.FLAG_CAPACITY)
    return rl, ref


@pytest.mark.parametrize("name", W.WORKLOAD_ORDER)
def test_rank_layout_full_size(oracle_mod, name):
    inp = W.make_inputs(name, 0)
    wl = inp.workload
    rl, ref = run_both(oracle_mod, inp.topk_idx, wl.num_experts, wl.num_ranks)
    run_both(oracle_mod, inp.topk_idx, wl.num_experts, wl.num_ranks, ref.max_count)   # padded, exact fit


def test_rank_layout_random_duplicates_bad_ids_overflow(oracle_mod):
    rng = np.random.default_rng(21)
    for n, k, E, R in [(1, 1, 4, 2), (300, 6, 24, 8), (1000, 8, 256, 64), (257, 13, 64, 64), (700, 8, 16, 4)]:
        idx = rng.integers(0, E, (n, k)).astype(np.int32)
        idx[rng.random((n, k)) < 0.05] = -1
        idx[rng.random((n, k)) < 0.01] = E + 3
        rl, ref = run_both(oracle_mod, idx, E, R)
        if ref.max_count > 1:
            run_both(oracle_mod, idx, E, R, max(1, ref.max_count // 2))   # overflow


def test_rank_layout_two_kernel_paths(oracle_mod):
    rng = np.random.default_rng(22)
    idx = np.argsort(rng.random((70000, 64)), axis=1)[:, :2].astype(np.int32)   # > co-resident blocks
    run_both(oracle_mod, idx, 64, 16)
    idx = rng.integers(0, 1024, (900, 32)).astype(np.int32)                       # large shared memory
    run_both(oracle_mod, idx, 1024, 1024)


def test_rank_layout_graph_replays(oracle_mod):
    ids = [W.make_inputs("prefill", s).topk_idx for s in (4, 5)]
    idx = i32(ids[0])
    ws = torch.empty(cgl.layout_workspace_bytes(4096, 8, 64, 64), dtype=torch.uint8, device=dev())
    rl = cgl.get_rank_layout(idx, 256, 64, workspace=ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        cgl.get_rank_layout(idx, 256, 64, workspace=ws, out=rl)
    for a in (ids[1], ids[0], ids[1]):
        idx.copy_(torch.from_numpy(a))
        g.replay()
        torch.cuda.synchronize()
        ref = oracle_mod.get_rank_layout(a, 256, 64)
        assert np.array_equal(rl.rank_dst.cpu().numpy(), ref.rank_dst)
        assert np.array_equal(rl.recv_token.cpu().numpy(), ref.recv_token)
    del g


@pytest.mark.parametrize("name", ["tiny", "prefill"])
def test_dedup_dispatch_and_combine(oracle_mod, name):
    inp = W.make_inputs(name, 0)
    wl = inp.workload
    E, R, h = wl.num_experts, wl.num_ranks, wl.hidden
    rl = cgl.get_rank_layout(i32(inp.topk_idx), E, R)
    ref = oracle_mod.get_rank_layout(inp.topk_idx, E, R)
    rows = rl.num_recv_rows
    # dispatch: one FP8 copy per (token, rank), bit-exact
    st = cgl.new_status(dev())
    rx, rs = cgl.dispatch_fp8(to_bf16(inp.x), rl.rank_dst, rows, status=st)
    ox, os_ = oracle_mod.dispatch_fp8(inp.x, ref.rank_dst, rows)
    used = ref.recv_token >= 0
    assert np.array_equal(rx.cpu().numpy()[used], ox[used])
    assert np.array_equal(rs.cpu().numpy()[used].view(np.uint32), os_[used].view(np.uint32))
    # combine: each rank returns one partial row per token; the origin sums them (unit weights)
    partial = W.expert_outputs(rows, h, 9)
    ones = np.where(ref.rank_dst >= 0, 1.0, 0.0).astype(np.float32)
    out = cgl.combine(to_bf16(partial), rl.rank_dst, f32(ones), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    oo = oracle_mod.combine(partial, ref.rank_dst, ones)
    got = bits(out)
    assert max_rel_err(got, oo) <= COMBINE_TOL and np.array_equal(got, oo)


def test_dedup_path_equals_expert_path_normwise(oracle_mod):
    # per-rank partial sums of the expert outputs, then the rank sum, match the
    # expert-level weighted combine up to the extra BF16 rounding of the partials
    inp = W.make_inputs("prefill", 3, num_tokens=512)
    wl = inp.workload
    E, R, h = wl.num_experts, wl.num_ranks, wl.hidden
    L = oracle_mod.get_layout(inp.topk_idx, E, R)
    y = W.expert_outputs(inp.topk_idx.size, h, 5)
    ref = oracle_mod.combine(y, L.dst_pos, inp.topk_w)
    RL = oracle_mod.get_rank_layout(inp.topk_idx, E, R)
    per = E // R
    yf = W.bf16_bits_to_f32(y)
    partial = np.zeros((inp.topk_idx.size, h), np.float32)
    for t in range(inp.topk_idx.shape[0]):
        for j in range(wl.topk):
            row = RL.rank_dst[t, j]
            if row < 0:
                continue
            r = inp.topk_idx[t, j] // per
            for jj in range(wl.topk):
                if inp.topk_idx[t, jj] // per == r:
                    partial[row] += np.float32(inp.topk_w[t, jj]) * yf[L.dst_pos[t, jj]]
    pb = W.f32_to_bf16_bits(partial)
    ones = np.where(RL.rank_dst >= 0, 1.0, 0.0).astype(np.float32)
    out = bits(cgl.combine(to_bf16(pb), i32(RL.rank_dst), f32(ones)))
    a = W.bf16_bits_to_f32(out).astype(np.float64)
    b = W.bf16_bits_to_f32(ref).astype(np.float64)
    assert np.linalg.norm(a - b) <= 2.0 ** -7 * np.linalg.norm(b)


@pytest.mark.parametrize("n,k,E,R", [(40, 8, 256, 64), (200, 8, 256, 32), (170, 3, 64, 8), (130, 6, 96, 12)])
def test_rank_layout_cluster_sizes(oracle_mod, n, k, E, R):
    """Rank keys on the thread-block-cluster path (2 to 8 one-chunk blocks)."""
    rng = np.random.default_rng(n + 13 * k)
    idx = rng.integers(0, E, (n, k)).astype(np.int32)        # repeated ranks and experts inside tokens
    idx[rng.random((n, k)) < 0.05] = -1
    idx[rng.random((n, k)) < 0.01] = E + 2
    rl, ref = run_both(oracle_mod, idx, E, R)
    run_both(oracle_mod, idx, E, R, max(1, ref.max_count - 1))

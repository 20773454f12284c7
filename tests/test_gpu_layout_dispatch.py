"""Layout + FP8 dispatch in one call (cgl_layout_dispatch_fp8) against the oracle,
bit for bit: every layout output, the FP8 codes and the scales of every
received row; rows that receive nothing stay untouched."""

import numpy as np
import pytest
import torch

import combine_get_layout_02_b200 as cgl
from combine_get_layout_02_b200 import workloads as W

from helpers import dev, i32, to_bf16

pytestmark = pytest.mark.gpu

LAYOUT_FIELDS = ("tokens_per_expert", "tokens_per_rank", "is_token_in_rank", "expert_offset", "dst_pos",
                 "recv_src")


def _check(oracle_mod, x, idx, E, R, cap=0, num_sms=0, scale_offset=0):
    n, h = x.shape
    st = cgl.new_status(dev())
    rows = E * cap if cap > 0 else idx.size
    rx0 = torch.full((rows, h), 0x5A, dtype=torch.uint8, device=dev())
    # scale_offset = 1: a recv_scale that is 4- but not 16-byte aligned (plain scale stores)
    rs_store = torch.full((rows * (h // 128) + 4,), -2.0, dtype=torch.float32, device=dev())
    rs0 = rs_store[scale_offset:scale_offset + rows * (h // 128)].view(rows, h // 128)
    lay, rx, rs = cgl.layout_dispatch_fp8(i32(idx), to_bf16(x), E, R, cap, recv_x=rx0, recv_scale=rs0,
                                          status=st, num_sms=num_sms)
    torch.cuda.synchronize()
    L = oracle_mod.get_layout(idx, E, R, cap)
    for f in LAYOUT_FIELDS:
        g, r = getattr(lay, f).cpu().numpy(), getattr(L, f)
        assert g.shape == r.shape and np.array_equal(g, r), f
    assert int(lay.max_count.item()) == L.max_count
    ox, os_ = oracle_mod.dispatch_fp8(x, L.dst_pos, rows)
    used = L.recv_src >= 0
    gx, gs = rx.cpu().numpy(), rs.cpu().numpy()
    assert np.array_equal(gx[used], ox[used]), "codes"
    assert np.array_equal(gs[used].view(np.uint32), os_[used].view(np.uint32)), "scales"
    assert np.all(gx[~used] == 0x5A) and np.all(gs[~used] == -2.0)
    b = int(st.item())
    assert bool(b & (1 << cgl.ECAPACITY)) == bool(L.flags & oracle_mod.FLAG_CAPACITY)
    assert bool(b & (1 << cgl.ERANGE)) == bool(L.flags & oracle_mod.FLAG_RANGE)
    assert not b & (1 << cgl.ETIMEOUT)


@pytest.mark.parametrize("name", ["prefill", "skewed", "decode", "tiny"])
def test_layout_dispatch_fp8_workloads(oracle_mod, name):
    inp = W.make_inputs(name, 0)
    wl = inp.workload
    _check(oracle_mod, inp.x, inp.topk_idx, wl.num_experts, wl.num_ranks)
    if wl.padded:
        cap = oracle_mod.get_layout(inp.topk_idx, wl.num_experts, wl.num_ranks).max_count
        _check(oracle_mod, inp.x, inp.topk_idx, wl.num_experts, wl.num_ranks, cap)


def test_layout_dispatch_fp8_takes_one_launch_at_prefill():
    wl = W.WORKLOADS["prefill"]
    assert cgl.layout_dispatch_kernel_count(wl.num_tokens, wl.topk, wl.num_experts, wl.num_ranks, wl.hidden) == 1
    # 16384 tokens at hidden 7168: 111 per CTA do not fit in shared memory -> separate kernels
    assert cgl.layout_dispatch_kernel_count(16384, 8, 256, 64, 7168) > 1
    # 128 tokens, at most one per SM: one CTA per token does layout and dispatch
    assert cgl.layout_dispatch_kernel_count(128, 8, 256, 32, 7168) == 1
    # 1000 tokens: too few pairs per SM for the fused prefill kernel -> layout, then dispatch
    assert cgl.layout_dispatch_kernel_count(1000, 8, 256, 64, 7168) > 1


def test_layout_dispatch_fp8_fused_on_fewer_sms(oracle_mod):
    inp = W.make_inputs("prefill", 4, num_tokens=2800)
    wl = inp.workload
    assert cgl.layout_dispatch_kernel_count(2800, wl.topk, wl.num_experts, wl.num_ranks, wl.hidden, num_sms=100) == 1
    _check(oracle_mod, inp.x, inp.topk_idx, wl.num_experts, wl.num_ranks, num_sms=100)   # 28 tokens per CTA
    cap = oracle_mod.get_layout(inp.topk_idx, wl.num_experts, wl.num_ranks).max_count
    _check(oracle_mod, inp.x, inp.topk_idx, wl.num_experts, wl.num_ranks, cap - 2, num_sms=100)


@pytest.mark.parametrize("n,h,k,E,R,seed", [
    (1, 128, 1, 4, 2, 0), (37, 384, 8, 64, 8, 1), (300, 256, 4, 16, 4, 2), (1000, 7168, 8, 256, 64, 3),
    (2049, 1024, 6, 96, 12, 4), (5000, 512, 8, 256, 32, 5), (9000, 2048, 8, 128, 16, 6)])
def test_layout_dispatch_fp8_ragged_masked_bad_ids(oracle_mod, n, h, k, E, R, seed):
    rng = np.random.default_rng(seed)
    x = W.f32_to_bf16_bits((rng.standard_normal((n, h)) * rng.choice([1e-3, 1.0, 300.0])).astype(np.float32))
    idx = np.stack([rng.permutation(E)[:k] for _ in range(n)]).astype(np.int32)
    idx[rng.random((n, k)) < 0.05] = -1
    idx[rng.random((n, k)) < 0.01] = E + 3
    _check(oracle_mod, x, idx, E, R)


def test_layout_dispatch_fp8_capacity_overflow_duplicates_and_zero_rows(oracle_mod):
    rng = np.random.default_rng(11)
    n, h, k, E, R = 3000, 1024, 8, 32, 8
    x = W.f32_to_bf16_bits(rng.standard_normal((n, h)).astype(np.float32))
    x[::7] = 0                                   # all-zero rows: amax clamps to 1e-4
    idx = rng.integers(0, E, (n, k)).astype(np.int32)      # repeated experts inside a token
    cap = oracle_mod.get_layout(idx, E, R).max_count
    _check(oracle_mod, x, idx, E, R, cap - 5)    # some experts overflow
    _check(oracle_mod, x, idx, E, R, cap + 3)


def test_layout_dispatch_fp8_unaligned_scales_and_fewer_sms(oracle_mod):
    inp = W.make_inputs("prefill", 1)
    wl = inp.workload
    _check(oracle_mod, inp.x, inp.topk_idx, wl.num_experts, wl.num_ranks, scale_offset=1)
    _check(oracle_mod, inp.x, inp.topk_idx, wl.num_experts, wl.num_ranks, num_sms=40)   # 103 per CTA: split path


def test_layout_dispatch_fp8_falls_back_when_fused_does_not_apply(oracle_mod):
    rng = np.random.default_rng(5)
    n, h, k, E, R = 600, 256, 32, 1024, 64      # the layout needs more than the default shared memory
    x = W.f32_to_bf16_bits(rng.standard_normal((n, h)).astype(np.float32))
    idx = np.stack([rng.permutation(E)[:k] for _ in range(n)]).astype(np.int32)
    _check(oracle_mod, x, idx, E, R)
    big = 150 * 300                              # more than 256 tokens per CTA on 148 SMs
    assert cgl.layout_dispatch_kernel_count(big, 4, 64, 8, 128) > 1


def test_layout_dispatch_fp8_graph_replays(oracle_mod):
    inps = [W.make_inputs("prefill", s) for s in (2, 3)]
    wl = inps[0].workload
    E, R = wl.num_experts, wl.num_ranks
    idx = i32(inps[0].topk_idx)
    x = to_bf16(inps[0].x)
    ws = torch.empty(cgl.layout_dispatch_workspace_bytes(wl.num_tokens, wl.topk, E, R), dtype=torch.uint8,
                     device=dev())
    lay, rx, rs = cgl.layout_dispatch_fp8(idx, x, E, R, workspace=ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        cgl.layout_dispatch_fp8(idx, x, E, R, out=lay, recv_x=rx, recv_scale=rs, workspace=ws)
    for i in (inps[1], inps[0], inps[1]):
        idx.copy_(torch.from_numpy(i.topk_idx))
        x.copy_(to_bf16(i.x))
        g.replay()
        torch.cuda.synchronize()
        L = oracle_mod.get_layout(i.topk_idx, E, R)
        assert np.array_equal(lay.dst_pos.cpu().numpy(), L.dst_pos)
        ox, os_ = oracle_mod.dispatch_fp8(i.x, L.dst_pos, idx.numel())
        used = L.recv_src >= 0
        assert np.array_equal(rx.cpu().numpy()[used], ox[used])
        assert np.array_equal(rs.cpu().numpy()[used].view(np.uint32), os_[used].view(np.uint32))
    del g


@pytest.mark.parametrize("num_tokens,num_sms", [(6000, 0), (16384, 0), (5000, 37)])
def test_layout_dispatch_fp8_two_kernels_hand_tokens_out_dynamically(oracle_mod, num_tokens, num_sms):
    """Past the fused kernel's range the call runs the layout and then the
    dispatch kernel, whose CTAs claim tokens from a counter at the workspace's
    tail (zeroed by the call).  Every token is dispatched exactly once, bit for
    bit, whatever the workspace held before (the counter word included), call
    after call on one workspace and in graph replays."""
    inp = W.make_inputs("skewed", 3, num_tokens=num_tokens)
    wl = inp.workload
    E, R = wl.num_experts, wl.num_ranks
    n, k = inp.topk_idx.shape
    assert cgl.layout_dispatch_kernel_count(n, k, E, R, wl.hidden, num_sms=num_sms) > 1
    nbytes = cgl.layout_dispatch_workspace_bytes(n, k, E, R)
    ws = torch.full((nbytes,), 0x7F, dtype=torch.uint8, device=dev())   # counter word far from zero
    idx, x = i32(inp.topk_idx), to_bf16(inp.x)
    L = oracle_mod.get_layout(inp.topk_idx, E, R)
    ox, os_ = oracle_mod.dispatch_fp8(inp.x, L.dst_pos, n * k)
    used = L.recv_src >= 0

    def check(rx, rs, st):
        assert np.array_equal(rx.cpu().numpy()[used], ox[used]), "codes"
        assert np.array_equal(rs.cpu().numpy()[used].view(np.uint32), os_[used].view(np.uint32)), "scales"
        assert st.item() == 0

    rx = torch.full((n * k, wl.hidden), 0x5A, dtype=torch.uint8, device=dev())
    rs = torch.full((n * k, wl.hidden // 128), -2.0, dtype=torch.float32, device=dev())
    st = cgl.new_status(dev())
    for _ in range(3):
        lay, rx, rs = cgl.layout_dispatch_fp8(idx, x, E, R, recv_x=rx, recv_scale=rs, workspace=ws, status=st,
                                              num_sms=num_sms)
        torch.cuda.synchronize()
        assert np.array_equal(lay.dst_pos.cpu().numpy(), L.dst_pos)
        check(rx, rs, st)
        rx.fill_(0x5A)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        cgl.layout_dispatch_fp8(idx, x, E, R, out=lay, recv_x=rx, recv_scale=rs, workspace=ws, status=st,
                                num_sms=num_sms)
    for _ in range(2):
        rx.fill_(0x5A)
        g.replay()
        torch.cuda.synchronize()
        check(rx, rs, st)
    del g

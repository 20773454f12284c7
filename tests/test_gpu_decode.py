"""Fused decode path (layout + FP8 dispatch in one launch) against the oracle, bit for bit."""

import numpy as np
import pytest
import torch

import combine_get_layout_02_b200 as cgl
from combine_get_layout_02_b200 import workloads as W

from helpers import dev, i32, to_bf16

pytestmark = pytest.mark.gpu


def _check(oracle_mod, inp_x, idx, E, R, cap, num_sms=0):
    n, h = inp_x.shape
    st = cgl.new_status(dev())
    rows = E * cap if cap > 0 else idx.size
    rx0 = torch.full((rows, h), 0x5A, dtype=torch.uint8, device=dev())
    rs0 = torch.full((rows, h // 128), -2.0, dtype=torch.float32, device=dev())
    lay, rx, rs = cgl.decode_dispatch_fp8(i32(idx), to_bf16(inp_x), E, R, cap, recv_x=rx0, recv_scale=rs0,
                                          status=st, num_sms=num_sms)
    torch.cuda.synchronize()
    L = oracle_mod.get_layout(idx, E, R, cap)
    for f in ("tokens_per_expert", "tokens_per_rank", "is_token_in_rank", "expert_offset", "dst_pos", "recv_src"):
        g, r = getattr(lay, f).cpu().numpy(), getattr(L, f)
        assert np.array_equal(g, r), f
    assert int(lay.max_count.item()) == L.max_count
    ox, os_ = oracle_mod.dispatch_fp8(inp_x, L.dst_pos, rows)
    used = L.recv_src >= 0
    gx, gs = rx.cpu().numpy(), rs.cpu().numpy()
    assert np.array_equal(gx[used], ox[used]) and np.array_equal(gs[used].view(np.uint32), os_[used].view(np.uint32))
    assert np.all(gx[~used] == 0x5A) and np.all(gs[~used] == -2.0)     # rows without a copy untouched
    b = int(st.item())
    assert bool(b & (1 << cgl.ECAPACITY)) == bool(L.flags & oracle_mod.FLAG_CAPACITY)
    assert bool(b & (1 << cgl.ERANGE)) == bool(L.flags & oracle_mod.FLAG_RANGE)


def test_fused_decode_padded(oracle_mod):
    inp = W.make_inputs("decode", 0)
    cap = oracle_mod.get_layout(inp.topk_idx, 256, 32).max_count
    _check(oracle_mod, inp.x, inp.topk_idx, 256, 32, cap)
    _check(oracle_mod, inp.x, inp.topk_idx, 256, 32, cap + 7, num_sms=16)     # spare rows, fewer CTAs


def test_fused_decode_overflow_and_compact(oracle_mod):
    inp = W.make_inputs("decode", 1)
    cap = oracle_mod.get_layout(inp.topk_idx, 256, 32).max_count
    _check(oracle_mod, inp.x, inp.topk_idx, 256, 32, max(1, cap - 3))          # some experts overflow
    _check(oracle_mod, inp.x, inp.topk_idx, 256, 32, 0)                        # compact rows
    t = W.make_inputs("tiny", 0)                                                 # k = 4, 128 tokens
    _check(oracle_mod, t.x, t.topk_idx, 16, 4, 0)


def test_fused_decode_masked_bad_ids_ragged(oracle_mod):
    rng = np.random.default_rng(17)
    for n, h, k, E, R in [(1, 128, 1, 4, 2), (37, 384, 8, 64, 8), (256, 256, 4, 16, 4), (100, 7168, 8, 256, 64)]:
        x = W.f32_to_bf16_bits(rng.standard_normal((n, h)).astype(np.float32))
        idx = np.stack([rng.permutation(E)[:k] for _ in range(n)]).astype(np.int32)
        idx[rng.random((n, k)) < 0.1] = -1
        idx[rng.random((n, k)) < 0.02] = E + 1
        _check(oracle_mod, x, idx, E, R, 0)


def test_fused_decode_in_a_graph(oracle_mod):
    inps = [W.make_inputs("decode", s) for s in (2, 3, 4)]
    cap = 24   # fixed in advance, above every batch's largest expert count here
    assert all(oracle_mod.get_layout(i.topk_idx, 256, 32).max_count <= cap for i in inps)
    idx = i32(inps[0].topk_idx)
    x = to_bf16(inps[0].x)
    lay, rx, rs = cgl.decode_dispatch_fp8(idx, x, 256, 32, cap)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        cgl.decode_dispatch_fp8(idx, x, 256, 32, cap, out=lay, recv_x=rx, recv_scale=rs)
    for i in (inps[1], inps[2], inps[0]):
        idx.copy_(torch.from_numpy(i.topk_idx))
        x.copy_(to_bf16(i.x))
        g.replay()
        torch.cuda.synchronize()
        L = oracle_mod.get_layout(i.topk_idx, 256, 32, cap)
        assert np.array_equal(lay.dst_pos.cpu().numpy(), L.dst_pos)
        ox, _ = oracle_mod.dispatch_fp8(i.x, L.dst_pos, 256 * cap)
        used = L.recv_src >= 0
        assert np.array_equal(rx.cpu().numpy()[used], ox[used])
    del g


@pytest.mark.parametrize("n,k,E,R", [(0, 8, 256, 32), (1, 8, 256, 32), (2, 8, 256, 64), (5, 8, 256, 256),
                                     (64, 8, 512, 512), (148, 3, 48, 12), (30, 32, 64, 8)])
def test_fused_decode_one_token_per_cta_shapes(oracle_mod, n, k, E, R):
    """Batches of at most one token per SM take one CTA per token: empty and
    one-token batches, more ranks than one CTA's 32 designated ranks (the
    general kernel then), k that is not a multiple of 4, top-32, and repeated
    experts inside tokens; compact, padded and overflowing."""
    rng = np.random.default_rng(n * 13 + k + E)
    h = 256
    x = W.f32_to_bf16_bits(rng.standard_normal((n, h)).astype(np.float32))
    idx = rng.integers(0, E, (n, k)).astype(np.int32)
    if n:
        idx[rng.random((n, k)) < 0.05] = -1
    _check(oracle_mod, x, idx, E, R, 0)
    mc = int(oracle_mod.get_layout(idx, E, R).max_count) if n else 0
    _check(oracle_mod, x, idx, E, R, max(1, mc))
    if mc > 1:
        _check(oracle_mod, x, idx, E, R, mc - 1)

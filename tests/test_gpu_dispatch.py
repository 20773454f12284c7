"""GPU FP8 / BF16 dispatch against the oracle through the C ABI: bit-exact bytes and scales."""

import numpy as np
import pytest
import torch

import combine_get_layout_02_b200 as cgl
from combine_get_layout_02_b200 import workloads as W

from helpers import bits, dev, i32, to_bf16

pytestmark = pytest.mark.gpu


def _fp8_case(oracle_mod, x, idx, E, R, cap=0, sentinel=None, num_sms=0):
    st = cgl.new_status(dev())
    lay = cgl.get_layout(i32(idx), E, R, cap, status=st)
    rows = lay.num_recv_rows
    rx = torch.full((rows, x.shape[1]), sentinel if sentinel is not None else 0, dtype=torch.uint8, device=dev())
    rs = torch.full((rows, x.shape[1] // 128), -1.0, dtype=torch.float32, device=dev())
    cgl.dispatch_fp8(to_bf16(x), lay.dst_pos, rows, recv_x=rx, recv_scale=rs, status=st, num_sms=num_sms)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    L = oracle_mod.get_layout(idx, E, R, cap)
    ox, os_ = oracle_mod.dispatch_fp8(x, L.dst_pos, rows)
    gx, gs = rx.cpu().numpy(), rs.cpu().numpy()
    used = L.recv_src >= 0
    assert np.array_equal(gx[used], ox[used]), f"fp8 bytes differ in rows {np.argwhere((gx != ox).any(1) & used)[:5].ravel().tolist()}"
    assert np.array_equal(gs[used].view(np.uint32), os_[used].view(np.uint32)), "scales differ"
    if sentinel is not None:   # rows that receive nothing stay untouched
        assert np.all(gx[~used] == sentinel) and np.all(gs[~used] == -1.0)
    return gx, gs


@pytest.mark.parametrize("name", ["tiny", "decode", "prefill", "skewed"])
def test_fp8_dispatch_full_size(oracle_mod, name):
    inp = W.make_inputs(name, 0)
    wl = inp.workload
    cap = 0
    if wl.padded:
        cap = oracle_mod.get_layout(inp.topk_idx, wl.num_experts, wl.num_ranks).max_count
    _fp8_case(oracle_mod, inp.x, inp.topk_idx, wl.num_experts, wl.num_ranks, cap,
              sentinel=0xAB if wl.padded else None)


def test_fp8_codec_every_bf16_value(oracle_mod):
    """Blocks whose absmax is 448 have inv == 1, so the codes are e4m3(x) of
    every finite BF16 value in [-448, 448]: checks the GPU's cvt rounding,
    saturation and byte order against the oracle's encoder."""
    b = np.arange(65536, dtype=np.uint32)
    v = (b << 16).view(np.float32)
    keep = np.isfinite(v) & (np.abs(v) <= 448.0)
    vals = b[keep].astype(np.uint16)
    per = 127
    nblk = -(-vals.size // per)
    vals = np.concatenate([vals, np.zeros(nblk * per - vals.size, np.uint16)])
    blocks = np.concatenate([np.full((nblk, 1), 0x43E0, np.uint16), vals.reshape(nblk, per)], axis=1)  # 0x43E0 = 448
    h = 1024
    blocks = np.concatenate([blocks, np.tile(blocks[:1], (-nblk % (h // 128), 1))])
    x = blocks.reshape(-1, h)
    n = x.shape[0]
    idx = np.zeros((n, 1), np.int32)
    gx, gs = _fp8_case(oracle_mod, x, idx, 1, 1)
    assert np.all(gs == 1.0)
    assert np.array_equal(gx.reshape(-1, 128)[:, 1:].ravel()[:keep.sum()],
                          oracle_mod.e4m3_encode((vals[:keep.sum()].astype(np.uint32) << 16).view(np.float32)))


def test_fp8_scales_across_magnitudes(oracle_mod):
    """Block maxima from 1e-38 to 3e38 (and all-zero blocks): the IEEE scale
    divisions, the 1e-4 floor and subnormal codes must match the oracle."""
    rng = np.random.default_rng(0)
    n, h = 300, 7168
    exps = rng.uniform(-126, 127, (n, h // 128, 1))
    x32 = (rng.standard_normal((n, h // 128, 128)) * np.exp2(exps)).astype(np.float32)
    x32[rng.random((n, h // 128)) < 0.05] = 0.0
    x32[:, :, 5] *= rng.choice([1, 1e3, 1e-3], (n, h // 128)).astype(np.float32)
    x = W.f32_to_bf16_bits(np.clip(x32, -3e38, 3e38).reshape(n, h))
    idx = np.stack([rng.permutation(32)[:4] for _ in range(n)]).astype(np.int32)
    _fp8_case(oracle_mod, x, idx, 32, 8)


def test_fp8_ragged_and_tiny_hidden(oracle_mod):
    rng = np.random.default_rng(5)
    for n, h, k, E in [(1, 128, 1, 1), (3, 256, 3, 5), (1001, 384, 6, 24), (257, 7168, 8, 256), (40, 16512, 2, 8)]:
        x = W.f32_to_bf16_bits(rng.standard_normal((n, h)).astype(np.float32))
        idx = np.stack([rng.permutation(E)[:k] for _ in range(n)]).astype(np.int32)
        idx[rng.random((n, k)) < 0.1] = -1
        _fp8_case(oracle_mod, x, idx, E, 1, sentinel=0x5C)


def test_fp8_sm_cap_gives_same_bytes(oracle_mod):
    inp = W.make_inputs("prefill", 1, num_tokens=1024)
    a = _fp8_case(oracle_mod, inp.x, inp.topk_idx, 256, 64, num_sms=7)
    b = _fp8_case(oracle_mod, inp.x, inp.topk_idx, 256, 64, num_sms=0)
    assert np.array_equal(a[0], b[0])


def test_dispatch_reports_rows_outside_the_buffer():
    x = torch.zeros((4, 256), dtype=torch.bfloat16, device=dev())
    dst = i32(np.array([[0, 1], [2, 3], [4, 5], [6, 99]], np.int32))
    st = cgl.new_status(dev())
    rx, rs = cgl.dispatch_fp8(x, dst, 8, status=st)
    torch.cuda.synchronize()
    assert cgl.status_bits(st) == ["CGL_ERANGE"]
    st.zero_()
    cgl.dispatch_bf16(x, dst, 8, status=st)
    torch.cuda.synchronize()
    assert cgl.status_bits(st) == ["CGL_ERANGE"]


def test_bf16_dispatch_shapes(oracle_mod):
    # staged bulk path (hidden % 16 == 0, <= 8192) and the flattened path (others)
    rng = np.random.default_rng(8)
    for n, h, k, E in [(1, 16, 1, 1), (5, 24, 3, 7), (300, 4096, 4, 16), (77, 8200, 2, 4), (33, 9000, 3, 6)]:
        x = W.f32_to_bf16_bits(rng.standard_normal((n, h)).astype(np.float32))
        idx = np.stack([rng.permutation(E)[:k] for _ in range(n)]).astype(np.int32)
        idx[rng.random((n, k)) < 0.1] = -1
        lay = cgl.get_layout(i32(idx), E, 1)
        rows = lay.num_recv_rows
        recv = torch.full((rows, h), 0x1234, dtype=torch.int16, device=dev()).view(torch.bfloat16)
        cgl.dispatch_bf16(to_bf16(x), lay.dst_pos, rows, recv_x=recv)
        L = oracle_mod.get_layout(idx, E, 1)
        ref = oracle_mod.dispatch_bf16(x, L.dst_pos, rows)
        used = L.recv_src >= 0
        got = bits(recv)
        assert np.array_equal(got[used], ref[used]) and np.all(got[~used] == 0x1234)


@pytest.mark.parametrize("name", ["tiny", "bf16"])
def test_bf16_dispatch_and_backward_full_size(oracle_mod, name):
    inp = W.make_inputs(name, 0)
    wl = inp.workload
    st = cgl.new_status(dev())
    lay = cgl.get_layout(i32(inp.topk_idx), wl.num_experts, wl.num_ranks, status=st)
    rows = lay.num_recv_rows
    recv = cgl.dispatch_bf16(to_bf16(inp.x), lay.dst_pos, rows, status=st)
    L = oracle_mod.get_layout(inp.topk_idx, wl.num_experts, wl.num_ranks)
    assert np.array_equal(bits(recv), oracle_mod.dispatch_bf16(inp.x, L.dst_pos, rows))
    if inp.grad is not None:   # combine-backward: grads re-dispatched by the same layout
        g = cgl.dispatch_bf16(to_bf16(inp.grad), lay.dst_pos, rows, status=st)
        assert np.array_equal(bits(g), oracle_mod.dispatch_bf16(inp.grad, L.dst_pos, rows))
    torch.cuda.synchronize()
    assert int(st.item()) == 0


@pytest.mark.parametrize("name,num_sms", [("prefill", 0), ("skewed", 0), ("decode", 0), ("prefill", 23)])
def test_fp8_dispatch_with_scratch_hands_tokens_out(oracle_mod, name, num_sms):
    """cgl_opts.scratch: the dispatch CTAs claim tokens from a counter in it.
    Same bytes and scales as the oracle (and the fixed order), call after call
    on one scratch, which every call leaves zero; in a graph replay too."""
    inp = W.make_inputs(name, 0)
    wl = inp.workload
    E, R = wl.num_experts, wl.num_ranks
    cap = oracle_mod.get_layout(inp.topk_idx, E, R).max_count if wl.padded else 0
    lay = cgl.get_layout(i32(inp.topk_idx), E, R, cap)
    rows = lay.num_recv_rows
    L = oracle_mod.get_layout(inp.topk_idx, E, R, cap)
    ox, os_ = oracle_mod.dispatch_fp8(inp.x, L.dst_pos, rows)
    used = L.recv_src >= 0
    x = to_bf16(inp.x)
    sc = cgl.new_scratch(dev())
    st = cgl.new_status(dev())
    rx = torch.zeros((rows, wl.hidden), dtype=torch.uint8, device=dev())
    rs = torch.zeros((rows, wl.hidden // 128), dtype=torch.float32, device=dev())

    def check():
        torch.cuda.synchronize()
        assert np.array_equal(rx.cpu().numpy()[used], ox[used])
        assert np.array_equal(rs.cpu().numpy()[used].view(np.uint32), os_[used].view(np.uint32))
        assert int(st.item()) == 0 and torch.count_nonzero(sc).item() == 0

    for _ in range(3):
        rx.zero_()
        cgl.dispatch_fp8(x, lay.dst_pos, rows, recv_x=rx, recv_scale=rs, status=st, num_sms=num_sms, scratch=sc)
        check()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        cgl.dispatch_fp8(x, lay.dst_pos, rows, recv_x=rx, recv_scale=rs, status=st, num_sms=num_sms, scratch=sc)
    for _ in range(2):
        rx.zero_()
        g.replay()
        check()
    del g
    # stream-ordered calls may share one scratch: FP8 and BF16 dispatches back to
    # back with no host synchronisation between them, each starting from the word
    # the one before left zero
    rx.zero_()
    check_bf16 = wl.hidden <= 8192 and rows * wl.hidden <= 1 << 28   # host copies stay under 1 GB
    for _ in range(3):
        cgl.dispatch_fp8(x, lay.dst_pos, rows, recv_x=rx, recv_scale=rs, status=st, num_sms=num_sms, scratch=sc)
        rb = cgl.dispatch_bf16(x, lay.dst_pos, rows, status=st, num_sms=num_sms, scratch=sc)
    check()
    if check_bf16:
        assert np.array_equal(bits(rb)[used], oracle_mod.dispatch_bf16(inp.x, L.dst_pos, rows)[used])


def test_bf16_dispatch_with_scratch_hands_tokens_out(oracle_mod):
    """cgl_opts.scratch on the BF16 dispatch (and the combine-backward re-dispatch):
    bit-exact rows at the BF16 workload's full size, scratch left zero; the
    flattened kernel (hidden above the staged path's limit) ignores it."""
    inp = W.make_inputs("bf16", 0)
    wl = inp.workload
    lay = cgl.get_layout(i32(inp.topk_idx), wl.num_experts, wl.num_ranks)
    rows = lay.num_recv_rows
    L = oracle_mod.get_layout(inp.topk_idx, wl.num_experts, wl.num_ranks)
    sc = cgl.new_scratch(dev())
    st = cgl.new_status(dev())
    for src in (inp.x, inp.grad, inp.x):
        recv = cgl.dispatch_bf16(to_bf16(src), lay.dst_pos, rows, status=st, scratch=sc)
        torch.cuda.synchronize()
        assert np.array_equal(bits(recv), oracle_mod.dispatch_bf16(src, L.dst_pos, rows))
        assert torch.count_nonzero(sc).item() == 0
    rng = np.random.default_rng(13)
    n, h, k, E = 40, 9000, 3, 6
    x = W.f32_to_bf16_bits(rng.standard_normal((n, h)).astype(np.float32))
    idx = np.stack([rng.permutation(E)[:k] for _ in range(n)]).astype(np.int32)
    lay2 = cgl.get_layout(i32(idx), E, 1)
    got = cgl.dispatch_bf16(to_bf16(x), lay2.dst_pos, lay2.num_recv_rows, status=st, scratch=sc)
    torch.cuda.synchronize()
    L2 = oracle_mod.get_layout(idx, E, 1)
    assert np.array_equal(bits(got), oracle_mod.dispatch_bf16(x, L2.dst_pos, lay2.num_recv_rows))
    assert int(st.item()) == 0 and torch.count_nonzero(sc).item() == 0


@pytest.mark.parametrize("start", [10**9, -1])
def test_dispatch_scratch_not_zero_is_reported(oracle_mod, start):
    """A scratch whose counter did not start at zero (here 1e9, or 2^64 - 1 as
    the int64 -1) is clamped by the kernel: every claim past the batch becomes
    "no token", nothing outside the buffers is touched, and CGL_ERANGE is set.
    The launch still leaves the scratch zero, so the next call is exact."""
    inp = W.make_inputs("prefill", 0)
    wl = inp.workload
    lay = cgl.get_layout(i32(inp.topk_idx), wl.num_experts, wl.num_ranks)
    rows = lay.num_recv_rows
    L = oracle_mod.get_layout(inp.topk_idx, wl.num_experts, wl.num_ranks)
    ox, os_ = oracle_mod.dispatch_fp8(inp.x, L.dst_pos, rows)
    x = to_bf16(inp.x)
    rx = torch.zeros((rows, wl.hidden), dtype=torch.uint8, device=dev())
    rs = torch.zeros((rows, wl.hidden // 128), dtype=torch.float32, device=dev())
    for kind in ("fp8", "bf16"):
        sc = torch.tensor([start, 0], dtype=torch.int64, device=dev())
        st = cgl.new_status(dev())
        if kind == "fp8":
            cgl.dispatch_fp8(x, lay.dst_pos, rows, recv_x=rx, recv_scale=rs, status=st, scratch=sc)
        else:
            cgl.dispatch_bf16(x, lay.dst_pos, rows, status=st, scratch=sc)
        torch.cuda.synchronize()
        assert int(st.item()) == 1 << cgl.ERANGE
        assert torch.count_nonzero(sc).item() == 0
        st.zero_()
        rx.zero_()
        if kind == "fp8":
            cgl.dispatch_fp8(x, lay.dst_pos, rows, recv_x=rx, recv_scale=rs, status=st, scratch=sc)
            torch.cuda.synchronize()
            used = L.recv_src >= 0
            assert np.array_equal(rx.cpu().numpy()[used], ox[used])
            assert np.array_equal(rs.cpu().numpy()[used].view(np.uint32), os_[used].view(np.uint32))
        else:
            got = cgl.dispatch_bf16(x, lay.dst_pos, rows, status=st, scratch=sc)
            torch.cuda.synchronize()
            assert np.array_equal(bits(got), oracle_mod.dispatch_bf16(inp.x, L.dst_pos, rows))
        assert int(st.item()) == 0

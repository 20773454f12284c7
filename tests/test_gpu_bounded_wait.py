"""Failure detection on the GPU without a fault.

The layout's bounded inter-block wait, run on flags that hold no tag it waits
for, gives up after about a second, reports CGL_ETIMEOUT in the status word,
advances the workspace's generation word (as a layout block that times out
does) and leaves the context usable.  A timed-out exchange must not let a
later layout call on the same workspace pass its exchange on flags left
behind, and no workspace contents may make a layout call wrong."""

import ctypes as C
import time

import numpy as np
import pytest
import torch

import combine_get_layout_02_b200 as cgl
from combine_get_layout_02_b200 import workloads as W

from helpers import dev, i32, to_bf16

pytestmark = pytest.mark.gpu

LAYOUT_FIELDS = ("tokens_per_expert", "tokens_per_rank", "is_token_in_rank", "expert_offset", "dst_pos",
                 "recv_src")


def _probe():
    f = cgl.lib().cgl_selftest_bounded_wait
    f.argtypes = [C.c_void_p, C.c_int, C.c_void_p, C.c_void_p]
    f.restype = C.c_int
    return f


def _words(ws: torch.Tensor) -> torch.Tensor:
    """The workspace as 64-bit words (generation word, then one flag per block)."""
    return ws.view(torch.int64)


def _assert_layout(oracle_mod, lay, idx_np, E, R, cap=0):
    L = oracle_mod.get_layout(idx_np, E, R, cap)
    for f in LAYOUT_FIELDS:
        g, r = getattr(lay, f).cpu().numpy(), getattr(L, f)
        assert g.shape == r.shape and np.array_equal(g, r), f
    assert int(lay.max_count.item()) == L.max_count


def test_bounded_wait_times_out_advances_generation_and_context_survives(oracle_mod):
    f = _probe()
    hdr = torch.zeros(1 + 4, dtype=torch.int64, device=dev())
    hdr[0] = 41                                   # generation word
    st = cgl.new_status(dev())
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    assert f(hdr.data_ptr(), 4, st.data_ptr(), torch.cuda.current_stream().cuda_stream) == cgl.OK
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert cgl.status_bits(st) == ["CGL_ETIMEOUT"]
    assert 0.3 < elapsed < 10.0
    assert int(hdr[0].item()) == 42               # the timed-out wait advanced the generation
    assert torch.count_nonzero(hdr[1:]).item() == 0
    # the device still works: a full layout afterwards matches the oracle
    inp = W.make_inputs("prefill", 7)
    lay = cgl.get_layout(i32(inp.topk_idx), 256, 64)
    _assert_layout(oracle_mod, lay, inp.topk_idx, 256, 64)


def test_graph_replay_after_a_timed_out_exchange_gets_a_new_tag(oracle_mod):
    """A captured layout call keeps its host salt on every replay, so only the
    generation tells its launches apart.  Put the workspace in the state a
    timed-out replay would have left without the generation advance (every
    flag published with the tag of the generation word's next launch), run
    the wait's timeout path on it, then replay with new ids: the replay must
    not take those flags for its own."""
    a, b = W.make_inputs("skewed", 2), W.make_inputs("skewed", 3)
    E, R = 256, 64
    n, k = a.topk_idx.shape
    assert n * k > 32768                                      # past the replicated-count layout:
    assert cgl.layout_kernel_count(n, k, E, R) == 1          # the cooperative exchange
    ws = torch.zeros(cgl.layout_workspace_bytes(n, k, E, R), dtype=torch.uint8, device=dev())
    idx = i32(a.topk_idx)
    st = cgl.new_status(dev())
    lay = cgl.get_layout(idx, E, R, workspace=ws, status=st)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        cgl.get_layout(idx, E, R, workspace=ws, out=lay, status=st)
    g.replay()
    torch.cuda.synchronize()
    _assert_layout(oracle_mod, lay, a.topk_idx, E, R)
    words = _words(ws)
    gen = int(words[0].item())
    nb = (n + 127) // 128                                     # 128 tokens per block at this size
    flags = words[1:1 + nb]
    assert torch.all(flags == flags[0]).item() and (int(flags[0].item()) & 0xFFFFFFFF) == (gen & 0xFFFFFFFF)
    # the state a replay that timed out before advancing would leave: generation
    # one back, every flag holding the tag the next replay would compute from it
    words[0] = gen - 1
    st_p = cgl.new_status(dev())
    assert _probe()(ws.data_ptr(), nb, st_p.data_ptr(), torch.cuda.current_stream().cuda_stream) == cgl.OK
    torch.cuda.synchronize()
    assert cgl.status_bits(st_p) == ["CGL_ETIMEOUT"]
    assert int(words[0].item()) == gen                        # the timeout path advanced it again
    idx.copy_(torch.from_numpy(b.topk_idx))
    g.replay()
    torch.cuda.synchronize()
    _assert_layout(oracle_mod, lay, b.topk_idx, E, R)
    assert int(words[0].item()) == gen + 1
    assert st.item() == 0
    del g


@pytest.mark.parametrize("fill", ["old_tag", "zeros", "ones"])
def test_layout_calls_are_right_on_any_workspace_contents(oracle_mod, fill):
    """A workspace with a generation word g, flags equal to the tag scheme an
    earlier build used for generation g + 1, and garbage count rows; or all
    zero, or all ones: both calls that exchange counts through it (the layout,
    and the layout + FP8 dispatch, which at 16384 tokens runs the layout and
    dispatch kernels) match the oracle bit for bit."""
    a = W.make_inputs("skewed", 5)
    E, R = 256, 64
    n, k = a.topk_idx.shape
    wl = a.workload
    assert cgl.layout_kernel_count(n, k, E, R) == 1
    assert cgl.layout_dispatch_kernel_count(n, k, E, R, wl.hidden) == 2
    nbytes = max(cgl.layout_workspace_bytes(n, k, E, R), cgl.layout_dispatch_workspace_bytes(n, k, E, R))
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev())
    words = _words(ws)
    rng = np.random.default_rng(9)
    if fill == "old_tag":
        g = 123456
        garbage = rng.integers(0, 2 ** 31, ws.numel() // 4, dtype=np.int64).astype(np.int32)
        ws.view(torch.int32).copy_(torch.from_numpy(garbage))
        words[0] = g
        words[1:257] = (0x9E3779B9 << 32 | (g + 1)) - (1 << 64)   # as a signed 64-bit value
    elif fill == "zeros":
        ws.zero_()
    else:
        ws.fill_(0xFF)
    for _ in range(2):   # the second call sees what the first left behind
        st = cgl.new_status(dev())
        lay = cgl.get_layout(i32(a.topk_idx), E, R, workspace=ws, status=st)
        torch.cuda.synchronize()
        _assert_layout(oracle_mod, lay, a.topk_idx, E, R)
        assert st.item() == 0
    st = cgl.new_status(dev())
    lay, rx, rs = cgl.layout_dispatch_fp8(i32(a.topk_idx), to_bf16(a.x), E, R, workspace=ws, status=st)
    torch.cuda.synchronize()
    _assert_layout(oracle_mod, lay, a.topk_idx, E, R)
    L = oracle_mod.get_layout(a.topk_idx, E, R)
    ox, os_ = oracle_mod.dispatch_fp8(a.x, L.dst_pos, n * k)
    assert np.array_equal(rx.cpu().numpy(), ox)
    assert np.array_equal(rs.cpu().numpy().view(np.uint32), os_.view(np.uint32))
    assert st.item() == 0 and wl.num_experts == E


def test_bounded_wait_rejects_bad_arguments():
    f = _probe()
    assert f(None, 4, 1 << 16, None) == cgl.EINVAL
    assert f(1 << 16, 0, 1 << 16, None) == cgl.EINVAL
    assert f(1 << 16, 4097, 1 << 16, None) == cgl.EINVAL
    assert f((1 << 16) + 4, 4, 1 << 16, None) == cgl.EALIGN

"""cgl_get_layout_noalloc through the C ABI: same results as cgl_get_layout.

This entry point is for callers that cannot allocate device memory (hosts that
pass only pre-planned input/output buffers, callers that must avoid the
synchronisation of cudaFree, C-only callers without a CUDA allocator); its
scratch is a fixed device array inside libcgl.so, shared by all calls.  The
test runs several calls in a row on different inputs and shapes, so that each
sees whatever the one before left in that array, and compares each with
cgl_get_layout (the existing entry point, with a caller-allocated workspace)
bit for bit, the
tolerance for integer outputs, and with the CPU oracle.  It also checks that
sizes past the array's limit are refused before any launch.  The file sorts last so that a run that
stops at the first failure has already run everything else.
"""

import ctypes as C

import numpy as np
import pytest
import torch

import combine_get_layout_02_b200 as cgl
from combine_get_layout_02_b200 import workloads as W

pytestmark = pytest.mark.gpu

FIELDS = ("tokens_per_expert", "tokens_per_rank", "is_token_in_rank", "expert_offset", "max_count",
          "dst_pos", "recv_src")


def _fn():
    f = cgl.lib().cgl_get_layout_noalloc
    P, I64, I = C.c_void_p, C.c_int64, C.c_int
    f.argtypes = [P, I64, I, I, I, C.POINTER(cgl.Opts), P, P, P, P, P, P, P, P, P]
    f.restype = I
    return f


def _noalloc(idx: torch.Tensor, E: int, R: int, cap: int = 0):
    n, k = idx.shape
    dev = idx.device
    rows = E * cap if cap > 0 else n * k
    # poison every output so that a skipped write shows up
    out = {
        "tokens_per_expert": torch.full((E,), -7, dtype=torch.int32, device=dev),
        "tokens_per_rank": torch.full((R,), -7, dtype=torch.int32, device=dev),
        "is_token_in_rank": torch.full((n, R), 0xEE, dtype=torch.uint8, device=dev),
        "expert_offset": torch.full((E + 1,), -7, dtype=torch.int32, device=dev),
        "max_count": torch.full((1,), -7, dtype=torch.int32, device=dev),
        "dst_pos": torch.full((n, k), -7, dtype=torch.int32, device=dev),
        "recv_src": torch.full((rows,), -7, dtype=torch.int32, device=dev),
    }
    st = cgl.new_status(dev)
    code = _fn()(idx.data_ptr(), n, k, E, R, C.byref(cgl.Opts(0, cap)),
                 *[out[f].data_ptr() for f in FIELDS], st.data_ptr(),
                 torch.cuda.current_stream().cuda_stream)
    assert code == cgl.OK, cgl.lib().cgl_status_string(code)
    return out, st


def _reference(idx: torch.Tensor, E: int, R: int, cap: int = 0):
    st = cgl.new_status(idx.device)
    lay = cgl.get_layout(idx, E, R, cap, status=st)
    return {f: getattr(lay, f) for f in FIELDS}, st


def _oracle_check(oracle_mod, got, idx_np, E, R, cap):
    L = oracle_mod.get_layout(idx_np, E, R, cap)
    for f in FIELDS:
        if f == "max_count":
            assert int(got[f].item()) == L.max_count
            continue
        g, r = got[f].cpu().numpy(), getattr(L, f)
        assert g.shape == r.shape and np.array_equal(g, r), f
    return L


def test_noalloc_matches_oracle_and_get_layout_on_calls_in_a_row(oracle_mod):
    """Consecutive calls of different shapes share the scratch array: each later
    call runs on what the one before left in it (generation word, flags and count
    rows of another block count, E and R).  Calls above 32768 (token, slot) pairs
    exchange counts through the array (cooperative blocks); the prefill-sized
    and decode calls in between need no scratch and check that the array's
    contents do not matter to them.  Each output is compared bit for bit with
    the oracle and with cgl_get_layout."""
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    pre = W.make_inputs("prefill", 0)
    skw = W.make_inputs("skewed", 0)
    dec = W.make_inputs("decode", 0)
    s9 = np.ascontiguousarray(skw.topk_idx[:9000])
    cap_s9 = oracle_mod.get_layout(s9, 256, 64).max_count
    cap_dec = oracle_mod.get_layout(dec.topk_idx, 256, 32).max_count
    cases = [
        (skw.topk_idx, 256, 64, 0),             # 128 blocks of 128 tokens
        (skw.topk_idx, 256, 32, 0),             # same blocks, other R
        (s9, 256, 64, cap_s9 - 3),              # 71 blocks, padded, some experts overflow (CGL_ECAPACITY)
        (pre.topk_idx, 256, 64, 0),             # replicated counts: no scratch
        (dec.topk_idx, 256, 32, cap_dec),
        (skw.topk_idx[:5000], 256, 64, 0),      # 40 blocks
        (skw.topk_idx, 256, 64, 0),
    ]
    for idx_np, E, R, c in cases:
        idx_np = np.ascontiguousarray(idx_np)
        idx = torch.from_numpy(idx_np).to(dev)
        got, st = _noalloc(idx, E, R, c)
        ref, st_ref = _reference(idx, E, R, c)
        torch.cuda.synchronize()
        L = _oracle_check(oracle_mod, got, idx_np, E, R, c)
        for f in FIELDS:
            assert torch.equal(got[f], ref[f]), f
        bits = int(st.item())
        assert bits == int(st_ref.item())
        assert bool(bits & (1 << cgl.ECAPACITY)) == bool(L.flags & oracle_mod.FLAG_CAPACITY)
        assert not bits & ~(1 << cgl.ECAPACITY)


def test_noalloc_refuses_sizes_past_its_scratch():
    dev = torch.device("cuda", 0)
    fake = 1 << 16   # never dereferenced: the size check comes first
    f = _fn()
    args = [fake] * 7
    # 60000 tokens at E=256, R=64 need more than the 512 KiB scratch array
    assert cgl.layout_workspace_bytes(60000, 8, 256, 64) > 512 * 1024
    assert f(fake, 60000, 8, 256, 64, None, *args, None, None) == cgl.EINVAL
    # E=1024 with k=8 would need more than 48 KiB of shared memory per block
    assert f(fake, 100, 8, 1024, 64, None, *args, None, None) == cgl.EINVAL
    # within the limits the same fake pointers are only refused for alignment
    assert f(fake + 2, 100, 8, 256, 64, None, *args, None, None) == cgl.EALIGN

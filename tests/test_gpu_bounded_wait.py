"""Failure detection on the GPU without a fault: the layout's bounded inter-block
wait, run on flags that nothing sets, gives up after about a second, reports
CGL_ETIMEOUT in the status word, and leaves the context usable."""

import ctypes as C
import time

import numpy as np
import pytest
import torch

import combine_get_layout_02_b200 as cgl
from combine_get_layout_02_b200 import workloads as W

from helpers import dev, i32

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives(oracle_mod):
    f = cgl.lib().cgl_selftest_bounded_wait
    f.argtypes = [C.c_void_p, C.c_int, C.c_void_p, C.c_void_p]
    f.restype = C.c_int
    flags = torch.zeros(4, dtype=torch.int64, device=dev())
    st = cgl.new_status(dev())
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    assert f(flags.data_ptr(), 4, st.data_ptr(), torch.cuda.current_stream().cuda_stream) == cgl.OK
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert cgl.status_bits(st) == ["CGL_ETIMEOUT"]
    assert 0.3 < elapsed < 10.0
    # the device still works: a full layout afterwards matches the oracle
    inp = W.make_inputs("prefill", 7)
    lay = cgl.get_layout(i32(inp.topk_idx), 256, 64)
    ref = oracle_mod.get_layout(inp.topk_idx, 256, 64)
    assert np.array_equal(lay.dst_pos.cpu().numpy(), ref.dst_pos)


def test_bounded_wait_rejects_bad_arguments():
    f = cgl.lib().cgl_selftest_bounded_wait
    f.argtypes = [C.c_void_p, C.c_int, C.c_void_p, C.c_void_p]
    f.restype = C.c_int
    assert f(None, 4, 1 << 16, None) == cgl.EINVAL
    assert f(1 << 16, 0, 1 << 16, None) == cgl.EINVAL
    assert f((1 << 16) + 4, 4, 1 << 16, None) == cgl.EALIGN

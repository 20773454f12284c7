"""FP8 dispatch with power-of-two (UE8M0) scales (CGL_OPT_UE8M0_SCALES) against the
oracle's power-of-two path, bit for bit: codes and scales of every received row,
through every kernel that quantises (the bulk and the flattened dispatch
kernels, the fused layout + dispatch kernel and its fallback, the fused decode
kernel).  The oracle's scale rule is pinned in tests/test_oracle_pow2_scales.py."""

import numpy as np
import pytest
import torch

import combine_get_layout_02_b200 as cgl
from combine_get_layout_02_b200 import workloads as W

from helpers import dev, i32, to_bf16

pytestmark = pytest.mark.gpu


def _compare(oracle_mod, x, dst_pos, rows, rx, rs):
    ox, os_ = oracle_mod.dispatch_fp8(x, dst_pos, rows, pow2_scales=True)
    used = np.zeros(rows, bool)
    used[dst_pos[dst_pos >= 0]] = True
    gx, gs = rx.cpu().numpy(), rs.cpu().numpy()
    assert np.array_equal(gx[used], ox[used]), "codes"
    assert np.array_equal(gs[used].view(np.uint32), os_[used].view(np.uint32)), "scales"
    assert np.all(np.frexp(gs[used])[0] == 0.5)          # every scale is a power of two


def _magnitudes(n, h, seed):
    rng = np.random.default_rng(seed)
    exps = rng.uniform(-40, 120, (n, h // 128, 1))
    x32 = (rng.standard_normal((n, h // 128, 128)) * np.exp2(exps)).astype(np.float32)
    x32[rng.random((n, h // 128)) < 0.05] = 0.0
    return W.f32_to_bf16_bits(np.clip(x32, -3e38, 3e38).reshape(n, h))


@pytest.mark.parametrize("h", [7168, 16512])   # bulk kernel; flattened kernel above 16384
def test_dispatch_fp8_pow2(oracle_mod, h):
    n, k, E = 300, 8, 64
    x = _magnitudes(n, h, 1)
    rng = np.random.default_rng(2)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(n)]).astype(np.int32)
    idx[rng.random((n, k)) < 0.05] = -1
    L = oracle_mod.get_layout(idx, E, 8)
    rx, rs = cgl.dispatch_fp8(to_bf16(x), i32(L.dst_pos), n * k, pow2_scales=True)
    torch.cuda.synchronize()
    _compare(oracle_mod, x, L.dst_pos, n * k, rx, rs)


@pytest.mark.parametrize("num_sms", [0, 40])   # the fused kernel; 40 SMs: the layout + dispatch kernels
def test_layout_dispatch_fp8_pow2_prefill(oracle_mod, num_sms):
    inp = W.make_inputs("prefill", 6)
    wl = inp.workload
    st = cgl.new_status(dev())
    lay, rx, rs = cgl.layout_dispatch_fp8(i32(inp.topk_idx), to_bf16(inp.x), wl.num_experts, wl.num_ranks,
                                          status=st, num_sms=num_sms, pow2_scales=True)
    torch.cuda.synchronize()
    L = oracle_mod.get_layout(inp.topk_idx, wl.num_experts, wl.num_ranks)
    assert np.array_equal(lay.dst_pos.cpu().numpy(), L.dst_pos)
    _compare(oracle_mod, inp.x, L.dst_pos, inp.topk_idx.size, rx, rs)
    assert st.item() == 0


def test_layout_dispatch_fp8_pow2_magnitudes(oracle_mod):
    n, h, k, E, R = 2000, 1024, 8, 64, 8
    x = _magnitudes(n, h, 5)
    rng = np.random.default_rng(6)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(n)]).astype(np.int32)
    lay, rx, rs = cgl.layout_dispatch_fp8(i32(idx), to_bf16(x), E, R, pow2_scales=True)
    torch.cuda.synchronize()
    L = oracle_mod.get_layout(idx, E, R)
    assert np.array_equal(lay.dst_pos.cpu().numpy(), L.dst_pos)
    _compare(oracle_mod, x, L.dst_pos, n * k, rx, rs)


def test_decode_dispatch_fp8_pow2(oracle_mod):
    inp = W.make_inputs("decode", 3)
    cap = oracle_mod.get_layout(inp.topk_idx, 256, 32).max_count
    x = inp.x.copy()
    x[5] = _magnitudes(1, 7168, 7)[0]
    x[9] = 0
    lay, rx, rs = cgl.decode_dispatch_fp8(i32(inp.topk_idx), to_bf16(x), 256, 32, cap, pow2_scales=True)
    torch.cuda.synchronize()
    L = oracle_mod.get_layout(inp.topk_idx, 256, 32, cap)
    assert np.array_equal(lay.dst_pos.cpu().numpy(), L.dst_pos)
    _compare(oracle_mod, x, L.dst_pos, 256 * cap, rx, rs)

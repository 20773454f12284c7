"""GPU combine backward against the oracle through the C ABI.

grad_y must match bit for bit (one fp32 product, then RNE).  grad_w is an fp32
dot product whose summation order is the kernel's (fused multiply-adds per
thread, a fixed tree over the block); it must lie within 2^-14 * sum|g*y| of
the oracle's exact (double-accumulated) value: a few fp32 roundings over
H <= 16384 terms stay far below that, while a wrong row, slot or sign lands
far above it.
"""

import numpy as np
import pytest
import torch

import combine_get_layout_02_b200 as cgl
from combine_get_layout_02_b200 import workloads as W

from helpers import bits, dev, f32, i32, to_bf16

pytestmark = pytest.mark.gpu

GW_TOL = 2.0 ** -14


def _check(oracle_mod, g, y, dst, w, rows_used=None):
    st = cgl.new_status(dev())
    gy = torch.full((y.shape[0], y.shape[1]), 0x1357, dtype=torch.int16, device=dev()).view(torch.bfloat16)
    gy, gw = cgl.combine_backward(to_bf16(g), to_bf16(y), i32(dst), f32(w), grad_y=gy, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ogy, ogw = oracle_mod.combine_backward(g, y, dst, w)
    used = np.zeros(y.shape[0], bool)
    used[dst[dst >= 0]] = True
    got = bits(gy)
    assert np.array_equal(got[used], ogy[used]), "grad_y differs"
    assert np.all(got[~used] == 0x1357), "rows without a slot were written"
    ggw = gw.cpu().numpy()
    gf, yf = W.bf16_bits_to_f32(g).astype(np.float64), W.bf16_bits_to_f32(y).astype(np.float64)
    valid = dst >= 0
    mag = np.zeros_like(ggw, dtype=np.float64)
    tt, jj = np.nonzero(valid)
    mag[tt, jj] = np.einsum("ij,ij->i", np.abs(gf[tt]), np.abs(yf[dst[tt, jj]]))
    assert np.all(np.abs(ggw.astype(np.float64) - ogw.astype(np.float64)) <= GW_TOL * mag + 1e-30)
    assert np.all(ggw[~valid] == 0.0)
    return ggw


def test_backward_full_size_bf16_workload(oracle_mod):
    inp = W.make_inputs("bf16", 0)
    wl = inp.workload
    L = oracle_mod.get_layout(inp.topk_idx, wl.num_experts, wl.num_ranks)
    y = W.expert_outputs(inp.topk_idx.size, wl.hidden, 0)
    _check(oracle_mod, inp.grad, y, L.dst_pos, inp.topk_w)


def test_backward_ragged_shapes_and_masks(oracle_mod):
    rng = np.random.default_rng(13)
    for n, h, k, rows in [(1, 16, 1, 1), (7, 48, 3, 30), (300, 4112, 8, 2400), (37, 16384, 13, 500), (128, 7168, 8, 1024)]:
        g = W.f32_to_bf16_bits(rng.standard_normal((n, h)).astype(np.float32))
        y = W.f32_to_bf16_bits(rng.standard_normal((rows, h)).astype(np.float32) * 2)
        # a layout maps slots to distinct rows (each grad_y row has one writer)
        dst = rng.permutation(rows)[: n * k].reshape(n, k).astype(np.int32)
        dst[rng.random((n, k)) < 0.15] = -1
        w = rng.standard_normal((n, k)).astype(np.float32)
        _check(oracle_mod, g, y, dst, w)


def test_backward_closed_forms():
    n, h, k = 256, 7168, 8
    rng = np.random.default_rng(14)
    idx = np.stack([rng.permutation(256)[:k] for _ in range(n)]).astype(np.int32)
    lay = cgl.get_layout(i32(idx), 256, 64)
    g = torch.randn((n, h), device=dev()).bfloat16()
    y = torch.randn((n * k, h), device=dev()).bfloat16()
    gy, gw = cgl.combine_backward(g, y, lay.dst_pos, torch.ones((n, k), device=dev()))
    assert torch.equal(gy[lay.dst_pos.flatten().long()].view(n, k, h), g[:, None, :].expand(n, k, h))
    cols = torch.from_numpy(rng.integers(0, h, n)).to(dev())
    onehot = torch.zeros((n, h), device=dev()).bfloat16()
    onehot[torch.arange(n, device=dev()), cols] = 1.0
    _, gw1 = cgl.combine_backward(onehot, y, lay.dst_pos, torch.ones((n, k), device=dev()))
    expect = y[lay.dst_pos.long(), cols[:, None]].float()
    assert torch.equal(gw1, expect)   # one nonzero term: exact


def test_backward_reports_rows_outside_the_buffer():
    g = torch.zeros((1, 32), dtype=torch.bfloat16, device=dev())
    y = torch.zeros((4, 32), dtype=torch.bfloat16, device=dev())
    st = cgl.new_status(dev())
    _, gw = cgl.combine_backward(g, y, i32(np.array([[1, 9]], np.int32)), torch.ones((1, 2), device=dev()), status=st)
    torch.cuda.synchronize()
    assert cgl.status_bits(st) == ["CGL_ERANGE"] and gw[0, 1].item() == 0.0

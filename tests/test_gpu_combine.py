"""GPU combine against the oracle through the C ABI: within 2^-7 relative error
per element (the contract) and, since both sides use the same operation order,
bit for bit; plus the closed-form identities."""

import numpy as np
import pytest
import torch

import combine_get_layout_02_b200 as cgl
from combine_get_layout_02_b200 import workloads as W

from helpers import COMBINE_TOL, bits, dev, f32, i32, max_rel_err, to_bf16

pytestmark = pytest.mark.gpu


def _combine_case(oracle_mod, y, dst, w, num_sms=0):
    st = cgl.new_status(dev())
    out = cgl.combine(to_bf16(y), i32(dst), f32(w), status=st, num_sms=num_sms)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    got = bits(out)
    ref = oracle_mod.combine(y, dst, w)
    assert max_rel_err(got, ref) <= COMBINE_TOL
    assert np.array_equal(got, ref), f"not bit-exact at {np.argwhere(got != ref)[:5].tolist()}"
    return got


@pytest.mark.parametrize("name", W.WORKLOAD_ORDER)
def test_combine_full_size(oracle_mod, name):
    inp = W.make_inputs(name, 0)
    wl = inp.workload
    L = oracle_mod.get_layout(inp.topk_idx, wl.num_experts, wl.num_ranks)
    y = W.expert_outputs(inp.topk_idx.size, wl.hidden, 0)
    _combine_case(oracle_mod, y, L.dst_pos, inp.topk_w)


def test_combine_padded_decode(oracle_mod):
    inp = W.make_inputs("decode", 0)
    wl = inp.workload
    cap = oracle_mod.get_layout(inp.topk_idx, 256, 32).max_count
    L = oracle_mod.get_layout(inp.topk_idx, 256, 32, cap)
    y = W.expert_outputs(256 * cap, wl.hidden, 1)
    _combine_case(oracle_mod, y, L.dst_pos, inp.topk_w)


def test_combine_masked_ragged_and_large_k(oracle_mod):
    rng = np.random.default_rng(3)
    for n, h, k, rows in [(1, 8, 1, 1), (5, 24, 3, 15), (999, 7168, 8, 7992), (300, 512, 32, 9600), (77, 128, 13, 1001)]:
        y = W.f32_to_bf16_bits(rng.standard_normal((rows, h)).astype(np.float32) * 3)
        dst = rng.integers(0, rows, (n, k)).astype(np.int32)
        dst[rng.random((n, k)) < 0.15] = -1
        w = rng.random((n, k)).astype(np.float32)
        _combine_case(oracle_mod, y, dst, w)


def test_combine_sm_cap(oracle_mod):
    inp = W.make_inputs("prefill", 2, num_tokens=512)
    L = oracle_mod.get_layout(inp.topk_idx, 256, 64)
    y = W.expert_outputs(inp.topk_idx.size, 7168, 2)
    _combine_case(oracle_mod, y, L.dst_pos, inp.topk_w, num_sms=3)


def test_combine_of_unweighted_fp8_dispatch_of_ones_is_k():
    n, h, k = 512, 7168, 8
    rng = np.random.default_rng(0)
    idx = np.stack([rng.permutation(256)[:k] for _ in range(n)]).astype(np.int32)
    lay = cgl.get_layout(i32(idx), 256, 64)
    x = torch.ones((n, h), dtype=torch.bfloat16, device=dev())
    rx, rs = cgl.dispatch_fp8(x, lay.dst_pos, lay.num_recv_rows)
    assert torch.all(rx == 0x7E)
    # identity experts: dequantise (448 * fl(1/448) == 1 exactly), then combine with unit weights
    y = (rx.view(torch.float8_e4m3fn).float().view(-1, h // 128, 128) * rs[:, :, None]).view(-1, h).bfloat16()
    out = cgl.combine(y, lay.dst_pos, torch.ones((n, k), dtype=torch.float32, device=dev()))
    assert torch.all(out.float() == k)


def test_bf16_round_trip_identities():
    n, h, k = 1000, 7168, 8
    rng = np.random.default_rng(1)
    idx = np.stack([rng.permutation(256)[:k] for _ in range(n)]).astype(np.int32)
    lay = cgl.get_layout(i32(idx), 256, 64)
    x = torch.randn((n, h), device=dev()).bfloat16()
    recv = cgl.dispatch_bf16(x, lay.dst_pos, lay.num_recv_rows)
    ones = torch.ones((n, k), dtype=torch.float32, device=dev())
    assert torch.equal(cgl.combine(recv, lay.dst_pos, ones), (x.float() * k).bfloat16())
    onehot = torch.zeros((n, k), dtype=torch.float32, device=dev())
    onehot[torch.arange(n), torch.from_numpy(rng.integers(0, k, n)).to(dev())] = 1.0
    assert torch.equal(cgl.combine(recv, lay.dst_pos, onehot), x)


def test_fp8_round_trip_within_fp8_bound():
    inp = W.make_inputs("prefill", 0)
    lay = cgl.get_layout(i32(inp.topk_idx), 256, 64)
    x = to_bf16(inp.x)
    rx, rs = cgl.dispatch_fp8(x, lay.dst_pos, lay.num_recv_rows)
    y = (rx.view(torch.float8_e4m3fn).float().view(-1, 56, 128) * rs[:, :, None]).view(-1, 7168).bfloat16()
    out = cgl.combine(y, lay.dst_pos, f32(inp.topk_w)).float()
    xf = x.float()
    # |out - x| <= (2^-4 e4m3 + 2^-8 bf16 + 2^-8 bf16) |x| + subnormal floor of the block scale
    scale = rs[lay.dst_pos[:, 0].long()].repeat_interleave(128, dim=1)
    bound = (2 ** -4 + 2 ** -7 + 2 ** -6) * xf.abs() + scale * 2 ** -9
    assert torch.all((out - xf).abs() <= bound)


def test_combine_reports_rows_outside_the_buffer():
    y = torch.zeros((8, 64), dtype=torch.bfloat16, device=dev())
    st = cgl.new_status(dev())
    cgl.combine(y, i32(np.array([[0, 8]], np.int32)), torch.ones((1, 2), device=dev()), status=st)
    torch.cuda.synchronize()
    assert cgl.status_bits(st) == ["CGL_ERANGE"]

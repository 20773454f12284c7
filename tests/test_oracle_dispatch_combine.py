"""Pins for the oracle's FP8 / BF16 dispatch and its combine.

Closed forms and bounds fixed by the arithmetic, not by re-typing the oracle:
  * x == 1 gives code 0x7E (448) and scale fl(1/448), and 448 * fl(1/448) == 1;
  * each block's largest |x| encodes as +-448; dequantisation error <= 2^-4 |x|
    in the normal range, <= scale * 2^-10 in the subnormal range;
  * an all-zero block has scale fl(1e-4 / 448) and zero codes;
  * combine of an unweighted dispatch of ones equals k; combine of a BF16
    dispatch with unit weights equals k*x bit for bit; one-hot weights give x;
    a masked slot equals a zero weight; random cases stay within the fp32
    summation bound of the exact (fp64) weighted sum plus one BF16 rounding.
"""

import numpy as np
import pytest

from combine_get_layout_02_b200 import workloads as W

f32 = np.float32


def _layout(oracle_mod, inp, cap=0):
    wl = inp.workload
    return oracle_mod.get_layout(inp.topk_idx, wl.num_experts, wl.num_ranks, cap)


def _dequant(oracle_mod, rx, rs):
    """BF16 bits of decode(q) * scale per block (test-side expert stand-in)."""
    v = oracle_mod.e4m3_decode(rx).reshape(rx.shape[0], -1, 128) * rs[:, :, None]
    return W.f32_to_bf16_bits(v.reshape(rx.shape).astype(f32))


def test_fp8_dispatch_of_ones_and_combine_gives_k(oracle_mod):
    for name in ("tiny", "prefill"):
        inp = W.make_inputs(name, 0, num_tokens=64)
        wl = inp.workload
        x = np.full((64, wl.hidden), 0x3F80, np.uint16)   # BF16 1.0
        L = _layout(oracle_mod, inp)
        M = inp.topk_idx.size
        rx, rs = oracle_mod.dispatch_fp8(x, L.dst_pos, M)
        assert np.all(rx == 0x7E)
        assert np.all(rs == f32(1.0) / f32(448.0))
        assert f32(448.0) * (f32(1.0) / f32(448.0)) == f32(1.0)
        y = _dequant(oracle_mod, rx, rs)
        assert np.all(y == 0x3F80)
        out = oracle_mod.combine(y, L.dst_pos, np.ones_like(inp.topk_w))
        assert np.all(W.bf16_bits_to_f32(out) == wl.topk)


@pytest.mark.parametrize("name", ["tiny", "prefill"])
def test_fp8_dispatch_block_properties(oracle_mod, name):
    inp = W.make_inputs(name, 0, num_tokens=256 if name == "prefill" else None)
    wl = inp.workload
    x = inp.x.copy()
    x[3, :128] = 0                                          # an all-zero block
    L = _layout(oracle_mod, inp)
    M = inp.topk_idx.size
    rx, rs = oracle_mod.dispatch_fp8(x, L.dst_pos, M)
    n, h = x.shape
    B = h // 128
    # every copy of token t is identical; every row got exactly one copy
    for t in range(n):
        rows = L.dst_pos[t]
        assert np.all(rx[rows] == rx[rows[0]]) and np.all(rs[rows] == rs[rows[0]])
    q = rx[L.dst_pos[:, 0]].reshape(n, B, 128)
    s = rs[L.dst_pos[:, 0]]
    xf = W.bf16_bits_to_f32(x).reshape(n, B, 128)
    amax = np.abs(xf).max(axis=2)
    zero = amax == 0
    assert np.all(s[zero] == f32(1e-4) / f32(448.0)) and np.all(q[zero] == 0)
    nz = ~zero
    # scale * 448 reproduces amax to within one fp32 rounding
    assert np.all(np.abs(s[nz].astype(np.float64) * 448 - amax[nz]) <= amax[nz] * 2.0 ** -23)
    # the block maximum encodes as +-448
    am = np.abs(xf).argmax(axis=2)
    top = np.take_along_axis(q, am[:, :, None], axis=2)[:, :, 0]
    assert np.all((top[nz] & 0x7F) == 0x7E)
    # dequantisation error
    deq = oracle_mod.e4m3_decode(q).astype(np.float64) * s[:, :, None]
    err = np.abs(deq - xf)
    scaled = np.abs(xf) / s[:, :, None]
    normal = scaled >= 2.0 ** -6
    assert np.all(err[normal] <= np.abs(xf[normal]) * 2.0 ** -4 * (1 + 2.0 ** -20))
    sub = ~normal
    assert np.all(err[sub] <= (np.broadcast_to(s[:, :, None], err.shape)[sub] * 2.0 ** -10) * (1 + 2.0 ** -20))
    # signs survive (zero keeps its sign bit)
    assert np.all((q >> 7) == (np.signbit(xf)).astype(np.uint8))


def test_prefill_hot_rows_scale_with_the_row(oracle_mod):
    inp = W.make_inputs("prefill", 0)
    hot = inp.hot_rows[:4]
    idx = inp.topk_idx[hot]
    sub = oracle_mod.get_layout(idx, 256, 64)
    rx, rs = oracle_mod.dispatch_fp8(inp.x[hot], sub.dst_pos, idx.size)
    assert rs.min() > 0.1   # x100 rows: amax ~ 100s -> scales ~ 0.5
    assert len(inp.hot_rows) == 41


def test_bf16_dispatch_copies_and_unit_weight_combine_is_kx(oracle_mod):
    for name in ("tiny", "bf16"):
        inp = W.make_inputs(name, 0, num_tokens=96)
        wl = inp.workload
        L = _layout(oracle_mod, inp)
        M = inp.topk_idx.size
        recv = oracle_mod.dispatch_bf16(inp.x, L.dst_pos, M)
        assert np.array_equal(recv[L.dst_pos], np.repeat(inp.x[:, None, :], wl.topk, axis=1))
        out = oracle_mod.combine(recv, L.dst_pos, np.ones_like(inp.topk_w))
        kx = W.bf16_bits_to_f32(inp.x) * f32(wl.topk)     # exact: k is a power of two
        assert np.array_equal(out, W.f32_to_bf16_bits(kx))
        assert np.array_equal(W.bf16_bits_to_f32(out), kx)


def test_one_hot_weights_return_x(oracle_mod):
    inp = W.make_inputs("tiny", 0)
    wl = inp.workload
    L = _layout(oracle_mod, inp)
    recv = oracle_mod.dispatch_bf16(inp.x, L.dst_pos, inp.topk_idx.size)
    rng = np.random.default_rng(0)
    w = np.zeros_like(inp.topk_w)
    w[np.arange(wl.num_tokens), rng.integers(0, wl.topk, wl.num_tokens)] = 1.0
    assert np.array_equal(oracle_mod.combine(recv, L.dst_pos, w), inp.x)


def test_masked_slot_equals_zero_weight(oracle_mod):
    inp = W.make_inputs("tiny", 1)
    wl = inp.workload
    idx = inp.topk_idx.copy()
    rng = np.random.default_rng(5)
    drop = rng.random(idx.shape) < 0.3
    idx[drop] = -1
    L = oracle_mod.get_layout(idx, wl.num_experts, wl.num_ranks)
    Lfull = oracle_mod.get_layout(inp.topk_idx, wl.num_experts, wl.num_ranks)
    y = W.expert_outputs(idx.size, wl.hidden, 3)
    # same expert output per (t, j) for both layouts
    y_masked = np.zeros_like(y)
    keep = L.dst_pos >= 0
    y_masked[L.dst_pos[keep]] = y[Lfull.dst_pos[keep]]
    w0 = np.where(drop, 0.0, inp.topk_w).astype(f32)
    a = oracle_mod.combine(y_masked, L.dst_pos, inp.topk_w)
    b = oracle_mod.combine(y, Lfull.dst_pos, w0)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("name", ["tiny", "decode", "prefill"])
def test_combine_within_bound_of_exact_sum(oracle_mod, name):
    inp = W.make_inputs(name, 0, num_tokens=128)
    wl = inp.workload
    L = _layout(oracle_mod, inp)
    M = inp.topk_idx.size
    y = W.expert_outputs(M, wl.hidden, 11)
    out = W.bf16_bits_to_f32(oracle_mod.combine(y, L.dst_pos, inp.topk_w)).astype(np.float64)
    terms = inp.topk_w.astype(np.float64)[:, :, None] * W.bf16_bits_to_f32(y)[L.dst_pos].astype(np.float64)
    exact = terms.sum(axis=1)
    mag = np.abs(terms).sum(axis=1)
    k = wl.topk
    bound = 2.0 ** -8 * np.abs(exact) + (k + 1) * 2.0 ** -24 * mag * (1 + 2.0 ** -8)
    assert np.all(np.abs(out - exact) <= bound)
    # a dropped term, sign flip or swapped slot shows up well beyond the bound
    wrong = terms[:, 1:, :].sum(axis=1)
    assert np.mean(np.abs(out - wrong) > bound) > 0.9

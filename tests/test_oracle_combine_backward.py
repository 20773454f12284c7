"""Pins for the oracle's combine backward (grad of the expert outputs and of the weights).

grad_y = bf16(w * g): checked against torch's own float32 product and bfloat16
rounding; w == 1 must copy g bit for bit.  grad_w = <g, y>: one-hot g picks a
single element of y exactly; all-ones g and y give H; an exact rational sum
(Python fractions) on a small case; and the derivative of the forward oracle
by finite differences along w.
"""

from fractions import Fraction

import numpy as np
import torch

from combine_get_layout_02_b200 import workloads as W


def _case(seed=0, n=64, h=256, E=16, R=4, k=4):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(n)]).astype(np.int32)
    idx[rng.random((n, k)) < 0.1] = -1
    w = rng.random((n, k)).astype(np.float32)
    g = W.f32_to_bf16_bits(rng.standard_normal((n, h)).astype(np.float32))
    y = W.f32_to_bf16_bits(rng.standard_normal((n * k, h)).astype(np.float32))
    return idx, w, g, y


def test_grad_y_matches_torch_product_and_rounding(oracle_mod):
    idx, w, g, y = _case()
    L = oracle_mod.get_layout(idx, 16, 4)
    gy, gw = oracle_mod.combine_backward(g, y, L.dst_pos, w)
    gt = torch.from_numpy(W.bf16_bits_to_f32(g))
    for t in range(idx.shape[0]):
        for j in range(idx.shape[1]):
            row = L.dst_pos[t, j]
            if row < 0:
                assert gw[t, j] == 0.0
                continue
            ref = (torch.tensor(w[t, j], dtype=torch.float32) * gt[t]).to(torch.bfloat16)
            assert np.array_equal(gy[row], ref.view(torch.int16).numpy().view(np.uint16))
    assert np.all(gy[L.recv_src < 0] == 0)


def test_unit_weight_copies_g(oracle_mod):
    idx, w, g, y = _case(1)
    L = oracle_mod.get_layout(idx, 16, 4)
    gy, _ = oracle_mod.combine_backward(g, y, L.dst_pos, np.ones_like(w))
    used = L.dst_pos >= 0
    assert np.array_equal(gy[L.dst_pos[used]], np.repeat(g[:, None, :], 4, axis=1)[used])


def test_grad_w_closed_forms(oracle_mod):
    n, h, k = 8, 128, 2
    idx = np.array([[0, 1]] * n, np.int32)
    L = oracle_mod.get_layout(idx, 2, 1)
    rng = np.random.default_rng(2)
    y = W.f32_to_bf16_bits(rng.standard_normal((n * k, h)).astype(np.float32))
    g = np.zeros((n, h), np.uint16)
    cols = rng.integers(0, h, n)
    g[np.arange(n), cols] = 0x3F80                      # one-hot ones
    _, gw = oracle_mod.combine_backward(g, y, L.dst_pos, np.ones((n, k), np.float32))
    yf = W.bf16_bits_to_f32(y)
    assert np.array_equal(gw, yf[L.dst_pos, cols[:, None]])
    ones = np.full((n, h), 0x3F80, np.uint16)
    _, gw1 = oracle_mod.combine_backward(ones, np.full((n * k, h), 0x3F80, np.uint16), L.dst_pos,
                                         np.ones((n, k), np.float32))
    assert np.all(gw1 == h)


def test_grad_w_exact_rational_sum(oracle_mod):
    idx, w, g, y = _case(3, n=6, h=96)
    L = oracle_mod.get_layout(idx, 16, 4)
    _, gw = oracle_mod.combine_backward(g, y, L.dst_pos, w)
    gf, yf = W.bf16_bits_to_f32(g), W.bf16_bits_to_f32(y)
    for t in range(6):
        for j in range(4):
            row = L.dst_pos[t, j]
            if row < 0:
                continue
            exact = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(gf[t], yf[row]))
            assert gw[t, j] == np.float32(float(exact))   # one rounding of the exact value


def test_grad_w_is_the_derivative_of_the_forward(oracle_mod):
    # d out / d w[t, j] = y_j, so <g, d out / d w> = <g, y_j>; checked with the
    # forward oracle in float64 terms: f(w) = <g, sum_j w_j y_j> is linear in w
    idx, w, g, y = _case(4, n=16, h=128)
    L = oracle_mod.get_layout(idx, 16, 4)
    _, gw = oracle_mod.combine_backward(g, y, L.dst_pos, w)
    gf, yf = W.bf16_bits_to_f32(g).astype(np.float64), W.bf16_bits_to_f32(y).astype(np.float64)
    for t in range(16):
        def f(wt):
            acc = np.zeros(128)
            for j in range(4):
                if L.dst_pos[t, j] >= 0:
                    acc += wt[j] * yf[L.dst_pos[t, j]]
            return float(gf[t] @ acc)
        for j in range(4):
            e = np.zeros(4)
            e[j] = 1.0
            d = f(w[t].astype(np.float64) + e) - f(w[t].astype(np.float64))
            assert abs(d - gw[t, j]) <= 1e-6 * (1 + abs(d))

"""Pins of the oracle's FP8 dispatch with power-of-two (UE8M0) scales.

Definition (the reading this library takes for the power-of-two variant of
FP8 dispatch, "原生FP8 调度支持" in the DeepEP key-technique list of brainleap
"Day2 DeepEP"): per 128-value block, amax_c = max(max |x|, 1e-4); scale = 2^e
for the smallest integer e with 448 * 2^e >= amax_c; inv = 2^-e;
q = e4m3(x * inv).  Checked against closed forms at exact powers of two, the
exact rational exponent on random blocks, and the properties the definition
implies (no saturation, minimal exponent, FP8 error bound).
"""

import math
from fractions import Fraction

import numpy as np

from combine_get_layout_02_b200 import workloads as W


def _bf16(vals):
    return W.f32_to_bf16_bits(np.asarray(vals, np.float32))


def _one_block(oracle_mod, x_bits):
    x = np.asarray(x_bits, np.uint16).reshape(1, 128)
    rx, rs = oracle_mod.dispatch_fp8(x, np.zeros((1, 1), np.int32), 1, pow2_scales=True)
    return rx[0], float(rs[0, 0])


def _exact_exponent(amax_c: float) -> int:
    """Smallest integer e with 448 * 2^e >= amax_c, in exact rational arithmetic."""
    q = Fraction(amax_c) / 448
    e = q.numerator.bit_length() - q.denominator.bit_length()
    while Fraction(2) ** e < q:
        e += 1
    while Fraction(2) ** (e - 1) >= q:
        e -= 1
    return e


def test_block_max_at_448_times_a_power_of_two(oracle_mod):
    # amax = 448 * 2^j exactly (1.75 * 2^(8+j) is a BF16 value): scale = 2^j and
    # the block maximum maps to 448 exactly (code 0x7E), its negative to 0xFE
    for j in (-20, -7, -1, 0, 1, 5, 30, 100):
        vals = np.zeros(128, np.float32)
        vals[3] = 448.0 * 2.0 ** j
        vals[77] = -448.0 * 2.0 ** j
        vals[10] = 224.0 * 2.0 ** j      # exactly half the maximum: 224 = e4m3 code 0x76
        rx, scale = _one_block(oracle_mod, _bf16(vals))
        assert scale == 2.0 ** j
        assert rx[3] == 0x7E and rx[77] == 0xFE and rx[10] == 0x76
        assert np.all(rx[[i for i in range(128) if i not in (3, 10, 77)]] == 0)


def test_just_above_a_power_the_scale_doubles(oracle_mod):
    # the next BF16 value above 448 * 2^j is 1.7578125 * 2^(8+j): 448 * 2^j no
    # longer covers it, so scale = 2^(j+1) and the maximum maps to 225 -> e4m3 224
    for j in (-3, 0, 4):
        v = 1.7578125 * 2.0 ** (8 + j)
        rx, scale = _one_block(oracle_mod, _bf16([v] + [0.0] * 127))
        assert scale == 2.0 ** (j + 1)
        assert oracle_mod.e4m3_decode(np.array([rx[0]], np.uint8))[0] == 224.0


def test_zero_block_takes_the_floor_exponent(oracle_mod):
    # amax_c = 1e-4: 448 * 2^-22 = 1.068e-4 >= 1e-4 > 448 * 2^-23 = 5.34e-5
    rx, scale = _one_block(oracle_mod, np.zeros(128, np.uint16))
    assert scale == 2.0 ** -22
    assert np.all(rx == 0)


def test_exponent_equals_exact_rational_search_across_magnitudes(oracle_mod):
    rng = np.random.default_rng(3)
    n, h = 64, 1024
    exps = rng.uniform(-40, 120, (n, h // 128, 1))
    x32 = (rng.standard_normal((n, h // 128, 128)) * np.exp2(exps)).astype(np.float32)
    x32[rng.random((n, h // 128)) < 0.05] = 0.0
    x = _bf16(np.clip(x32, -3e38, 3e38).reshape(n, h))
    idx = np.arange(n, dtype=np.int32).reshape(n, 1)
    rx, rs = oracle_mod.dispatch_fp8(x, idx, n, pow2_scales=True)
    xf = (x.astype(np.uint32) << 16).view(np.float32).reshape(n, h // 128, 128)
    amax_c = np.maximum(np.abs(xf).max(axis=2), np.float32(1e-4))
    for t in range(n):
        for b in range(h // 128):
            e = _exact_exponent(float(amax_c[t, b]))
            assert rs[t, b] == 2.0 ** e, (t, b)


def test_no_saturation_minimal_exponent_and_error_bound(oracle_mod):
    inp = W.make_inputs("prefill", 0, num_tokens=200)
    x = inp.x
    n, h = x.shape
    idx = np.arange(n, dtype=np.int32).reshape(n, 1)
    rx, rs = oracle_mod.dispatch_fp8(x, idx, n, pow2_scales=True)
    rx_ieee, rs_ieee = oracle_mod.dispatch_fp8(x, idx, n)
    xf = (x.astype(np.uint32) << 16).view(np.float32).reshape(n, h // 128, 128).astype(np.float64)
    dec = oracle_mod.e4m3_decode(rx.reshape(-1)).astype(np.float64).reshape(n, h // 128, 128)
    sc = rs.astype(np.float64)[:, :, None]
    amax_c = np.maximum(np.abs(xf).max(axis=2), 1e-4)
    # the scale is a power of two, covers the block, and is the smallest that does
    assert np.all(np.frexp(rs)[0] == 0.5)
    assert np.all(448.0 * rs >= amax_c) and np.all(224.0 * rs < amax_c)
    # nothing saturates: every decoded code is within +-448, and the largest is >= 224
    assert np.all(np.abs(dec) <= 448.0)
    big = amax_c > 1e-4
    assert np.all(np.abs(dec).max(axis=2)[big] >= 224.0)
    # FP8 E4M3 (3 mantissa bits) round to nearest: relative error <= 2^-4 in the normal range
    recon = dec * sc
    normal = np.abs(xf / sc) >= 2.0 ** -6
    assert np.all(np.abs(recon - xf)[normal] <= 2.0 ** -4 * np.abs(xf)[normal])
    # against the IEEE-division scale: never smaller, at most twice as large
    assert np.all(rs >= rs_ieee) and np.all(rs <= 2 * rs_ieee)
    assert math.isfinite(float(rs.max()))

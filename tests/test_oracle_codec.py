"""Pins for the oracle's number formats: E4M3 encode/decode and BF16 rounding.

The oracle's codecs are written from the OCP FP8 and bfloat16 definitions; these
tests pin them to torch's own float8_e4m3fn / bfloat16 conversions (a library
routine the oracle does not call) and to the OCP anchor values.
"""

import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_ocp_anchors.txt")


def _torch_e4m3(v: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(v, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_decode_all_256_codes_match_torch(oracle_mod):
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle_mod.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert nan.sum() == 2 and nan[0x7F] and nan[0xFF]
    assert np.array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))  # signed zeros too


def test_decode_ocp_anchor_values(oracle_mod):
    rows = [l.split() for l in open(GOLDEN) if l.strip() and not l.startswith("#")]
    assert len(rows) >= 10
    for code_hex, val in rows:
        got = float(oracle_mod.e4m3_decode(np.array([int(code_hex, 16)], np.uint8))[0])
        if val == "nan":
            assert math.isnan(got), code_hex
        else:
            assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val)), code_hex


def test_encode_every_bf16_in_range_matches_torch(oracle_mod):
    bits = np.arange(65536, dtype=np.uint32) << np.uint32(16)
    v = bits.view(np.float32)
    v = v[np.isfinite(v) & (np.abs(v) <= 464.0)]
    assert np.array_equal(oracle_mod.e4m3_encode(v), _torch_e4m3(v))


def test_encode_random_fp32_matches_torch(oracle_mod):
    g = np.random.default_rng(7)
    mag = np.exp2(g.uniform(-14, np.log2(464.0), 400_000)).astype(np.float32)
    v = (mag * g.choice([-1, 1], mag.size)).astype(np.float32)
    v = v[np.abs(v) <= 464.0]
    assert np.array_equal(oracle_mod.e4m3_encode(v), _torch_e4m3(v))


def test_encode_ties_go_to_even(oracle_mod):
    # midpoints between adjacent finite codes (exactly representable in fp32),
    # and the fp32 neighbours on either side of each midpoint
    vals = oracle_mod.e4m3_decode(np.arange(0x00, 0x7F, dtype=np.uint8)).astype(np.float64)
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    below = np.nextafter(mids, np.float32(0))
    above = np.nextafter(mids, np.float32(np.inf))
    lo_code = np.arange(0x00, 0x7E, dtype=np.uint8)
    even = np.where(lo_code % 2 == 0, lo_code, lo_code + 1).astype(np.uint8)
    assert np.array_equal(oracle_mod.e4m3_encode(mids), even)
    assert np.array_equal(oracle_mod.e4m3_encode(below), lo_code)
    assert np.array_equal(oracle_mod.e4m3_encode(above), (lo_code + 1).astype(np.uint8))
    assert np.array_equal(oracle_mod.e4m3_encode(-mids), even | 0x80)
    assert np.array_equal(oracle_mod.e4m3_encode(np.concatenate([mids, below, above])),
                          _torch_e4m3(np.concatenate([mids, below, above])))


def test_encode_saturates_and_keeps_specials(oracle_mod):
    big = np.array([448.0, 449.0, 463.99, 464.0, 464.01, 480.0, 1e4, 3e38, np.inf], np.float32)
    assert np.all(oracle_mod.e4m3_encode(big) == 0x7E)
    assert np.all(oracle_mod.e4m3_encode(-big) == 0xFE)
    assert oracle_mod.e4m3_encode(np.array([np.nan], np.float32))[0] & 0x7F == 0x7F
    z = oracle_mod.e4m3_encode(np.array([0.0, -0.0, 1e-30, -1e-30, 2.0 ** -10, 2.0 ** -10 * 1.0001], np.float32))
    # 2^-10 is half the smallest subnormal: ties to even -> 0; just above -> 1
    assert list(z) == [0x00, 0x80, 0x00, 0x80, 0x00, 0x01]


def test_encode_decode_round_trip_all_finite_codes(oracle_mod):
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    assert np.array_equal(oracle_mod.e4m3_encode(oracle_mod.e4m3_decode(codes)), codes)


def test_bf16_rounding_matches_torch(oracle_mod):
    g = np.random.default_rng(3)
    u = g.integers(0, 2 ** 32, 500_000, dtype=np.uint64).astype(np.uint32)
    v = u.view(np.float32)
    v = v[np.isfinite(v)]
    # exact ties: low 16 bits == 0x8000, with both parities of the kept part
    ties = ((g.integers(0, 2 ** 16, 2000).astype(np.uint32) << 16) | 0x8000).view(np.float32)
    ties = ties[np.isfinite(ties)]
    v = np.concatenate([v, ties, np.array([0.0, -0.0, 1.0, -1.0, 3.3895314e38], np.float32)])
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle_mod.bf16_from_f32(v), ref)

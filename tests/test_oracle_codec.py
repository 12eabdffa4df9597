"""Pins for the oracle's E4M3 and BF16 codecs.

The OCP 8-bit floating point specification fixes E4M3: exponent bias 7, three
mantissa bits, no infinities, NaN = S.1111.111, largest finite 448, smallest
normal 2^-6, subnormal step 2^-9.  The encoder is checked against a
brute-force nearest-value search over the decoded table (ties to the even
code) and against torch's float8_e4m3fn cast where that cast is defined by
the same rule (|x| below the rounding threshold 464; torch does not saturate).
"""

import math

import numpy as np
import pytest
import torch

import oracle


def test_decode_table_spec_values():
    d = oracle.e4m3_decode(np.arange(256))
    assert d[0x00] == 0.0 and math.copysign(1.0, d[0x80]) == -1.0
    assert d[0x01] == 2.0 ** -9 and d[0x07] == 7 * 2.0 ** -9
    assert d[0x08] == 2.0 ** -6
    assert d[0x38] == 1.0
    assert d[0x7E] == 448.0 and d[0xFE] == -448.0
    assert math.isnan(d[0x7F]) and math.isnan(d[0xFF])
    assert d[0x78] == 256.0 and d[0x77] == 240.0
    pos = d[:0x7F]
    assert np.all(np.diff(pos) > 0)                      # monotone finite codes
    assert np.array_equal(d[0x80:0xFF], -pos)


def _brute_force_codes(x):
    """Nearest finite E4M3 value by search; ties to the code with even LSB;
    saturate beyond 448.  Independent of the oracle's encoder."""
    table = oracle.e4m3_decode(np.arange(0x7F))         # +0 .. 448
    out = []
    for v in x:
        a = abs(float(v))
        if a >= 448.0:
            c = 0x7E
        else:
            dist = np.abs(table - a)
            best = np.flatnonzero(dist == dist.min())
            c = int(best[0]) if len(best) == 1 else int([b for b in best if b % 2 == 0][0])
        if math.copysign(1.0, float(v)) < 0:
            c |= 0x80
        out.append(c)
    return np.array(out, dtype=np.uint8)


def test_encoder_ties_and_neighbours_brute_force():
    table = oracle.e4m3_decode(np.arange(0x7F))
    mids = (table[:-1] + table[1:]) / 2.0               # exact in float32
    pts = []
    for m in mids.astype(np.float32):
        pts += [m, np.nextafter(m, np.float32(0)), np.nextafter(m, np.float32(1000))]
    pts += list(table.astype(np.float32))
    pts += [np.float32(449.0), np.float32(463.99), np.float32(464.0), np.float32(1e30),
            np.float32(np.inf)]
    pts = np.array(pts, dtype=np.float32)
    pts = np.concatenate([pts, -pts])
    assert np.array_equal(oracle.e4m3_encode(pts), _brute_force_codes(pts))


def test_encoder_random_brute_force():
    rng = np.random.default_rng(1)
    x = (np.exp(rng.uniform(-14, 7, 20000)) * rng.choice([-1, 1], 20000)).astype(np.float32)
    assert np.array_equal(oracle.e4m3_encode(x), _brute_force_codes(x))


def test_encoder_matches_torch_in_range():
    rng = np.random.default_rng(2)
    x = (np.exp(rng.uniform(-16, 6.1, 1 << 20)) * rng.choice([-1, 1], 1 << 20)).astype(np.float32)
    x = x[np.abs(x) < 464.0]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(x), ref)


def test_bf16_round_matches_torch_for_float32_inputs():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal(1 << 18) * np.exp(rng.uniform(-20, 20, 1 << 18))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.bf16_round(x.astype(np.float64)), ref)


def test_bf16_round_binary64_single_rounding():
    # a binary64 value a hair above a BF16 midpoint rounds up; a float32 detour
    # would land exactly on the midpoint and round to even (down).
    mid = (1.0 + 1.0078125) / 2.0
    assert oracle.bf16_round(np.array([mid]))[0] == 0x3F80
    assert oracle.bf16_round(np.array([mid + 2.0 ** -40]))[0] == 0x3F81
    assert oracle.bf16_round(np.array([-mid - 2.0 ** -40]))[0] == 0xBF81
    assert oracle.bf16_round(np.array([0.0, -0.0])).tolist() == [0x0000, 0x8000]

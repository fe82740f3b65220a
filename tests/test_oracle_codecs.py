"""Pins of the oracle's code formats against things other than itself.

* e2m1 / e4m3 / e8m0 values against the format specifications' tables
  (tests/golden, each file cites its source).
* e4m3 encode/decode against torch's float8_e4m3fn conversion (a library
  routine), over every code and over random fp32 inputs in range.
* e2m1 encode against a brute-force nearest-value search with ties to even.
* exhaustive round trips and monotonicity.
"""
import math
import os

import numpy as np
import pytest
import torch

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _read(name):
    rows = []
    for line in open(os.path.join(GOLD, name)):
        line = line.strip()
        if line and not line.startswith("#"):
            rows.append(line)
    return rows


def _same(a, b):
    if math.isnan(a) or math.isnan(b):
        return math.isnan(a) and math.isnan(b)
    return a == b and math.copysign(1.0, a) == math.copysign(1.0, b)


E2M1_GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def brute_e2m1(v: float) -> int:
    """Nearest e2m1 magnitude; on a tie the candidate whose mantissa bit is 0."""
    a = abs(v)
    best = None
    for code, m in enumerate(E2M1_GRID):
        d = abs(a - m)
        if best is None or d < best[0] or (d == best[0] and (code & 1) == 0):
            best = (d, code)
    sign = 8 if math.copysign(1.0, v) < 0 else 0
    return sign | best[1]


def test_e2m1_values_match_spec(orc):
    for row in _read("e2m1_values.txt"):
        c, v = row.split()
        assert _same(orc.e2m1_decode(int(c, 16)), float(v)), row


def test_e2m1_rounding_golden(orc):
    for row in _read("e2m1_rounding.txt"):
        v, c = row.split()
        assert orc.e2m1_encode(float(v)) == int(c, 16), row


def test_e2m1_encode_matches_brute_force(orc):
    rng = np.random.default_rng(1)
    vals = list(rng.uniform(-8, 8, 4000).astype(np.float32))
    vals += [m + d for m in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0) for d in (-1e-6, 0.0, 1e-6)]
    vals += [-x for x in vals[-21:]]
    for v in vals:
        v = float(np.float32(v))
        assert orc.e2m1_encode(v) == brute_e2m1(v), v


def test_e2m1_round_trip_all_codes(orc):
    for c in range(16):
        assert orc.e2m1_encode(orc.e2m1_decode(c)) == c


def test_e4m3_points_match_spec(orc):
    for row in _read("e4m3_points.txt"):
        c, v = row.split()
        assert _same(orc.e4m3_decode(int(c, 16)), float(v)), row


def test_e4m3_decode_matches_torch_all_codes(orc):
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).float().tolist()
    for c in range(256):
        assert _same(orc.e4m3_decode(c), ref[c]), hex(c)


def test_e4m3_encode_matches_torch_in_range(orc):
    rng = np.random.default_rng(2)
    v = np.concatenate([
        rng.uniform(-464, 464, 3000), rng.normal(0, 1, 3000), rng.normal(0, 0.01, 2000),
        rng.uniform(-2 ** -6, 2 ** -6, 2000),
    ]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([orc.e4m3_encode(float(x)) for x in v], dtype=np.uint8)
    assert np.array_equal(got, ref)


def test_e4m3_saturates_instead_of_nan(orc):
    for v in (465.0, 1e6, float(np.finfo(np.float32).max)):
        assert orc.e4m3_encode(v) == 0x7E
        assert orc.e4m3_encode(-v) == 0xFE


def test_e4m3_round_trip_and_monotone(orc):
    prev = -1.0
    for c in range(0x7F):
        v = orc.e4m3_decode(c)
        assert v > prev or c == 0
        prev = v
        assert orc.e4m3_encode(v) == c
        assert orc.e4m3_encode(-v) == (c | 0x80)


def test_e8m0_points_match_spec(orc):
    for row in _read("e8m0_points.txt"):
        c, v = row.split()
        assert _same(orc.e8m0_decode(int(c)), float(v)), row
    for c in range(255):
        assert orc.e8m0_decode(c) == math.ldexp(1.0, c - 127)


def test_format_maxima(orc):
    assert max(orc.e2m1_decode(c) for c in range(16)) == 6.0
    finite = [orc.e4m3_decode(c) for c in range(256) if not math.isnan(orc.e4m3_decode(c))]
    assert max(finite) == 448.0 and min(finite) == -448.0
    assert orc.e8m0_decode(254) == 2.0 ** 127


def test_bf16_rounding_matches_torch(orc):
    """fp32 -> bf16 round-to-nearest-even against torch's conversion: random
    values over the whole range, exact ties both ways, subnormals, overflow to
    infinity; NaN stays NaN."""
    rng = np.random.default_rng(11)
    bits = rng.integers(0, 2 ** 32, 20000, dtype=np.uint64).astype(np.uint32)
    ties = (rng.integers(0, 2 ** 16, 2000, dtype=np.uint32) << 16) | 0x8000
    edge = np.array([0x7F7FFFFF, 0x7F7F8000, 0x00000001, 0x80008000, 0x3F808000, 0x3F818000, 0xFF7FFFFF],
                    np.uint32)
    u = np.concatenate([bits, ties, edge])
    f = u.view(np.float32)
    ours = np.ascontiguousarray(orc.quant_bf16(f.reshape(1, -1))).view(np.uint16).reshape(-1)
    ref = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    nan = np.isnan(f)
    assert np.array_equal(ours[~nan], ref[~nan])
    ob = (ours[nan].astype(np.uint32) << 16).view(np.float32)
    assert np.all(np.isnan(ob))
    # decoding the codes gives the bf16 values exactly
    d = orc.dequant(4, orc.quant_bf16(f[~nan].reshape(1, -1)), None, 1.0, 1, int((~nan).sum()))
    assert np.array_equal(d.reshape(-1), (ref[~nan].astype(np.uint32) << 16).view(np.float32).astype(np.float64))

"""Pins of the oracle's block quantisers.

* worked examples computed by hand from the definitions (tests/golden);
* a brute-force re-derivation of every scale and code on random blocks, using
  nearest-value search over all codes instead of the oracle's rounding
  arithmetic (the fp32 operation sequence is the definition and is shared);
* the per-tensor FP8 quantiser against torch's float8_e4m3fn conversion;
* reconstruction bounds and degenerate blocks (zero, saturating).
"""
import math
import os

import numpy as np
import torch

GOLD = os.path.join(os.path.dirname(__file__), "golden")
E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _rows(name):
    for line in open(os.path.join(GOLD, name)):
        line = line.strip()
        if line and not line.startswith("#"):
            yield [f.strip() for f in line.split("|")]


def _nearest_e2m1(v):
    a = abs(v)
    best = min(range(8), key=lambda c: (abs(a - E2M1[c]), c & 1))
    return (8 if math.copysign(1, v) < 0 else 0) | best


def _e4m3_values():
    return torch.arange(0x7F, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().numpy()


def _nearest_e4m3_pos(s):
    vals = _e4m3_values()
    if s >= vals[-1]:
        return 0x7E
    d = np.abs(vals - s)
    m = d.min()
    cands = [c for c in range(0x7F) if d[c] == m]
    even = [c for c in cands if (c & 1) == 0]
    return (even or cands)[0]


def _unpack(codes_row, K):
    out = []
    for i in range(K):
        b = int(codes_row[i // 2])
        out.append((b >> (4 * (i % 2))) & 15)
    return out


def test_nvfp4_golden_blocks(orc):
    for g, xs, sc, qs in _rows("nvfp4_blocks.txt"):
        x = np.array([float(v) for v in xs.split()], np.float32)[None, :]
        codes, sf = orc.quant_nvfp4(x, float(g))
        assert int(sf[0, 0]) == int(sc, 16), (g, xs)
        assert _unpack(codes[0], 16) == [int(q, 16) for q in qs.split()], (g, xs)


def test_mxfp4_golden_blocks(orc):
    for xs, sc, qs in _rows("mxfp4_blocks.txt"):
        vals = [float(v) for v in xs.split()]
        x = np.zeros((1, 32), np.float32)
        x[0, :len(vals)] = vals
        codes, sf = orc.quant_mxfp4(x)
        assert int(sf[0, 0]) == int(sc), xs
        assert _unpack(codes[0], 32)[:len(vals)] == [int(q, 16) for q in qs.split()], xs


def test_nvfp4_matches_brute_force(orc):
    rng = np.random.default_rng(3)
    rows, K = 24, 64
    x = (rng.standard_normal((rows, K)) * rng.uniform(0.01, 5, (rows, 1))).astype(np.float32)
    x[3, 16:32] = 0.0
    g = np.float32(orc.nvfp4_global_scale(orc.amax(x)))
    codes, sf = orc.quant_nvfp4(x, float(g))
    for r in range(rows):
        q = _unpack(codes[r], K)
        for b in range(K // 16):
            blk = x[r, b * 16:(b + 1) * 16]
            bmax = np.float32(np.abs(blk).max())
            s = np.float32(bmax / np.float32(np.float32(6.0) * g))
            sc = _nearest_e4m3_pos(float(s))
            assert int(sf[r, b]) == sc
            dec = np.float32(_e4m3_values()[sc])
            for i in range(16):
                if dec == 0:
                    assert q[b * 16 + i] == 0
                else:
                    rcp = np.float32(np.float32(1.0) / np.float32(dec * g))
                    assert q[b * 16 + i] == _nearest_e2m1(float(np.float32(blk[i] * rcp)))


def test_mxfp4_matches_brute_force(orc):
    rng = np.random.default_rng(4)
    rows, K = 16, 128
    x = (rng.standard_normal((rows, K)) * rng.uniform(1e-3, 50, (rows, 1))).astype(np.float32)
    x[5, 32:64] = 0.0
    codes, sf = orc.quant_mxfp4(x)
    for r in range(rows):
        q = _unpack(codes[r], K)
        for b in range(K // 32):
            blk = x[r, b * 32:(b + 1) * 32]
            bmax = float(np.abs(blk).max())
            if bmax == 0:
                c = 0
            else:
                m, e = math.frexp(bmax)
                c = min(max(e - 1 - 2 + 127, 0), 254)
            assert int(sf[r, b]) == c
            for i in range(32):
                v = float(np.float32(blk[i] * np.float32(2.0 ** (127 - c))))
                assert q[b * 32 + i] == _nearest_e2m1(v)


def test_fp8_matches_torch(orc):
    rng = np.random.default_rng(5)
    x = rng.standard_normal(5000).astype(np.float32) * 3
    a = orc.amax(x)
    assert a == float(np.abs(x).max())
    s = orc.fp8_scale(a)
    assert s == float(np.float32(np.float32(a) / np.float32(448.0)))
    codes = orc.quant_fp8(x, s)
    inv = np.float32(np.float32(1.0) / np.float32(s))
    ref = torch.from_numpy((x * inv).astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes, ref)


def test_reconstruction_bounds(orc):
    rng = np.random.default_rng(6)
    x = rng.standard_normal((8, 256)).astype(np.float32)
    g = orc.nvfp4_global_scale(orc.amax(x))
    c, s = orc.quant_nvfp4(x, g)
    d = orc.dequant(orc.FMT_NVFP4, c, s, g, 8, 256)
    for r in range(8):
        for b in range(16):
            blk = x[r, b * 16:(b + 1) * 16].astype(np.float64)
            db = d[r, b * 16:(b + 1) * 16]
            step = float(orc.e4m3_decode(int(s[r, b]))) * g
            # e2m1 spacing is at most 2 units of the block scale
            assert np.all(np.abs(db - blk) <= 1.0 * step + 1e-12)
            assert np.abs(db).max() <= np.abs(blk).max() * (1 + 2 ** -3) + 1e-12
    c2, s2 = orc.quant_mxfp4(x)
    d2 = orc.dequant(orc.FMT_MXFP4, c2, s2, 1.0, 8, 256)
    for r in range(8):
        for b in range(8):
            blk = x[r, b * 32:(b + 1) * 32].astype(np.float64)
            step = float(orc.e8m0_decode(int(s2[r, b])))
            err = np.abs(d2[r, b * 32:(b + 1) * 32] - blk)
            # inside the grid: half the local spacing (<= 1 unit); the
            # saturated top (values in (6, 8) units) loses at most 2 units
            assert np.all(err <= 2.0 * step + 1e-12)


def test_dequant_nibble_and_scale_layout(orc):
    # byte 0x21: element 0 = code 1 (0.5), element 1 = code 2 (1.0); the second
    # byte 0xF7: element 2 = code 7 (6), element 3 = code 15 (-6).  Block 0 of
    # row 0 has scale 0x38 (1.0); row 1's scale 0x30 (0.5).
    codes = np.zeros((2, 8), np.uint8)
    codes[0, 0], codes[0, 1] = 0x21, 0xF7
    codes[1, 0] = 0x21
    sf = np.array([[0x38], [0x30]], np.uint8)
    d = orc.dequant(orc.FMT_NVFP4, codes, sf, 2.0, 2, 16)
    assert list(d[0, :4]) == [1.0, 2.0, 12.0, -12.0]
    assert list(d[1, :2]) == [0.5, 1.0]
    d2 = orc.dequant(orc.FMT_MXFP4, np.pad(codes, ((0, 0), (0, 8))), np.array([[128], [126]], np.uint8), 1.0, 2, 32)
    assert list(d2[0, :4]) == [1.0, 2.0, 12.0, -12.0]
    assert list(d2[1, :2]) == [0.25, 0.5]
    d3 = orc.dequant(orc.FMT_FP8, np.array([[0x38, 0xB8, 0x7E]], np.uint8), None, 0.5, 1, 3)
    assert list(d3[0]) == [0.5, -0.5, 224.0]


def test_zero_tensor_scales(orc):
    assert orc.nvfp4_global_scale(0.0) == 1.0
    assert orc.fp8_scale(0.0) == 1.0
    c, s = orc.quant_nvfp4(np.zeros((1, 16), np.float32), 1.0)
    assert not c.any() and not s.any()

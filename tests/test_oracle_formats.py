"""Pins of the oracle's number formats against things other than the oracle.

References used: the OCP MX v1.0 E2M1 value table (tests/golden/e2m1_values.txt),
torch's float8_e4m3fn / float8_e8m0fnu / bfloat16 conversions, numpy's float16,
brute-force nearest-value search, and hand-built blocks whose decoded values
follow from the documented bit layouts.
"""
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def golden_e2m1():
    vals = {}
    with open(os.path.join(GOLDEN, "e2m1_values.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            c, v = line.split()
            vals[int(c)] = float(v)
    return vals


E2M1 = golden_e2m1()
E2M1_NP = np.array([E2M1[c] for c in range(16)])


# ---- element formats -------------------------------------------------------

def test_e2m1_exhaustive_decode(ora):
    for c in range(16):
        v = ora.e2m1_value(c)
        assert v == E2M1[c] and math.copysign(1, v) == math.copysign(1, E2M1[c]), c


def test_e2m1_encode_matches_nearest_on_grid_and_ties(ora):
    # every tie point between neighbours, and a dense grid around them
    mags = sorted(set(abs(v) for v in E2M1.values()))
    ties = [(a + b) / 2 for a, b in zip(mags, mags[1:])]
    grid = np.concatenate([np.linspace(0, 8, 4001), ties, [6.0, 7.0, 100.0, 1e30]])
    for y in grid:
        for s in (1.0, -1.0):
            assert ora.e2m1_encode(s * y) == ora.e2m1_encode_nearest(s * y), (s * y)
    # ties go to the even mantissa (code with lsb 0)
    for t in ties:
        assert ora.e2m1_encode(t) & 1 == 0, t
    # saturation and signed zero
    assert ora.e2m1_encode(6.5) == 7 and ora.e2m1_encode(-1e9) == 15
    assert ora.e2m1_encode(-0.0) == 8 and ora.e2m1_encode(-0.1) == 8 and ora.e2m1_encode(0.1) == 0


def test_e2m1_nearest_is_nearest(ora):
    rng = np.random.default_rng(1)
    for y in rng.uniform(-7, 7, 3000):
        c = ora.e2m1_encode_nearest(y)
        err = abs(y - E2M1[c])
        assert err <= np.min(np.abs(y - E2M1_NP)) + 0.0, y


def test_e8m0_decode_vs_torch(ora):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e8m0fnu).double().numpy()
    for e in range(256):
        v = ora.e8m0_value(e)
        if e == 255:
            assert math.isnan(v) and math.isnan(ref[e])
        else:
            assert v == ref[e] == 2.0 ** (e - 127), e


def test_e4m3_exhaustive_decode_vs_torch(ora):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).double().numpy()
    for c in range(256):
        v = ora.e4m3_value(c)
        if math.isnan(ref[c]):
            assert math.isnan(v), c
        else:
            assert v == ref[c] and math.copysign(1, v) == math.copysign(1, ref[c]), c


def test_e4m3_all_codes_roundtrip(ora):
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            continue  # NaN
        assert ora.e4m3_encode(ora.e4m3_value(c)) == c, c


def test_e4m3_encode_vs_torch_and_nearest(ora):
    rng = np.random.default_rng(2)
    ys = np.concatenate([
        rng.normal(0, 1, 2000), rng.normal(0, 100, 2000), rng.uniform(-2**-6, 2**-6, 2000),
        # midpoints between consecutive codes (ties)
        [(ora.e4m3_value(c) + ora.e4m3_value(c + 1)) / 2 for c in range(0, 0x7E)],
    ]).astype(np.float32)
    ref = torch.from_numpy(ys).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for y, r in zip(ys, ref):
        c = ora.e4m3_encode(float(y))
        assert c == ora.e4m3_encode_nearest(float(y)), y
        if abs(y) <= 448:
            assert c == r, (y, c, r)
    # saturation (torch turns these into NaN; the MX conversion clamps)
    assert ora.e4m3_encode(449.0) == 0x7E and ora.e4m3_encode(-1e6) == 0xFE
    assert ora.e4m3_encode(-0.0) == 0x80


def test_f16_vs_numpy(ora):
    allc = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = allc.view(np.float16).astype(np.float64)
    for h in range(0, 65536, 7):
        v = ora.f16_value(h)
        assert (math.isnan(v) and math.isnan(ref[h])) or v == ref[h], h
    rng = np.random.default_rng(3)
    xs = np.concatenate([rng.normal(0, 1e-3, 3000), rng.normal(0, 1e3, 3000),
                         rng.uniform(-7e-5, 7e-5, 3000), [65504, 65519.99, 65520, 1e9, 2**-25, 3 * 2**-26]])
    xs = xs.astype(np.float32)
    ref = xs.astype(np.float16).view(np.uint16)
    for x, r in zip(xs, ref):
        assert ora.f32_to_f16(float(x)) == r, x


def test_bf16_vs_torch(ora):
    rng = np.random.default_rng(4)
    xs = np.concatenate([rng.normal(0, 1, 5000), rng.normal(0, 1e-30, 1000),
                         rng.uniform(-1e-38, 1e-38, 1000)]).astype(np.float32)
    ref = torch.from_numpy(xs).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    for x, r in zip(xs, ref):
        assert ora.f64_to_bf16(float(x)) == r, x
        assert ora.bf16_value(int(r)) == float(torch.tensor([int(r)], dtype=torch.int32)
                                               .to(torch.int16).view(torch.bfloat16).float())


# ---- MXFP4 blocks ----------------------------------------------------------

def np_decode_mxfp4(codes, scales):
    lo, hi = codes & 15, codes >> 4
    c = np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)
    return E2M1_NP[c] * np.repeat(np.exp2(scales.astype(np.float64) - 127), 32, axis=1)


def test_mxfp4_dequantize_vs_numpy_decode(ora):
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 256, (16, 64), dtype=np.uint8)
    scales = rng.integers(100, 140, (16, 4), dtype=np.uint8)
    out = ora.mxfp4_dequantize(codes, scales)
    np.testing.assert_array_equal(out.astype(np.float64), np_decode_mxfp4(codes, scales))


def test_mxfp4_roundtrip_exact_blocks(ora):
    """encode(decode(b)) == b when the block's largest |code| is 4 or 6."""
    rng = np.random.default_rng(6)
    rows, K = 64, 256
    codes = rng.integers(0, 256, (rows, K // 2), dtype=np.uint8)
    # force one element of every block to magnitude code 6 or 7 (value 4 or 6)
    for r in range(rows):
        for b in range(K // 32):
            codes[r, b * 16] = (codes[r, b * 16] & 0xF0) | rng.choice([6, 7, 14, 15])
    scales = rng.integers(1, 253, (rows, K // 32), dtype=np.uint8)  # 6*2^(s-127) fits fp32
    w = np_decode_mxfp4(codes, scales).astype(np.float32)
    c2, s2 = ora.mxfp4_quantize(w)
    np.testing.assert_array_equal(s2, scales)
    np.testing.assert_array_equal(c2, codes)


def test_mxfp4_error_bound_and_scale_rule(ora, syn):
    w = syn.normal_f32(0, 99, 0, 128 * 512, 0.0, 0.02).reshape(128, 512)
    w[3, :32] = 0.0          # all-zero block
    w[4, 32:64] *= 1e-3      # small block
    codes, scales = ora.mxfp4_quantize(w)
    wd = np_decode_mxfp4(codes, scales)
    X = np.repeat(np.exp2(scales.astype(np.float64) - 127), 32, axis=1)
    y = np.abs(w.astype(np.float64)) / X
    assert scales[3, 0] == 127 and not codes[3, :16].any()
    # the largest element of every nonzero block lands in [4, 8) after scaling
    bmax = y.reshape(128, -1, 32).max(axis=2)
    nz = bmax > 0
    assert np.all((bmax[nz] >= 4) & (bmax[nz] < 8))
    # half-ulp bound for unsaturated elements; saturated ones decode to +-6 X
    ulp = np.where(y < 2, 0.5, np.where(y < 4, 1.0, 2.0))
    err = np.abs(w - wd) / X
    sat = y > 6
    assert np.all(err[~sat] <= ulp[~sat] / 2)
    assert np.all(np.abs(wd[sat]) == 6 * X[sat])


# ---- MXFP8 blocks ----------------------------------------------------------

def test_mxfp8_quantize_vs_torch(ora, syn):
    x = syn.normal_bf16(0, 98, 0, 32 * 256).reshape(32, 256)
    x[0, :32] = 0
    codes, scales = ora.mxfp8_quantize_bf16(x)
    xf = torch.from_numpy(x.astype(np.int16)).view(torch.bfloat16).double().numpy()
    blk = np.abs(xf).reshape(32, -1, 32).max(axis=2)
    for r in range(32):
        for b in range(8):
            if blk[r, b] == 0:
                assert scales[r, b] == 127 and not codes[r, b * 32:(b + 1) * 32].any()
                continue
            se = int(scales[r, b]) - 127
            y = xf[r, b * 32:(b + 1) * 32] / 2.0 ** se
            assert 256 <= np.abs(y).max() < 512
            ys = np.clip(y, -448, 448).astype(np.float32)  # MX conversion saturates
            ref = torch.from_numpy(ys).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            np.testing.assert_array_equal(codes[r, b * 32:(b + 1) * 32], ref)
    back = ora.mxfp8_dequantize(codes, scales)
    X = np.repeat(np.exp2(scales.astype(np.float64) - 127), 32, axis=1)
    y = np.abs(xf) / X
    rel = np.abs(back - xf) / np.maximum(np.abs(xf), 1e-30)
    # normal-range, unsaturated elements: within half an ulp (2^-4 relative)
    keep = (y >= 2**-6) & (y <= 448)
    assert np.all(rel[keep] <= 2**-4)
    assert np.all(np.abs(back[y > 448]) == 448 * X[y > 448])


# ---- Q2_K super-blocks -----------------------------------------------------

def build_q2k_block(d16, dmin16, sc, m, q):
    """Bytes of one super-block laid out as documented in the oracle."""
    b = np.zeros(84, np.uint8)
    b[:16] = (sc | (m << 4)).astype(np.uint8)
    for n in range(256):
        b[16 + n // 4] |= np.uint8(q[n] << (2 * (n % 4)))
    b[80:82] = np.frombuffer(np.uint16(d16).tobytes(), np.uint8)
    b[82:84] = np.frombuffer(np.uint16(dmin16).tobytes(), np.uint8)
    return b


def test_q2k_decode_hand_built_blocks(ora):
    rng = np.random.default_rng(7)
    blocks, refs = [], []
    for _ in range(32):
        d = np.float16(rng.uniform(1e-4, 1e-2))
        dmin = np.float16(rng.uniform(0, 1e-2))
        sc = rng.integers(0, 16, 16)
        m = rng.integers(0, 16, 16)
        q = rng.integers(0, 4, 256)
        blocks.append(build_q2k_block(d.view(np.uint16), dmin.view(np.uint16), sc, m, q))
        # w = d*sc*q - dmin*m: products exact, one rounding to fp32
        w = (float(d) * np.repeat(sc, 16) * q - float(dmin) * np.repeat(m, 16)).astype(np.float32)
        refs.append(w)
    blocks = np.stack(blocks).reshape(32, 84)
    out = ora.q2k_dequantize(blocks, 256)
    np.testing.assert_array_equal(out, np.stack(refs))


def test_q2k_roundtrip_bound(ora, syn):
    w = syn.normal_f32(0, 97, 0, 64 * 512, 0.0, 0.02).reshape(64, 512)
    blocks = ora.q2k_quantize(w)
    wd = ora.q2k_dequantize(blocks, 512)
    for r in range(64):
        for sb in range(2):
            blk = blocks[r, sb * 84:(sb + 1) * 84]
            d = float(np.frombuffer(blk[80:82].tobytes(), np.float16)[0])
            dmin = float(np.frombuffer(blk[82:84].tobytes(), np.float16)[0])
            # d and dmin follow the documented max-range / 15 rule
            seg = w[r, sb * 256:(sb + 1) * 256].reshape(16, 16)
            mn = np.maximum(0, -seg.min(axis=1))
            rng_ = (seg.max(axis=1) + mn) / 3
            assert d == float(np.float16(np.float32(rng_.max()) / np.float32(15)))
            assert dmin == float(np.float16(np.float32(mn.max()) / np.float32(15)))
            for i in range(16):
                sc, m = int(blk[i] & 15), int(blk[i] >> 4)
                lo, hi = -dmin * m, d * sc * 3 - dmin * m
                x = seg[i].astype(np.float64)
                xd = wd[r, sb * 256 + 16 * i: sb * 256 + 16 * i + 16].astype(np.float64)
                inside = (x >= lo) & (x <= hi)
                # inside the grid's range: within half a step (+ rounding slack)
                assert np.all(np.abs(x - xd)[inside] <= 0.5 * d * sc * (1 + 1e-5) + 1e-7)
                # the grid covers the sub-block up to the 4-bit rounding of sc and m
                assert np.all(np.abs(x - xd) <= 0.5 * d * sc + d * 1.5 + dmin * 0.5 + 1e-7)

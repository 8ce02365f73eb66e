"""Pins of the oracle's expert FFN, shared expert, combine and layer.

The central pin is the dense-FFN equivalence: expert weights are drawn as
MXFP4 (or Q2_K) codes, decoded here in numpy from the format tables, and a
plain dense SwiGLU FFN written independently below must reproduce the
oracle's MoE outputs. A dropped term, a swapped gate/up operand, a transposed
matrix or a wrong scale shows up as an O(1) relative error.
"""
import os

import numpy as np
import pytest
import torch

from test_oracle_formats import E2M1_NP, build_q2k_block


def bf16_vals(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).astype(np.int16)).view(torch.bfloat16).double().numpy()


def to_bf16(v):
    """Round float64 values to bf16 (through fp32, torch's conversion)."""
    return torch.from_numpy(np.asarray(v, np.float64)).float().to(torch.bfloat16).double().numpy()


def mxfp8_roundtrip(v):
    """MX FP8 (E4M3) quantise-dequantise along the last axis, 32-blocks, via torch."""
    v = np.asarray(v, np.float64)
    blk = v.reshape(*v.shape[:-1], -1, 32)
    amax = np.abs(blk).max(axis=-1, keepdims=True)
    e = np.frexp(np.where(amax > 0, amax, 1.0))[1] - 1 - 8
    X = np.exp2(np.clip(e, -127, 127))
    y = np.clip(blk / X, -448, 448).astype(np.float32)
    q = torch.from_numpy(y).to(torch.float8_e4m3fn).double().numpy()
    return (q * X).reshape(v.shape)


E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])  # OCP MX v1.0 E2M1 magnitudes, codes 0..7


def mxfp4_roundtrip(v):
    """MX FP4 (E2M1) quantise-dequantise along the last axis, 32-blocks, by
    brute force over the format's eight magnitudes: the nearest one, a tie to
    the even code (mantissa bit 0), values past 6 to 6; scale 2^(floor(log2
    amax) - 2) as for the weights."""
    v = np.asarray(v, np.float64)
    blk = v.reshape(*v.shape[:-1], -1, 32)
    amax = np.abs(blk).max(axis=-1, keepdims=True)
    e = np.frexp(np.where(amax > 0, amax, 1.0))[1] - 1 - 2
    X = np.exp2(np.clip(e, -127, 127))
    y = blk / X
    dist = np.abs(np.abs(y)[..., None] - E2M1_MAG)
    best = dist == dist.min(axis=-1, keepdims=True)
    even = best & (np.arange(8) % 2 == 0)
    pick = np.where(even.any(axis=-1), np.argmax(even, axis=-1), np.argmax(best, axis=-1))
    q = np.where(amax > 0, np.sign(y) * E2M1_MAG[pick], 0.0)
    return (q * X).reshape(v.shape)


def silu(g):
    return g / (1 + np.exp(-g))


def dense_ffn(a, W1, W3, W2, act="bf16"):
    roundtrip = {"mxfp8": mxfp8_roundtrip, "mxfp4": mxfp4_roundtrip}.get(act)
    if roundtrip:
        a = roundtrip(a)
    g, u = W1 @ a, W3 @ a
    h = silu(g) * u
    h = roundtrip(h) if roundtrip else to_bf16(h)
    return W2 @ h


def random_mxfp4(rng, E, rows, K, scale_lo=118, scale_hi=124):
    codes = rng.integers(0, 256, (E, rows, K // 2), dtype=np.uint8)
    scales = rng.integers(scale_lo, scale_hi, (E, rows, K // 32), dtype=np.uint8)
    lo, hi = codes & 15, codes >> 4
    c = np.stack([lo, hi], axis=-1).reshape(E, rows, K)
    vals = E2M1_NP[c] * np.repeat(np.exp2(scales.astype(np.float64) - 127), 32, axis=2)
    return codes, scales, vals


def make_layer(ora, cfg, rng, shared=False):
    c1, s1, W1 = random_mxfp4(rng, cfg.E, cfg.F, cfg.d)
    c3, s3, W3 = random_mxfp4(rng, cfg.E, cfg.F, cfg.d)
    c2, s2, W2 = random_mxfp4(rng, cfg.E, cfg.d, cfg.F)
    kw = {}
    if shared:
        sh = [rng.normal(0, 0.05, shp).astype(np.float32) for shp in
              ((cfg.Fs, cfg.d), (cfg.Fs, cfg.d), (cfg.d, cfg.Fs))]
        kw = {n: torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
              for n, a in zip(("sw1", "sw3", "sw2"), sh)}
    wr = torch.from_numpy(rng.normal(0, 0.1, (cfg.E, cfg.d)).astype(np.float32)).to(
        torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    L = ora.LayerWeights(cfg, c1, s1, c3, s3, c2, s2, wr=wr, **kw)
    return L, (W1, W3, W2)


def rand_x(rng, T, d):
    return torch.from_numpy(rng.normal(0, 1, (T, d)).astype(np.float32)).to(
        torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("act", ["bf16", "mxfp8", "mxfp4"])
def test_dense_equivalence_single_expert(ora, syn, act):
    """E = 1, k = 1: the MoE layer is exactly one dense SwiGLU FFN."""
    cfg = syn.LayerConfig("t", T=3, d=256, F=512, E=1, k=1, act=act)
    rng = np.random.default_rng(20)
    L, (W1, W3, W2) = make_layer(ora, cfg, rng)
    x = rand_x(rng, 3, cfg.d)
    idx, w, y = ora.layer_tokens(L, x, np.arange(3))
    assert np.all(idx == 0) and np.all(w == 1.0)
    for t in range(3):
        ref = dense_ffn(bf16_vals(x[t]), W1[0], W3[0], W2[0], act)
        tol = {"bf16": 1e-4, "mxfp8": 3e-3, "mxfp4": 1e-6}[act] * np.abs(ref).max()
        np.testing.assert_allclose(y[t], ref, rtol=0, atol=tol)
        o = ora.expert_ffn_token(L, 0, x[t])
        np.testing.assert_allclose(o, ref, rtol=0, atol=tol)


def test_dense_equivalence_moe_with_shared(ora, syn):
    """General MoE: y = sum_j w_j FFN_{e_j}(x) + shared(x)."""
    cfg = syn.LayerConfig("t", T=5, d=256, F=256, E=6, k=3, Fs=128)
    rng = np.random.default_rng(21)
    L, (W1, W3, W2) = make_layer(ora, cfg, rng, shared=True)
    x = rand_x(rng, 5, cfg.d)
    idx, w, y = ora.layer_tokens(L, x, np.arange(5))
    # the routing is the oracle's own top-k of its own logits
    idx2, w2 = ora.topk_softmax(ora.router_logits(x, L.wr), 3)
    np.testing.assert_array_equal(idx, idx2)
    np.testing.assert_array_equal(w, w2)
    S1, S3, S2 = (bf16_vals(a) for a in (L.sw1, L.sw3, L.sw2))
    for t in range(5):
        a = bf16_vals(x[t])
        ref = sum(float(w[t, j]) * dense_ffn(a, W1[idx[t, j]], W3[idx[t, j]], W2[idx[t, j]])
                  for j in range(3))
        ref = ref + S2 @ to_bf16(silu(S1 @ a) * (S3 @ a))
        np.testing.assert_allclose(y[t], ref, rtol=0, atol=1e-4 * np.abs(ref).max())


def np_decode_q2k(blocks, K):
    rows = blocks.shape[0]
    out = np.empty((rows, K))
    for r in range(rows):
        for sb in range(K // 256):
            b = blocks[r, sb * 84:(sb + 1) * 84]
            d = float(np.frombuffer(b[80:82].tobytes(), np.float16)[0])
            dmin = float(np.frombuffer(b[82:84].tobytes(), np.float16)[0])
            sc, m = (b[:16] & 15).astype(np.float64), (b[:16] >> 4).astype(np.float64)
            q = np.array([(b[16 + n // 4] >> (2 * (n % 4))) & 3 for n in range(256)], np.float64)
            out[r, sb * 256:(sb + 1) * 256] = d * np.repeat(sc, 16) * q - dmin * np.repeat(m, 16)
    return out


def random_q2k(rng, rows, K):
    blks = []
    for _ in range(rows * (K // 256)):
        d = np.float16(rng.uniform(1e-3, 4e-3)).view(np.uint16)
        dmin = np.float16(rng.uniform(1e-3, 4e-3)).view(np.uint16)
        blks.append(build_q2k_block(d, dmin, rng.integers(0, 16, 16), rng.integers(0, 16, 16),
                                    rng.integers(0, 4, 256)))
    return np.stack(blks).reshape(rows, -1)


def test_dense_equivalence_q2k(ora, syn):
    cfg = syn.LayerConfig("t", T=2, d=256, F=512, E=2, k=1, wfmt="q2k")
    rng = np.random.default_rng(22)
    b1 = np.stack([random_q2k(rng, cfg.F, cfg.d) for _ in range(2)])
    b3 = np.stack([random_q2k(rng, cfg.F, cfg.d) for _ in range(2)])
    b2 = np.stack([random_q2k(rng, cfg.d, cfg.F) for _ in range(2)])
    L = ora.LayerWeights(cfg, b1, None, b3, None, b2, None)
    x = rand_x(rng, 2, cfg.d)
    for e in range(2):
        W1, W3, W2 = np_decode_q2k(b1[e], cfg.d), np_decode_q2k(b3[e], cfg.d), np_decode_q2k(b2[e], cfg.F)
        for t in range(2):
            ref = dense_ffn(bf16_vals(x[t]), W1, W3, W2)
            o = ora.expert_ffn_token(L, e, x[t])
            np.testing.assert_allclose(o, ref, rtol=0, atol=1e-4 * np.abs(ref).max())


def test_identical_tokens_identical_rows_and_rows_api(ora, syn):
    cfg = syn.LayerConfig("t", T=4, d=256, F=256, E=4, k=2)
    rng = np.random.default_rng(23)
    L, _ = make_layer(ora, cfg, rng)
    x = rand_x(rng, 4, cfg.d)
    x[2] = x[0]
    idx, w, y = ora.layer_tokens(L, x, np.arange(4))
    np.testing.assert_array_equal(y[2], y[0])
    counts, offsets, perm, inv = ora.permute(idx, cfg.E)
    rows = ora.expert_ffn_rows(L, x, offsets, perm)
    for s in range(8):
        t, j = divmod(s, 2)
        np.testing.assert_array_equal(rows[inv[s]], ora.expert_ffn_token(L, idx[t, j], x[t]).astype(np.float32))
    y2 = ora.combine(rows, inv, w)
    np.testing.assert_allclose(y2, y, rtol=0, atol=1e-6 * np.abs(y).max())


def test_combine_closed_forms(ora):
    rng = np.random.default_rng(24)
    T, k, d = 6, 3, 64
    rows = rng.normal(0, 1, (T * k, d)).astype(np.float32)
    inv = rng.permutation(T * k).astype(np.int32)
    onehot = np.zeros((T, k), np.float32)
    onehot[:, 1] = 1.0
    y = ora.combine(rows, inv, onehot)
    np.testing.assert_array_equal(y, rows[inv.reshape(T, k)[:, 1]])
    w = rng.uniform(0, 1, (T, k)).astype(np.float32)
    sh = rng.normal(0, 1, (T, d)).astype(np.float32)
    ref = np.einsum("tk,tkd->td", w.astype(np.float64), rows[inv.reshape(T, k)].astype(np.float64)) + sh
    np.testing.assert_allclose(ora.combine(rows, inv, w, sh), ref, rtol=1e-6, atol=1e-6)


def test_mxfp4_activation_quantiser_vs_brute_force(ora):
    """The fp64 MXFP4 quantiser (w4a4 activations) decodes to the brute-force
    nearest-value roundtrip above, over six decades, zero blocks and exact
    ties; on fp32 inputs it writes the bytes of the weights' quantiser."""
    rng = np.random.default_rng(23)
    v = rng.normal(0, 1, (64, 256)) * np.exp2(rng.integers(-20, 20, (64, 1)))
    v[0, :32] = 0.0
    v[1, :32] = np.tile([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 4.0], 4) * rng.choice([-1, 1], 32)  # ties at scale 1
    v[1, 0] = 6.0 * 1.0  # amax 6: scale 2^0
    v[2, :32] = 7.0 * rng.choice([-1, 1], 32)
    codes, scales = ora.mxfp4_quantize_f64(v)
    dec = ora.mxfp4_dequantize(codes, scales).astype(np.float64)
    np.testing.assert_array_equal(dec, mxfp4_roundtrip(v))
    f = v.astype(np.float32)
    c32, s32 = ora.mxfp4_quantize(f)
    c64, s64 = ora.mxfp4_quantize_f64(f.astype(np.float64))
    np.testing.assert_array_equal(c32, c64)
    np.testing.assert_array_equal(s32, s64)

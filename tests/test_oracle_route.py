"""Pins of the oracle's router, top-k, hash routing and permutation.

References: exact integer dot products, a hand-worked example of the fixed
reduction order, brute force over all expert subsets, numpy's softmax and
stable argsort, the golden-ratio constant computed from its definition, and
distributional properties of the hash.
"""
import decimal
import itertools
import math

import numpy as np
import pytest
import torch


def bf16_bits(vals):
    t = torch.tensor(np.asarray(vals, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_vals(bits):
    return torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16).double().numpy()


# ---- router logits ----------------------------------------------------------

def test_router_logits_exact_on_small_integers(ora):
    # small-integer bf16 values: every product and partial sum is exact in fp32
    rng = np.random.default_rng(10)
    x = bf16_bits(rng.integers(-8, 9, (5, 256)))
    wr = bf16_bits(rng.integers(-8, 9, (7, 256)))
    ref = bf16_vals(x) @ bf16_vals(wr).T
    np.testing.assert_array_equal(ora.router_logits(x, wr).astype(np.float64), ref)
    bias = np.arange(7, dtype=np.float32) - 3
    np.testing.assert_array_equal(ora.router_logits(x, wr, bias).astype(np.float64), ref + bias)


def test_router_logits_fp32_error_bound(ora, syn):
    x = syn.normal_bf16(0, 11, 0, 6 * 4096).reshape(6, 4096)
    wr = syn.normal_bf16(0, 12, 0, 16 * 4096, 0, 0.02).reshape(16, 4096)
    xv, wv = bf16_vals(x), bf16_vals(wr)
    ref = xv @ wv.T
    absdot = np.abs(xv) @ np.abs(wv).T
    got = ora.router_logits(x, wr).astype(np.float64)
    # 128 fmaf steps + 5 tree levels, each at most one fp32 rounding
    u = 2.0 ** -24
    assert np.all(np.abs(got - ref) <= (128 + 5) * u * absdot * 1.01)


def test_router_logits_reduction_order(ora):
    """Worked example of the documented order (d = 64: 32 chunks of 2).

    Chunk partials p0 = 2^25, p1 = 1, p2 = -2^25, p3 = 1, others 0.
    Tree: (p0 + p1) rounds to 2^25 (fp32 spacing 4 there), (p2 + p3) rounds to
    -2^25 (a tie between -33554430 and -33554432, resolved to the even
    significand 2^25), so the logit is exactly 0. A left-to-right sum would
    give 1 instead.
    """
    xs = np.zeros(64, np.float32)
    ws = np.zeros(64, np.float32)
    xs[0], ws[0] = 2.0 ** 13, 2.0 ** 12       # chunk 0: 2^25
    xs[2], ws[2] = 1.0, 1.0                   # chunk 1: 1
    xs[4], ws[4] = -(2.0 ** 13), 2.0 ** 12    # chunk 2: -2^25
    xs[6], ws[6] = 1.0, 1.0                   # chunk 3: 1
    got = ora.router_logits(bf16_bits(xs)[None], bf16_bits(ws)[None])
    assert got[0, 0] == 0.0
    # within a chunk the sum runs left to right: 2^25 + 1 - 2^25 + 1 = 2
    xs2, ws2 = np.zeros(64, np.float32), np.zeros(64, np.float32)
    xs2[0], ws2[0] = 2.0 ** 13, 2.0 ** 12
    xs2[1], ws2[1] = 1.0, 1.0
    got2 = ora.router_logits(bf16_bits(xs2)[None], bf16_bits(ws2)[None])
    assert got2[0, 0] == 2.0 ** 25  # fmaf(1, 1, 2^25) rounds back to 2^25


# ---- top-k ------------------------------------------------------------------

def brute_topk(l, k):
    E = len(l)
    good = []
    for S in itertools.combinations(range(E), k):
        ok = all(l[i] > l[j] or (l[i] == l[j] and i < j)
                 for i in S for j in range(E) if j not in S)
        if ok:
            good.append(S)
    assert len(good) == 1
    S = sorted(good[0], key=lambda e: (-l[e], e))
    return S


def test_topk_bruteforce_with_ties(ora):
    rng = np.random.default_rng(13)
    for trial in range(300):
        E, k = 8, int(rng.integers(1, 5))
        l = rng.integers(-3, 4, E).astype(np.float32)  # small integers force ties
        if trial % 3 == 0:
            l[rng.integers(0, E)] = -0.0
        idx, w = ora.topk_softmax(l[None], k)
        assert list(idx[0]) == brute_topk(list(l), k), (l, k)


def test_topk_nan_last_and_gates(ora):
    l = np.array([[1.0, np.nan, 3.0, 2.0, np.nan, -1.0]], np.float32)
    idx, w = ora.topk_softmax(l, 5)
    assert list(idx[0]) == [2, 3, 0, 5, 1]


def test_gates_softmax_renormalised(ora, syn):
    rng = np.random.default_rng(14)
    logits = rng.normal(0, 2, (50, 64)).astype(np.float32)
    idx, w = ora.topk_softmax(logits, 8)
    full = torch.softmax(torch.from_numpy(logits).double(), dim=1).numpy()
    sel = np.take_along_axis(full, idx.astype(np.int64), axis=1)
    ref = sel / sel.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(w, ref, rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, atol=1e-6)
    assert np.all(np.diff(w, axis=1) <= 0)


# ---- hash routing ------------------------------------------------------------

def test_splitmix_increment_is_golden_ratio_constant(ora):
    """The SplitMix64 state step is floor(2^64 / phi), an odd integer."""
    decimal.getcontext().prec = 60
    phi = (1 + decimal.Decimal(5).sqrt()) / 2
    gamma = int(decimal.Decimal(2) ** 64 / phi)
    assert gamma % 2 == 1
    # the first output for state 0 is the finaliser of gamma; the finaliser is
    # a bijection, so the outputs for states s and s + gamma are one step apart
    a = ora.splitmix64_outputs(0, 3)
    b = ora.splitmix64_outputs(gamma, 2)
    assert a[1:] == b


def test_splitmix_outputs_match_a_library_splitmix64(ora):
    """numba's xoroshiro128+ seeding is a library implementation of the
    SplitMix64 generator's first output (state + golden-ratio increment, then
    the finaliser). Output j for a seed is the first output for the seed
    advanced by j increments, so it pins every draw the hash routing takes."""
    rnd = pytest.importorskip("numba.cuda.random")
    st = np.zeros(1, dtype=rnd.xoroshiro128p_dtype)
    gamma = 0x9E3779B97F4A7C15
    for seed in (0, 1, 7, 12345, 129279, 2**32 + 3, 2**63 + 5):
        ours = ora.splitmix64_outputs(seed, 4)
        for j, o in enumerate(ours):
            rnd.init_xoroshiro128p_state(st, 0, np.uint64((seed + j * gamma) % 2**64))
            assert int(st[0]["s0"]) == o, (seed, j)


def test_splitmix_outputs_distinct_and_uniform(ora):
    outs = ora.splitmix64_outputs(12345, 20000)
    assert len(set(outs)) == len(outs)
    bits = np.array([[(o >> b) & 1 for b in range(64)] for o in outs[:4000]])
    assert np.all(np.abs(bits.mean(axis=0) - 0.5) < 0.05)


def test_hash_route_properties(ora, syn):
    tok = syn.uniform_int(0, 20, 0, 16384, 0, 129280)
    idx, w, failed = ora.hash_route(tok, 256, 8)
    assert failed == 0
    assert np.all((idx >= 0) & (idx < 256))
    assert all(len(set(r)) == 8 for r in idx)
    assert np.all(w == np.float32(0.125))
    # same token id -> same experts
    tok2 = tok.copy()
    tok2[1] = tok2[0]
    idx2, _, _ = ora.hash_route(tok2, 256, 8)
    assert list(idx2[1]) == list(idx2[0])
    # roughly uniform expert load (chi-square, 255 dof)
    counts = np.bincount(idx.ravel(), minlength=256)
    exp = idx.size / 256
    chi2 = ((counts - exp) ** 2 / exp).sum()
    assert chi2 < 255 + 6 * math.sqrt(2 * 255)
    # the first accepted expert is the first draw mod E
    first = [ora.splitmix64_outputs(int(t), 1)[0] % 256 for t in tok[:50]]
    assert list(idx[:50, 0]) == first


def test_hash_route_cap(ora):
    # E = k forces every expert; a tiny draw cap must report failure
    idx, w, failed = ora.hash_route(np.arange(4, dtype=np.int32), 8, 8, max_draws=3)
    assert failed == 4 and np.all(idx[:, 3:] == -1)
    idx, w, failed = ora.hash_route(np.arange(4, dtype=np.int32), 8, 8)
    assert failed == 0 and all(sorted(r) == list(range(8)) for r in idx)


# ---- permute ------------------------------------------------------------------

def test_permute_vs_stable_argsort(ora):
    rng = np.random.default_rng(15)
    for T, k, E in ((1, 8, 256), (7, 2, 8), (64, 8, 256), (33, 4, 16)):
        idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
        counts, offsets, perm, inv = ora.permute(idx, E)
        np.testing.assert_array_equal(counts, np.bincount(idx.ravel(), minlength=E))
        np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(counts)]))
        np.testing.assert_array_equal(perm, np.argsort(idx.ravel(), kind="stable"))
        np.testing.assert_array_equal(perm[inv], np.arange(T * k))


def test_permute_rejects_bad_index(ora):
    with pytest.raises(ValueError):
        ora.permute(np.array([[0, 9]], np.int32), 8)
    with pytest.raises(ValueError):
        ora.permute(np.array([[-1, 2]], np.int32), 8)

"""GPU parity: the CUDA library (through the C ABI) against the oracle.

Bit-exact: quantised weights, dequantised weights, MXFP8 activation codes,
routing indices, counts, offsets, permutations. Floating point: gates to 1e-6,
layer outputs to 2e-3 * max|ref| (bf16 activations) or 1e-2 * max|ref| (MXFP8
activations), the bounds the layer is specified to.
"""
import numpy as np
import pytest

import oracle
import synth
from harness import Case, bf16_to_f32

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import routed_expert_ffn_05_b200 as M  # noqa: E402

DEV = torch.device("cuda:0")
TOL = {"bf16": 2e-3, "mxfp8": 1e-2}


def dev(a):
    if a.dtype == np.uint16:
        a = a.astype(np.int16)
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def host(t, dtype=None):
    a = t.cpu().numpy()
    return a.view(dtype) if dtype is not None else a


def assert_rel(got, ref, rel, what=""):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref).max()
    scale = np.abs(ref).max()
    assert err <= rel * scale, f"{what}: max|err| {err:.3e} > {rel} * max|ref| {scale:.3e}"


def cfg_of(name, T=None):
    c = synth.CONFIGS[name]
    return c.with_T(T) if T is not None else c


LAYER_CASES = [("tiny", None), ("decode", 1), ("decode", 2), ("decode", 4), ("decode", 8),
               ("q2k", 1), ("q2k", 8), ("q2k", 16), ("prefill", 9), ("prefill", None), ("hash", None)]
_cases = {}


def get_case(name, T=None):
    key = (name, T)
    if key not in _cases:
        cfg = cfg_of(name, T)
        _cases[key] = Case(cfg, experts="all" if cfg.T * cfg.k >= cfg.E * 4 else "routed")
    return _cases[key]


def tile_edge_rows(offsets, tile=128):
    """Per expert with rows: the first and last row of its last 128-row token
    tile (the partial tile, when the count is not a multiple of 128)."""
    out = []
    for e in range(len(offsets) - 1):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi > lo:
            out += [lo + (hi - lo - 1) // tile * tile, hi - 1]
    return np.unique(np.array(out, np.int64))


def sample_tokens(cfg, ora_idx=None, n=512, seed=0):
    """All tokens of a small batch; else n random tokens, the first and last,
    and the tokens of the first and last row of every expert's last token tile."""
    if cfg.T <= n:
        return np.arange(cfg.T, dtype=np.int32)
    rng = np.random.default_rng(seed)
    s = rng.choice(cfg.T, n - 2, replace=False)
    extra = []
    if ora_idx is not None:
        _, offsets, perm, _ = oracle.permute(ora_idx, cfg.E)
        extra = perm[tile_edge_rows(offsets)] // cfg.k
    return np.unique(np.concatenate([[0, cfg.T - 1], s, extra])).astype(np.int32)


# ---- formats ----------------------------------------------------------------

def special_weights(rows, K, rng):
    w = rng.normal(0, 0.02, (rows, K)).astype(np.float32)
    w[0, :32] = 0.0
    w[0, 32:64] = -0.0
    w[1, :32] = np.float32(2.0 ** -130) * rng.integers(-3, 4, 32)     # subnormal fp32
    w[1, 32:64] = rng.normal(0, 1e30, 32)
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 4.0], np.float32)
    w[2, :32] = np.tile(np.concatenate([ties, -ties]), 2) * np.float32(2.0 ** -7)  # amax 5 -> scale 2^-7 *... exact ties
    w[2, 64:96] = np.float32(7.5) * rng.choice([-1, 1], 32)           # saturates to 6
    w[3, :] = -np.abs(w[3, :])                                         # all negative
    return w


@pytest.mark.parametrize("wfmt", ["mxfp4", "q2k"])
def test_quantize_weights_bitexact(wfmt):
    cfg = synth.LayerConfig("q", T=1, d=512, F=256, E=2, k=1, wfmt=wfmt)
    dims = M.make_dims(1, cfg.d, cfg.F, cfg.E, 1, wfmt=M.MOE_W_Q2K if wfmt == "q2k" else M.MOE_W_MXFP4)
    rng = np.random.default_rng(30)
    for which, (N, K) in ((M.MOE_MAT_W1, (cfg.F, cfg.d)), (M.MOE_MAT_W2, (cfg.d, cfg.F))):
        w = np.stack([special_weights(N, K, rng) for _ in range(cfg.E)])
        ref_a, ref_b = oracle.quantize_expert(cfg, w.reshape(-1, K))
        ref = np.concatenate([ref_a.ravel(), ref_b.ravel()]) if ref_b is not None else ref_a.ravel()
        out = torch.zeros(ref.size, dtype=torch.uint8, device=DEV)
        M.moe_quantize_weights(dims, which, dev(w), out)
        got = host(out)
        bad = np.nonzero(got != ref)[0]
        assert bad.size == 0, f"{bad.size} bytes differ, first at {bad[:8]}"


@pytest.mark.parametrize("wfmt", ["mxfp4", "q2k"])
def test_debug_dequant_bitexact(wfmt):
    cfg = synth.LayerConfig("q", T=1, d=512, F=256, E=3, k=1, wfmt=wfmt)
    dims = M.make_dims(1, cfg.d, cfg.F, cfg.E, 1, wfmt=M.MOE_W_Q2K if wfmt == "q2k" else M.MOE_W_MXFP4)
    rng = np.random.default_rng(31)
    for which, (N, K) in ((M.MOE_MAT_W3, (cfg.F, cfg.d)), (M.MOE_MAT_W2, (cfg.d, cfg.F))):
        w = rng.normal(0, 0.02, (cfg.E * N, K)).astype(np.float32)
        a, b = oracle.quantize_expert(cfg, w)
        if b is not None:
            b[0, 0], b[1, 1] = 0, 254    # extreme (finite) scales
        canon = dev(np.concatenate([a.ravel(), b.ravel()]) if b is not None else a.ravel())
        packed = torch.empty(M.moe_packed_size(dims, which), dtype=torch.uint8, device=DEV)
        M.moe_pack_weights(dims, which, canon, packed)
        for e in range(cfg.E):
            out = torch.empty((N, K), dtype=torch.float32, device=DEV)
            M.moe_debug_dequant(dims, which, packed, e, out)
            if b is not None:
                ref = oracle.mxfp4_dequantize(a[e * N:(e + 1) * N], b[e * N:(e + 1) * N])
            else:
                ref = oracle.q2k_dequantize(a[e * N:(e + 1) * N], K)
            np.testing.assert_array_equal(host(out).view(np.uint32), ref.view(np.uint32))


def test_debug_dequant_nan_scale():
    dims = M.make_dims(1, 256, 256, 1, 1)
    a = np.full((256, 128), 0x21, np.uint8)
    b = np.full((256, 8), 127, np.uint8)
    b[5, 2] = 0xFF
    canon = dev(np.concatenate([a.ravel(), b.ravel()]))
    packed = torch.empty(M.moe_packed_size(dims, M.MOE_MAT_W1), dtype=torch.uint8, device=DEV)
    M.moe_pack_weights(dims, M.MOE_MAT_W1, canon, packed)
    out = torch.empty((256, 256), dtype=torch.float32, device=DEV)
    M.moe_debug_dequant(dims, M.MOE_MAT_W1, packed, 0, out)
    o = host(out)
    assert np.all(np.isnan(o[5, 64:96])) and not np.any(np.isnan(np.delete(o[5], np.s_[64:96])))


def test_quant_act_bitexact():
    rng = np.random.default_rng(32)
    x = synth.normal_bf16(0, 77, 0, 64 * 512).reshape(64, 512)
    x[0, :32] = 0
    x[0, 32:64] = 0x8000                                        # -0.0
    x[1, :32] = rng.integers(1, 0x7F, 32).astype(np.uint16)     # bf16 subnormals
    x[1, 32:64] = 0x7E00 | rng.integers(0, 0x7F, 32).astype(np.uint16)  # ~1e38
    x[2, :32] = rng.integers(0x3F00, 0x4000, 32).astype(np.uint16)      # ties after scaling
    codes = torch.empty((64, 512), dtype=torch.uint8, device=DEV)
    scales = torch.empty((64, 16), dtype=torch.uint8, device=DEV)
    M.moe_debug_quant_act(dev(x), 64, 512, codes, scales)
    rc, rs = oracle.mxfp8_quantize_bf16(x)
    np.testing.assert_array_equal(host(scales), rs)
    np.testing.assert_array_equal(host(codes), rc)


# ---- routing and permutation ------------------------------------------------

ROUTE_CASES = LAYER_CASES


@pytest.mark.parametrize("name,T", ROUTE_CASES)
def test_route_bitexact(name, T):
    c = get_case(name, T)
    cfg = c.cfg
    idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=DEV)
    w = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device=DEV)
    M.moe_route(c.dims, c.x_d, c.weights, c.tok_d, idx, w, c.ws)
    assert M.moe_get_device_error() == 0
    gi = host(idx)
    bad = np.nonzero(np.any(gi != c.ora_idx, axis=1))[0]
    assert bad.size == 0, f"{bad.size} tokens routed differently, first {bad[:5]}"
    np.testing.assert_allclose(host(w), c.ora_w, rtol=0, atol=2e-6)


@pytest.mark.parametrize("T", [8, 40])
def test_route_ties_to_lower_index(T):
    """T = 8 runs the per-token router, T = 40 the batch router on the tensor cores."""
    cfg = synth.LayerConfig("ties", T=T, d=256, F=256, E=16, k=4)
    wr = synth.make_router(cfg)
    wr[5] = wr[2]            # experts 2 and 5 always tie
    wr[9] = wr[2]
    x = synth.make_x(cfg)
    x[3] = 0                 # all logits +0: picks experts 0..3
    idx_ref, w_ref = oracle.topk_softmax(oracle.router_logits(x, wr), cfg.k)
    dims = M.make_dims(cfg.T, cfg.d, cfg.F, cfg.E, cfg.k)
    ws = torch.empty(M.moe_workspace_size(dims), dtype=torch.uint8, device=DEV)
    weights = M.make_weights(None, None, None, w_router=dev(wr))
    idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=DEV)
    w = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device=DEV)
    M.moe_route(dims, dev(x), weights, None, idx, w, ws)
    np.testing.assert_array_equal(host(idx), idx_ref)
    assert list(idx_ref[3]) == [0, 1, 2, 3]
    np.testing.assert_allclose(host(w), w_ref, atol=2e-6)


@pytest.mark.parametrize("T", [8, 40])
def test_route_nan_logits_rank_last(T):
    """A token whose x row holds a NaN has NaN logits for every expert: they
    all rank after every number and tie among themselves, so the token takes
    experts 0 .. k-1 (and NaN gates); a token with one NaN-free logit row is
    untouched. T = 40 runs the tiled router, T = 8 the per-token one."""
    cfg = synth.LayerConfig("nan", T=T, d=256, F=256, E=16, k=4)
    wr = synth.make_router(cfg)
    x = synth.make_x(cfg)
    x[1, 7] = 0x7FC0                      # bf16 quiet NaN
    logits = oracle.router_logits(x, wr)
    assert np.all(np.isnan(logits[1])) and not np.any(np.isnan(np.delete(logits, 1, axis=0)))
    idx_ref, w_ref = oracle.topk_softmax(logits, cfg.k)
    assert list(idx_ref[1]) == [0, 1, 2, 3]
    dims = M.make_dims(cfg.T, cfg.d, cfg.F, cfg.E, cfg.k)
    ws = torch.empty(M.moe_workspace_size(dims), dtype=torch.uint8, device=DEV)
    weights = M.make_weights(None, None, None, w_router=dev(wr))
    idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=DEV)
    w = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device=DEV)
    M.moe_route(dims, dev(x), weights, None, idx, w, ws)
    np.testing.assert_array_equal(host(idx), idx_ref)
    np.testing.assert_allclose(host(w), w_ref, atol=2e-6)   # NaN gates compare equal


@pytest.mark.parametrize("name,T", ROUTE_CASES)
def test_permute_bitexact(name, T):
    c = get_case(name, T)
    cfg = c.cfg
    counts_r, offsets_r, perm_r, inv_r = oracle.permute(c.ora_idx, cfg.E)
    counts = torch.empty(cfg.E, dtype=torch.int32, device=DEV)
    offsets = torch.empty(cfg.E + 1, dtype=torch.int32, device=DEV)
    perm = torch.empty(cfg.T * cfg.k, dtype=torch.int32, device=DEV)
    inv = torch.empty(cfg.T * cfg.k, dtype=torch.int32, device=DEV)
    M.moe_permute(c.dims, dev(c.ora_idx), counts, offsets, perm, inv, c.ws)
    np.testing.assert_array_equal(host(counts), counts_r)
    np.testing.assert_array_equal(host(offsets), offsets_r)
    np.testing.assert_array_equal(host(perm), perm_r)
    np.testing.assert_array_equal(host(inv), inv_r)


def test_permute_bad_expert_sets_device_error():
    dims = M.make_dims(4, 256, 256, 8, 2)
    ws = torch.empty(M.moe_workspace_size(dims), dtype=torch.uint8, device=DEV)
    idx = dev(np.array([[0, 1], [2, 8], [3, 4], [5, 6]], np.int32))
    bufs = [torch.empty(n, dtype=torch.int32, device=DEV) for n in (8, 9, 8, 8)]
    M.moe_permute(dims, idx, *bufs, ws)
    assert M.moe_get_device_error() == M.MOE_DEVERR_EXPERT_RANGE
    assert M.moe_get_device_error() == 0   # read clears it


# ---- expert FFN, shared expert, combine, layer ------------------------------

@pytest.mark.parametrize("name,T", LAYER_CASES)
def test_expert_ffn(name, T):
    c = get_case(name, T)
    cfg = c.cfg
    _, offsets_r, perm_r, _ = oracle.permute(c.ora_idx, cfg.E)
    out = torch.empty((cfg.T * cfg.k, cfg.d), dtype=torch.float32, device=DEV)
    M.moe_expert_ffn(c.dims, c.weights, c.x_d, dev(offsets_r), dev(perm_r), out, c.ws)
    got = host(out)
    S = cfg.T * cfg.k
    if S <= 64:
        ranges = [(0, S)]
    else:  # rows from the busiest expert, the last expert, random places, every expert's last tile edges
        e_big = int(np.argmax(np.diff(offsets_r)))
        rng = np.random.default_rng(3)
        starts = [offsets_r[e_big], S - 4] + list(rng.integers(0, S - 4, 64))
        ranges = [(int(s), int(s) + 4) for s in starts]
        ranges += [(int(r), int(r) + 1) for r in tile_edge_rows(offsets_r)]
    for a, b in ranges:
        ref = oracle.expert_ffn_rows(c.ora, c.x, offsets_r, perm_r, a, b)
        assert_rel(got[a:b], ref, TOL[cfg.act], f"{name} rows {a}:{b}")


def test_shared_ffn():
    c = get_case("decode", 4)
    out = torch.empty((4, c.cfg.d), dtype=torch.float32, device=DEV)
    M.moe_shared_ffn(c.dims, c.weights, c.x_d, out, c.ws)
    ref = np.stack([oracle.shared_ffn_token(c.ora, c.x[t]) for t in range(4)])
    assert_rel(host(out), ref, 1e-4, "shared expert")


def test_combine():
    rng = np.random.default_rng(33)
    T, k, d = 37, 8, 512
    dims = M.make_dims(T, d, 256, 64, k)
    rows = rng.normal(0, 1, (T * k, d)).astype(np.float32)
    inv = rng.permutation(T * k).astype(np.int32)
    w = rng.uniform(0, 1, (T, k)).astype(np.float32)
    sh = rng.normal(0, 1, (T, d)).astype(np.float32)
    y = torch.empty((T, d), dtype=torch.float32, device=DEV)
    for shared in (None, sh):
        M.moe_combine(dims, dev(rows), dev(inv), dev(w), None if shared is None else dev(shared), y)
        np.testing.assert_allclose(host(y), oracle.combine(rows, inv, w, shared), rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("name,T", LAYER_CASES)
def test_layer(name, T):
    c = get_case(name, T)
    cfg = c.cfg
    y = torch.empty((cfg.T, cfg.d), dtype=torch.float32, device=DEV)
    M.moe_layer(c.dims, c.weights, c.x_d, c.tok_d, y, c.ws)
    assert M.moe_get_device_error() == 0
    toks = sample_tokens(cfg, c.ora_idx)
    idx, w, ref = oracle.layer_tokens(c.ora, c.x, toks, c.token_ids)
    np.testing.assert_array_equal(idx, c.ora_idx[toks])
    assert_rel(host(y)[toks], ref, TOL[cfg.act], f"{name} T={cfg.T}")


# ---- edge cases -----------------------------------------------------------------

@pytest.mark.parametrize("T,k,E", [(0, 2, 8), (1, 1, 8), (5, 8, 8), (33, 2, 8), (130, 3, 16)])
def test_layer_edges(T, k, E):
    """Empty batch, k = 1, k = E (every expert), ragged token counts."""
    cfg = synth.LayerConfig("edge", T=T, d=256, F=512, E=E, k=k)
    c = Case(cfg, experts="all")
    y = torch.full((max(T, 1), cfg.d), 7.0, dtype=torch.float32, device=DEV)
    M.moe_layer(c.dims, c.weights, c.x_d, None, y, c.ws)
    assert M.moe_get_device_error() == 0
    if T == 0:
        assert torch.all(y == 7.0)
        return
    toks = np.arange(T, dtype=np.int32)
    _, _, ref = oracle.layer_tokens(c.ora, c.x, toks)
    assert_rel(host(y), ref, TOL["bf16"], f"T={T} k={k} E={E}")


@pytest.mark.parametrize("T,k,E", [(1, 1, 8), (37, 2, 8), (300, 3, 16), (260, 4, 4)])
def test_expert_ffn_w4a8_every_row(T, k, E):
    """w4a8 expert FFN, every row against the oracle: a single token, ragged
    token tiles (not multiples of 16), experts with several 128-token tiles and
    an expert taking every token."""
    cfg = synth.LayerConfig("w4a8", T=T, d=256, F=512, E=E, k=k, act="mxfp8")
    c = Case(cfg, experts="all")
    _, offsets_r, perm_r, _ = oracle.permute(c.ora_idx, cfg.E)
    out = torch.full((T * k, cfg.d), float("nan"), dtype=torch.float32, device=DEV)
    M.moe_expert_ffn(c.dims, c.weights, c.x_d, dev(offsets_r), dev(perm_r), out, c.ws)
    assert M.moe_get_device_error() == 0
    ref = oracle.expert_ffn_rows(c.ora, c.x, offsets_r, perm_r, 0, T * k)
    assert_rel(host(out), ref, TOL["mxfp8"], f"w4a8 T={T} k={k} E={E}")


@pytest.mark.parametrize("bad", ["duplicate", "out_of_range"])
def test_expert_ffn_w4a8_bad_perm_sets_device_error(bad):
    """The w4a8 path inverts perm to quantise each token once; a perm that is
    not a permutation of the T*k slots is reported, not followed."""
    cfg = synth.LayerConfig("w4a8", T=37, d=256, F=512, E=8, k=2, act="mxfp8")
    c = Case(cfg, experts="all")
    _, offsets_r, perm_r, _ = oracle.permute(c.ora_idx, cfg.E)
    perm_bad = perm_r.copy()
    if bad == "duplicate":
        perm_bad[5] = perm_bad[4]
    else:
        perm_bad[3] = cfg.T * cfg.k + 5
    out = torch.empty((cfg.T * cfg.k, cfg.d), dtype=torch.float32, device=DEV)
    M.moe_expert_ffn(c.dims, c.weights, c.x_d, dev(offsets_r), dev(perm_bad), out, c.ws)
    assert M.moe_get_device_error() == M.MOE_DEVERR_PERM
    M.moe_expert_ffn(c.dims, c.weights, c.x_d, dev(offsets_r), dev(perm_r), out, c.ws)
    assert M.moe_get_device_error() == 0   # the next good call is clean
    ref = oracle.expert_ffn_rows(c.ora, c.x, offsets_r, perm_r, 0, cfg.T * cfg.k)
    assert_rel(host(out), ref, TOL["mxfp8"], f"w4a8 after bad perm ({bad})")


def test_identical_tokens_identical_outputs():
    cfg = synth.LayerConfig("dup", T=6, d=256, F=512, E=8, k=2)
    c = Case(cfg, experts="all")
    x = c.x.copy()
    x[4] = x[1]
    y = torch.empty((6, cfg.d), dtype=torch.float32, device=DEV)
    M.moe_layer(c.dims, c.weights, dev(x), None, y, c.ws)
    yh = host(y)
    np.testing.assert_array_equal(yh[4], yh[1])


def test_decode_route_ties_to_lower_index():
    """The decode layer's own routing kernels break ties by the lower expert
    index. Token 0's last pick a shares its router row with the two lowest
    experts token 0 leaves out, so the three tie bit for bit at token 0's
    k-th place and only the lowest of them may be taken. Each expert has its
    own weights, so another pick shows in y."""
    from dataclasses import replace
    cfg = replace(synth.CONFIGS["decode"], E=16).with_T(8)
    assert synth.make_bias(cfg, 0) is None
    idx0, _ = oracle.topk_softmax(oracle.router_logits(synth.make_x(cfg, 0, 0), synth.make_router(cfg, 0)), cfg.k)
    a = int(idx0[0, -1])
    b, c = [e for e in range(cfg.E) if e not in idx0[0]][:2]

    def tie(wr):
        wr[b] = wr[a]
        wr[c] = wr[a]

    case = Case(cfg, experts="all", router_fn=tie)
    assert len({a, b, c} & set(case.ora_idx[0].tolist())) == 1
    assert min(a, b, c) in case.ora_idx[0]
    y = torch.empty((cfg.T, cfg.d), dtype=torch.float32, device=DEV)
    M.moe_layer(case.dims, case.weights, case.x_d, None, y, case.ws)
    assert M.moe_get_device_error() == 0
    toks = np.arange(cfg.T, dtype=np.int32)
    idx, _, ref = oracle.layer_tokens(case.ora, case.x, toks)
    np.testing.assert_array_equal(idx, case.ora_idx)
    assert_rel(host(y), ref, TOL[cfg.act], "decode ties")


@pytest.mark.parametrize("wfmt,T,E", [("mxfp4", 8, 8), ("mxfp4", 3, 16), ("q2k", 8, 8), ("q2k", 5, 16)])
def test_decode_path_dense_experts(wfmt, T, E):
    """The fused decode kernel (d 4096, d_ff 2048, shared expert) with few
    experts: with E = k = 8 every token goes to every expert, so each expert
    has T rows — the most token columns its gate/up epilogue and its down
    units handle; E = 16 gives a ragged mix. Every token against the oracle."""
    from dataclasses import replace
    cfg = replace(synth.CONFIGS["q2k" if wfmt == "q2k" else "decode"], E=E).with_T(T)
    c = Case(cfg, experts="all")
    y = torch.empty((T, cfg.d), dtype=torch.float32, device=DEV)
    M.moe_layer(c.dims, c.weights, c.x_d, None, y, c.ws)
    assert M.moe_get_device_error() == 0
    toks = np.arange(T, dtype=np.int32)
    idx, _, ref = oracle.layer_tokens(c.ora, c.x, toks)
    np.testing.assert_array_equal(idx, c.ora_idx)
    assert_rel(host(y), ref, TOL[cfg.act], f"{wfmt} T={T} E={E}")

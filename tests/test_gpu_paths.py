"""GPU parity of the paths and failure cases the main parity file does not reach.

- The tensor-core path's MXFP8 activation staging, byte for byte against the
  oracle's quantiser: the codes and scale atoms the block-scaled GEMM reads.
- The generic CUDA-core path with Q2_K weights (T above the decode batch, small
  dims, MXFP8 activations).
- Hash routing at its draw cap, and slots without a valid expert through
  permute and combine.
- The decode kernel's inter-CTA wait running out (a count nobody publishes),
  and two decode layers at once on two streams.
"""
import time
from dataclasses import replace

import numpy as np
import pytest

import oracle
import synth
from harness import Case

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


def host(t):
    return t.cpu().numpy()


def assert_rel(got, ref, rel, what=""):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err, scale = np.abs(got - ref).max(), np.abs(ref).max()
    assert err <= rel * scale, f"{what}: max|err| {err:.3e} > {rel} * max|ref| {scale:.3e}"


# ---- tensor-core activation staging, byte for byte ------------------------------

def special_x(T, d, rng):
    """N(0, 1) bf16 rows with the MX rule's corner cases in the first tokens."""
    x = synth.normal_bf16(0, 91, 0, T * d).reshape(T, d)
    x[0, :32] = 0                                                        # all-zero block: scale 127
    x[0, 32:64] = 0x8000                                                 # -0.0
    x[1, :32] = rng.integers(1, 0x7F, 32).astype(np.uint16)              # bf16 subnormals
    x[1, 32:64] = 0x7E00 | rng.integers(0, 0x7F, 32).astype(np.uint16)   # ~1e38: the top of the scale range
    x[2, :32] = rng.integers(0x3F00, 0x4000, 32).astype(np.uint16)       # exact E4M3 ties after scaling
    x[3, :32] = 0x43E0 | rng.integers(0, 0x20, 32).astype(np.uint16)     # near 448 x 2^s: saturation edge
    x[3, 32:64] = x[3, :32] | 0x8000
    return x


@pytest.mark.parametrize("T,d,E,k", [(300, 512, 8, 2), (37, 256, 4, 4), (600, 4096, 64, 8)])
def test_tc_gather_codes_and_atoms_bitexact(T, d, E, k):
    """Codes and E8M0 scale atoms that the w4a8 GEMM reads, for every routed row:
    ragged token tiles (counts not multiples of 128, some experts empty) and
    the special rows above."""
    rng = np.random.default_rng(40 + T)
    x = special_x(T, d, rng)
    pool = np.array([e for e in range(E) if E <= k or e != E // 2])    # expert E/2 gets no rows (E > k)
    idx = np.stack([rng.choice(pool, k, replace=False) for _ in range(T)]).astype(np.int32)
    counts, offsets, perm, _ = oracle.permute(idx, E)
    S = T * k
    dims = M.make_dims(T, d, 256, E, k, act=M.MOE_A_MXFP8)
    ws = torch.empty(M.moe_workspace_size(dims), dtype=torch.uint8, device=DEV)
    tiles = (S + 127) // 128 + E
    codes = torch.zeros((S, d), dtype=torch.uint8, device=DEV)
    atoms = torch.zeros((tiles, d // 128, 512), dtype=torch.uint8, device=DEV)
    ustart = torch.zeros(E + 1, dtype=torch.int32, device=DEV)
    M.moe_debug_tc_gather(dims, dev(x), dev(offsets), dev(perm), codes, atoms, ustart, ws)
    assert M.moe_get_device_error() == 0
    xc, xs = oracle.mxfp8_quantize_bf16(x)
    tok = perm // k
    np.testing.assert_array_equal(host(codes), xc[tok])
    nt = (counts + 127) // 128
    us = np.concatenate([[0], np.cumsum(nt)]).astype(np.int32)
    np.testing.assert_array_equal(host(ustart), us)
    at = host(atoms).reshape(-1)
    e_of_row = np.repeat(np.arange(E), counts)
    rloc = np.arange(S) - offsets[e_of_row]
    tile = us[e_of_row] + rloc // 128
    b = np.arange(d // 32)
    pos = ((tile[:, None] * (d // 128) + b[None, :] // 4) * 512
           + (rloc[:, None] % 32) * 16 + ((rloc[:, None] % 128) // 32) * 4 + b[None, :] % 4)
    np.testing.assert_array_equal(at[pos], xs[tok])


# ---- generic path with Q2_K weights ----------------------------------------------

GENERIC_Q2K = [
    ("q2k-T16", replace(synth.CONFIGS["q2k"], T=16)),                         # decode dims, above the decode batch
    ("q2k-small", synth.LayerConfig("q2k-small", T=37, d=512, F=256, E=8, k=2, wfmt="q2k")),
    ("q2k-w4a8", synth.LayerConfig("q2k-w4a8", T=37, d=512, F=256, E=8, k=2, wfmt="q2k", act="mxfp8")),
    ("q2k-w4a8-shared", synth.LayerConfig("q2k-w4a8-sh", T=20, d=512, F=256, E=8, k=3, wfmt="q2k",
                                          act="mxfp8", Fs=256)),
]


@pytest.mark.parametrize("name,cfg", GENERIC_Q2K, ids=[n for n, _ in GENERIC_Q2K])
def test_generic_q2k_layer_and_rows(name, cfg):
    c = Case(cfg, experts="all" if cfg.E <= 16 else "routed")
    y = torch.empty((cfg.T, cfg.d), dtype=torch.float32, device=DEV)
    M.moe_layer(c.dims, c.weights, c.x_d, None, y, c.ws)
    assert M.moe_get_device_error() == 0
    toks = np.arange(cfg.T, dtype=np.int32)
    idx, _, ref = oracle.layer_tokens(c.ora, c.x, toks)
    np.testing.assert_array_equal(idx, c.ora_idx)
    assert_rel(host(y), ref, TOL[cfg.act], name)
    # the routed rows alone, every row
    _, offsets, perm, _ = oracle.permute(c.ora_idx, cfg.E)
    S = cfg.T * cfg.k
    out = torch.full((S, cfg.d), float("nan"), dtype=torch.float32, device=DEV)
    M.moe_expert_ffn(c.dims, c.weights, c.x_d, dev(offsets), dev(perm), out, c.ws)
    assert M.moe_get_device_error() == 0
    assert_rel(host(out), oracle.expert_ffn_rows(c.ora, c.x, offsets, perm, 0, S), TOL[cfg.act], name + " rows")


# ---- hash routing at its draw cap; slots without an expert ----------------------

def test_hash_route_draw_cap():
    """With E = k every token needs all E experts; a cap of 12 draws leaves some
    tokens short: they get -1 in the slots they could not fill, exactly where
    the oracle's capped routing leaves them, and the device error is set."""
    T, E, k, cap = 200, 8, 8, 12
    tok = synth.uniform_int(0, synth.TOK, 7, T, 0, 129280)
    idx_r, w_r, failed = oracle.hash_route(tok, E, k, max_draws=cap)
    assert 0 < failed < T
    dims = M.make_dims(T, 256, 256, E, k, route=M.MOE_ROUTE_HASH)
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, k), dtype=torch.float32, device=DEV)
    M.moe_debug_hash_route(dims, dev(tok), cap, idx, w)
    assert M.moe_get_device_error() == M.MOE_DEVERR_HASH_CAP
    np.testing.assert_array_equal(host(idx), idx_r)
    np.testing.assert_array_equal(host(w), w_r)
    M.moe_debug_hash_route(dims, dev(tok), 1024, idx, w)   # the layer's cap: nobody is short here
    assert M.moe_get_device_error() == 0
    idx_full, _, failed_full = oracle.hash_route(tok, E, k)
    assert failed_full == 0
    np.testing.assert_array_equal(host(idx), idx_full)


def test_slots_without_an_expert_take_no_row():
    """Expert indices outside [0, E) are reported; those slots get no row and
    inv_perm -1, the other slots keep their stable order, and the combine
    skips them."""
    T, k, E, d = 6, 3, 8, 256
    idx = np.array([[0, 1, 2], [3, -1, 4], [1, 8, 0], [5, 6, 7], [-1, -1, 2], [4, 3, 1]], np.int32)
    dims = M.make_dims(T, d, 256, E, k)
    ws = torch.empty(M.moe_workspace_size(dims), dtype=torch.uint8, device=DEV)
    S = T * k
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    perm = torch.full((S,), -7, dtype=torch.int32, device=DEV)
    inv = torch.full((S,), 99, dtype=torch.int32, device=DEV)
    M.moe_permute(dims, dev(idx), counts, offsets, perm, inv, ws)
    assert M.moe_get_device_error() == M.MOE_DEVERR_EXPERT_RANGE
    flat = idx.ravel()
    valid = np.nonzero((flat >= 0) & (flat < E))[0]
    order = valid[np.argsort(flat[valid], kind="stable")]      # rows: valid slots by (expert, slot)
    cnt = np.bincount(flat[valid], minlength=E)
    np.testing.assert_array_equal(host(counts), cnt)
    np.testing.assert_array_equal(host(offsets), np.concatenate([[0], np.cumsum(cnt)]))
    np.testing.assert_array_equal(host(perm)[:valid.size], order)
    inv_r = np.full(S, -1, np.int32)
    inv_r[order] = np.arange(valid.size)
    np.testing.assert_array_equal(host(inv), inv_r)
    rng = np.random.default_rng(5)
    rows = rng.normal(0, 1, (S, d)).astype(np.float32)
    gates = rng.uniform(0, 1, (T, k)).astype(np.float32)
    y = torch.empty((T, d), dtype=torch.float32, device=DEV)
    M.moe_combine(dims, dev(rows), inv, dev(gates), None, y)
    ref = np.zeros((T, d), np.float64)
    for t in range(T):
        for j in range(k):
            r = inv_r[t * k + j]
            if r >= 0:
                ref[t] += np.float64(gates[t, j]) * rows[r]
    np.testing.assert_allclose(host(y), ref, rtol=1e-5, atol=1e-5)


# ---- the decode kernel's one inter-CTA wait ---------------------------------------

def _decode_case(T=8):
    return Case(synth.CONFIGS["decode"].with_T(T))


def test_decode_wait_timeout_reports_and_recovers():
    """A down tile waits for its expert's gate/up tiles. With the test hook the
    wait asks for one tile more than exist and gives up after 1 ms: the call
    reports MOE_DEVERR_TIMEOUT promptly (every role of a CTA leaves when one
    fails, instead of waiting out the 2 s limit), and the next call with the
    defaults restored is clean and matches the oracle."""
    c = _decode_case()
    cfg = c.cfg
    y = torch.empty((cfg.T, cfg.d), dtype=torch.float32, device=DEV)
    M.moe_layer(c.dims, c.weights, c.x_d, None, y, c.ws)   # warm: attributes, tensor maps, code
    assert M.moe_get_device_error() == 0
    try:
        M.moe_debug_set_wait(1_000_000, 1)
        t0 = time.perf_counter()
        M.moe_layer(c.dims, c.weights, c.x_d, None, y, c.ws)
        code = M.moe_get_device_error()
        dt = time.perf_counter() - t0
    finally:
        M.moe_debug_set_wait(0, 0)
    assert code == M.MOE_DEVERR_TIMEOUT
    assert dt < 1.0, f"the timed-out call took {dt:.3f} s"
    y.fill_(float("nan"))
    M.moe_layer(c.dims, c.weights, c.x_d, None, y, c.ws)
    assert M.moe_get_device_error() == 0
    toks = np.arange(cfg.T, dtype=np.int32)
    _, _, ref = oracle.layer_tokens(c.ora, c.x, toks)
    assert_rel(host(y), ref, TOL["bf16"], "decode after a timeout")


def test_two_decode_layers_on_two_streams():
    """Two decode layers (T = 8, distinct inputs and workspaces) issued
    alternately on two streams, so their kernels overlap and neither gets every
    SM: the work claim needs no co-residency, both match the oracle and no
    wait gives up."""
    from harness import host_weights
    cfg = synth.CONFIGS["decode"].with_T(8)
    x2 = synth.make_x(cfg, 0, 1)
    idx2, _ = oracle.topk_softmax(oracle.router_logits(x2, synth.make_router(cfg), synth.make_bias(cfg)), cfg.k)
    host_weights(cfg).ensure(np.unique(idx2))  # the second batch's experts too, before the device copy is packed
    c = _decode_case()
    ora = c.hw.oracle_layer(cfg, c.wr, c.bias, c.shared)
    ws2 = torch.empty_like(c.ws)
    x2_d = dev(x2)
    ya = torch.empty((cfg.T, cfg.d), dtype=torch.float32, device=DEV)
    yb = torch.empty((cfg.T, cfg.d), dtype=torch.float32, device=DEV)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    for _ in range(6):
        M.moe_layer(c.dims, c.weights, c.x_d, None, ya, c.ws, stream=s1)
        M.moe_layer(c.dims, c.weights, x2_d, None, yb, ws2, stream=s2)
    torch.cuda.synchronize()
    assert M.moe_get_device_error() == 0
    toks = np.arange(cfg.T, dtype=np.int32)
    _, _, ref_a = oracle.layer_tokens(ora, c.x, toks)
    _, _, ref_b = oracle.layer_tokens(ora, x2, toks)
    assert_rel(host(ya), ref_a, TOL["bf16"], "stream 1")
    assert_rel(host(yb), ref_b, TOL["bf16"], "stream 2")


@pytest.mark.parametrize("name", ["decode", "q2k"])
def test_decode_wide_range_activations(name):
    """Activations spanning twelve binades within a token (N(0, 1) times
    2^u, u uniform in [-10, 2]): the decode kernel's per-token power-of-two
    prescale (f16 for MXFP4; the 16-bit integer split for the Q2_K main term,
    exact within 2^7 of the token's largest element) keeps the layer within
    the w4a16 bound of the fp64 oracle."""
    from harness import host_weights
    cfg = synth.CONFIGS[name].with_T(2)
    rng = np.random.default_rng(77)
    xf = (rng.standard_normal((cfg.T, cfg.d)) * np.exp2(rng.uniform(-10, 2, (cfg.T, cfg.d)))).astype(np.float32)
    xw = (xf.view(np.uint32) >> 16).astype(np.uint16)            # bf16 by truncation: exact bits, any rounding will do
    idx, _ = oracle.topk_softmax(oracle.router_logits(xw, synth.make_router(cfg), synth.make_bias(cfg)), cfg.k)
    host_weights(cfg).ensure(np.unique(idx))   # the experts this batch routes to, before the device copy is packed
    c = Case(cfg)
    ora = c.hw.oracle_layer(cfg, c.wr, c.bias, c.shared)
    y = torch.empty((cfg.T, cfg.d), dtype=torch.float32, device=DEV)
    M.moe_layer(c.dims, c.weights, dev(xw), None, y, c.ws)
    assert M.moe_get_device_error() == 0
    toks = np.arange(cfg.T, dtype=np.int32)
    got_idx, _, ref = oracle.layer_tokens(ora, xw, toks)
    np.testing.assert_array_equal(got_idx, idx)
    assert_rel(host(y), ref, TOL["bf16"], f"{name} wide-range x")


# ---- the batch router on the tensor cores ------------------------------------------

def _router_bound(x, wnorm, approx, bias, d):
    """The documented bound B of |approx - canonical| (fp64, from the same
    inputs the kernel uses: the fp32 norms it reports, the approximate logits)."""
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    nx = np.sqrt((xf * xf).sum(axis=1)) * (1 + 2.0 ** -8)
    b = np.zeros(approx.shape[1]) if bias is None else np.abs(bias.astype(np.float64))
    return ((d * 2.0 ** -21 * nx[:, None] * (wnorm.astype(np.float64) * (1 + 2.0 ** -8))[None, :]
             + 2.0 ** -20 * (np.abs(approx) + b[None, :]) + 2.0 ** -100) * (1 + 2.0 ** -8))


def _approx(cfg, x, wr, bias):
    dims = M.make_dims(cfg.T, cfg.d, cfg.F, cfg.E, cfg.k)
    w = M.make_weights(None, None, None, w_router=dev(wr), router_bias=None if bias is None else dev(bias))
    a = torch.empty((cfg.T, cfg.E), dtype=torch.float32, device=DEV)
    n = torch.empty(cfg.E, dtype=torch.float32, device=DEV)
    M.moe_debug_router_approx(dims, dev(x), w, a, n)
    assert M.moe_get_device_error() == 0
    return host(a).astype(np.float64), host(n)


@pytest.mark.parametrize("case", ["prefill", "cancel"])
def test_router_approx_within_its_bound(case):
    """The tensor-core logits stay inside the bound the router relies on, with
    room to spare: on the Zipf-biased prefill batch, and on rows built for
    cancellation (large entries of both signs beside small ones)."""
    if case == "prefill":
        cfg = synth.CONFIGS["prefill"]
        x, wr, bias = synth.make_x(cfg), synth.make_router(cfg), synth.make_bias(cfg)
    else:
        cfg = synth.LayerConfig("cancel", T=256, d=4096, F=256, E=64, k=8)
        rng = np.random.default_rng(11)
        xf = rng.normal(0, 1, (cfg.T, cfg.d)).astype(np.float32)
        big = rng.integers(0, cfg.d, (cfg.T, 64))
        np.put_along_axis(xf, big, (rng.choice([-1, 1], big.shape) * 3e3).astype(np.float32), axis=1)
        x = (xf.view(np.uint32) >> 16).astype(np.uint16)
        wr, bias = synth.make_router(cfg), None
    a, wn = _approx(cfg, x, wr, bias)
    exact = oracle.router_logits(x, wr, bias).astype(np.float64)
    B = _router_bound(x, wn, a, bias, cfg.d)
    ratio = np.abs(a - exact) / B
    assert ratio.max() <= 0.5, f"approximate logits use {ratio.max():.3f} of their bound"


@pytest.mark.parametrize("T", [40, 300])
def test_route_tc_near_ties_and_ties(T):
    """Experts whose router rows differ by one bf16 ulp in one element (their
    canonical logits differ in the last bits, far inside the tensor-core error
    bound) and exact duplicates (equal logits: the lower index wins), through
    the batch router: the expert choice is the oracle's, bit for bit."""
    cfg = synth.LayerConfig("nearties", T=T, d=512, F=256, E=32, k=4)
    wr = synth.make_router(cfg)
    rng = np.random.default_rng(12)
    for grp in range(4):
        base = wr[grp]
        for j in range(1, 6):
            e = grp + 4 * j
            wr[e] = base
            if j % 2:
                i = rng.integers(0, cfg.d)
                wr[e, i] = base[i] + 1 if j % 4 == 1 else base[i] - 1   # one ulp of one element
    x = synth.make_x(cfg)
    idx_ref, w_ref = oracle.topk_softmax(oracle.router_logits(x, wr), cfg.k)
    dims = M.make_dims(cfg.T, cfg.d, cfg.F, cfg.E, cfg.k)
    ws = torch.empty(M.moe_workspace_size(dims), dtype=torch.uint8, device=DEV)
    weights = M.make_weights(None, None, None, w_router=dev(wr))
    idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=DEV)
    w = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device=DEV)
    M.moe_route(dims, dev(x), weights, None, idx, w, ws)
    assert M.moe_get_device_error() == 0
    np.testing.assert_array_equal(host(idx), idx_ref)
    np.testing.assert_allclose(host(w), w_ref, rtol=0, atol=2e-6)

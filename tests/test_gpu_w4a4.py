"""w4a4: MXFP4 activations against MXFP4 weights (kind::mxf4 on the tensor
cores; the generic CUDA-core path for other shapes and Q2_K weights).

x's MXFP4 codes and scale atoms are compared byte for byte with the oracle's
quantiser. Layer outputs are compared within 2e-2 * max|ref|: the x codes are
exact, but h is formed in fp32 on the GPU and in fp64 in the oracle, so an h
element that lies within rounding distance of an E2M1 decision boundary may
take the neighbouring code (one E2M1 step, at most a third of the element's
magnitude); a handful of such elements in a row of d_ff = 2048 moves an output
by well under 1% of max|ref| each.
"""
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
TOL = 2e-2


def dev(a):
    if a.dtype == np.uint16:
        a = a.astype(np.int16)
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def rel_err(got, ref):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    assert np.all(np.isfinite(got))
    return np.abs(got - ref).max() / np.abs(ref).max()


@pytest.mark.parametrize("T,d,E,k", [(300, 512, 8, 2), (600, 4096, 64, 8)])
def test_w4a4_staging_bitexact(T, d, E, k):
    """MXFP4 codes (two per byte) and E8M0 scale atoms of every routed row."""
    rng = np.random.default_rng(50 + T)
    x = synth.normal_bf16(0, 93, 0, T * d).reshape(T, d)
    x[0, :32] = 0
    x[0, 32:64] = 0x8000                                                 # -0.0
    x[1, :32] = rng.integers(1, 0x7F, 32).astype(np.uint16)              # subnormals
    x[2, :32] = (np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 4.0] * 4, np.float32).view(np.uint32)
                 >> 16).astype(np.uint16)                                # E2M1 ties at scale 2^0
    x[3, :32] = 0x40E0 | rng.integers(0, 0x20, 32).astype(np.uint16)     # 7 .. 8: saturation at 6 x 2^0
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    counts, offsets, perm, _ = oracle.permute(idx, E)
    S = T * k
    dims = M.make_dims(T, d, 256, E, k, act=M.MOE_A_MXFP4)
    ws = torch.empty(M.moe_workspace_size(dims), dtype=torch.uint8, device=DEV)
    tiles = (S + 127) // 128 + E
    codes = torch.zeros((S, d // 2), dtype=torch.uint8, device=DEV)
    atoms = torch.zeros((tiles, d // 128, 512), dtype=torch.uint8, device=DEV)
    ustart = torch.zeros(E + 1, dtype=torch.int32, device=DEV)
    M.moe_debug_tc_gather(dims, dev(x), dev(offsets), dev(perm), codes, atoms, ustart, ws)
    assert M.moe_get_device_error() == 0
    xc, xs = oracle.mxfp4_quantize((x.astype(np.uint32) << 16).view(np.float32))
    tok = perm // k
    np.testing.assert_array_equal(codes.cpu().numpy(), xc[tok])
    us = np.concatenate([[0], np.cumsum((counts + 127) // 128)]).astype(np.int32)
    at = atoms.cpu().numpy().reshape(-1)
    e_of_row = np.repeat(np.arange(E), counts)
    rloc = np.arange(S) - offsets[e_of_row]
    tile = us[e_of_row] + rloc // 128
    b = np.arange(d // 32)
    pos = ((tile[:, None] * (d // 128) + b[None, :] // 4) * 512
           + (rloc[:, None] % 32) * 16 + ((rloc[:, None] % 128) // 32) * 4 + b[None, :] % 4)
    np.testing.assert_array_equal(at[pos], xs[tok])


CASES = [
    ("tc-small", synth.LayerConfig("w4a4", T=300, d=256, F=512, E=8, k=3, act="mxfp4")),
    ("tc-prefill", replace(synth.CONFIGS["prefill"], T=384, act="mxfp4")),
    ("tc-hash", replace(synth.CONFIGS["hash"], T=512, act="mxfp4")),
    ("generic-q2k", synth.LayerConfig("w4a4q", T=37, d=512, F=256, E=8, k=2, wfmt="q2k", act="mxfp4")),
    ("generic-decode", replace(synth.CONFIGS["decode"], T=4, act="mxfp4")),
]


@pytest.mark.parametrize("name,cfg", CASES, ids=[n for n, _ in CASES])
def test_w4a4_layer_and_rows(name, cfg):
    c = Case(cfg, experts="all" if cfg.E <= 16 else "routed")
    y = torch.empty((cfg.T, cfg.d), dtype=torch.float32, device=DEV)
    M.moe_layer(c.dims, c.weights, c.x_d, c.tok_d, y, c.ws)
    assert M.moe_get_device_error() == 0
    toks = np.arange(min(cfg.T, 48), dtype=np.int32)
    idx, _, ref = oracle.layer_tokens(c.ora, c.x, toks, c.token_ids)
    np.testing.assert_array_equal(idx, c.ora_idx[toks])
    err = rel_err(y.cpu().numpy()[toks], ref)
    assert err <= TOL, f"{name}: layer max|err| = {err:.2e} max|ref|"
    _, offsets, perm, _ = oracle.permute(c.ora_idx, cfg.E)
    S = cfg.T * cfg.k
    out = torch.full((S, cfg.d), float("nan"), dtype=torch.float32, device=DEV)
    M.moe_expert_ffn(c.dims, c.weights, c.x_d, dev(offsets), dev(perm), out, c.ws)
    assert M.moe_get_device_error() == 0
    rows = np.arange(S) if S <= 1024 else np.unique(np.concatenate([np.arange(64), np.arange(S - 64, S)]))
    got = out.cpu().numpy()
    ref_rows = np.concatenate([oracle.expert_ffn_rows(c.ora, c.x, offsets, perm, int(r), int(r) + 1) for r in rows]) \
        if S > 1024 else oracle.expert_ffn_rows(c.ora, c.x, offsets, perm, 0, S)
    err = rel_err(got[rows], ref_rows)
    assert err <= TOL, f"{name}: rows max|err| = {err:.2e} max|ref|"

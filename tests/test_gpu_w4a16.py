"""w4a16 on the tensor cores: bf16 activations against MXFP4 weights decoded
into tensor memory (kind::f16), for every batch the decode kernel does not take
(T > 8, or dims other than d_model 4096 / d_ff 2048). Every routed row, and the
layer, against the oracle within the w4a16 bound 2e-3 * max|ref|.
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
TOL = 2e-3


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def rel_err(got, ref):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    assert np.all(np.isfinite(got))
    return np.abs(got - ref).max() / np.abs(ref).max()


CASES = [
    ("small-ragged", synth.LayerConfig("w4a16", T=300, d=256, F=512, E=8, k=3)),
    ("small-one-token", synth.LayerConfig("w4a16", T=1, d=512, F=256, E=4, k=2)),
    ("decode-dims-T9", replace(synth.CONFIGS["decode"], T=9)),     # one token past the decode kernel
    ("decode-dims-T31", replace(synth.CONFIGS["decode"], T=31)),    # below the tensor-core router
    ("decode-dims-T64", replace(synth.CONFIGS["decode"], T=64)),
    ("prefill-dims", replace(synth.CONFIGS["prefill"], T=384, act="bf16")),
]


@pytest.mark.parametrize("name,cfg", CASES, ids=[n for n, _ in CASES])
def test_w4a16_tensor_core_rows_and_layer(name, cfg):
    c = Case(cfg, experts="all" if cfg.E <= 16 else "routed")
    _, offsets, perm, _ = oracle.permute(c.ora_idx, cfg.E)
    S = cfg.T * cfg.k
    out = torch.full((S, cfg.d), float("nan"), dtype=torch.float32, device=DEV)
    M.moe_expert_ffn(c.dims, c.weights, c.x_d, dev(offsets), dev(perm), out, c.ws)
    assert M.moe_get_device_error() == 0
    got = out.cpu().numpy()
    rows = np.arange(S) if S <= 1024 else np.unique(np.concatenate([np.arange(96), np.arange(S - 96, S)]))
    ref = (oracle.expert_ffn_rows(c.ora, c.x, offsets, perm, 0, S) if S <= 1024 else
           np.concatenate([oracle.expert_ffn_rows(c.ora, c.x, offsets, perm, int(r), int(r) + 1) for r in rows]))
    assert rel_err(got[rows], ref) <= TOL, name
    y = torch.empty((cfg.T, cfg.d), dtype=torch.float32, device=DEV)
    M.moe_layer(c.dims, c.weights, c.x_d, c.tok_d, y, c.ws)
    assert M.moe_get_device_error() == 0
    toks = np.arange(min(cfg.T, 48), dtype=np.int32)
    idx, _, ly = oracle.layer_tokens(c.ora, c.x, toks, c.token_ids)
    np.testing.assert_array_equal(idx, c.ora_idx[toks])
    assert rel_err(y.cpu().numpy()[toks], ly) <= TOL, name

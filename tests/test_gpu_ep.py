"""Expert-parallel layer on one GPU: the ranks of an N-way split, run one after
another (none waits for another), each with only its own experts' weights.

The sum of the ranks' partial outputs is the whole layer: it matches the
oracle within the layer's tolerance, and moe_layer's own output up to the
order of the fp32 sums. Each partial also matches the oracle's sum over that
rank's experts. Covers the fused decode path, Q2_K decode, the tensor-core
w4a8 path and hash routing.
"""
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


def local_weights(c, b, e):
    """Packed routed weights of experts [b, e) only (what rank b..e holds)."""
    cfg = c.cfg
    dl = M.make_dims(cfg.T, cfg.d, cfg.F, e - b, cfg.k, c.dims.route, c.dims.act, c.dims.wfmt, 0)
    packed = {}
    for t, which in ((synth.W1, M.MOE_MAT_W1), (synth.W3, M.MOE_MAT_W3), (synth.W2, M.MOE_MAT_W2)):
        a, s = c.hw.arr[t]
        blob = a[b:e].ravel() if s is None else np.concatenate([a[b:e].ravel(), s[b:e].ravel()])
        out = torch.empty(M.moe_packed_size(dl, which), dtype=torch.uint8, device=DEV)
        M.moe_pack_weights(dl, which, torch.from_numpy(np.ascontiguousarray(blob)).to(DEV), out)
        packed[which] = out
    return packed


def oracle_partial(c, toks, b, e, add_shared):
    cfg = c.cfg
    y = np.zeros((len(toks), cfg.d))
    for i, t in enumerate(toks):
        for j in range(cfg.k):
            ex = int(c.ora_idx[t, j])
            if b <= ex < e:
                y[i] += float(c.ora_w[t, j]) * oracle.expert_ffn_token(c.ora, ex, c.x[t])
        if add_shared and c.shared is not None:
            y[i] += oracle.shared_ffn_token(c.ora, c.x[t])
    return y


CASES = [("decode", 8, 4), ("decode", 1, 8), ("q2k", 8, 2), ("prefill", 256, 4), ("hash", 512, 3)]


@pytest.mark.parametrize("name,T,world", CASES)
def test_expert_parallel_ranks_sum_to_the_layer(name, T, world):
    cfg = synth.CONFIGS[name].with_T(T)
    c = Case(cfg)  # the experts no token routes to stay zero: no rank reads them
    full = torch.empty((T, cfg.d), dtype=torch.float32, device=DEV)
    M.moe_layer(c.dims, c.weights, c.x_d, c.tok_d, full, c.ws)
    total = np.zeros((T, cfg.d))
    toks = np.arange(min(T, 24), dtype=np.int32)
    for r in range(world):
        b, e = M.moe_ep_range(cfg.E, r, world)
        p = local_weights(c, b, e)
        sh = [c.sh_d[i] if r == 0 else None for i in range(3)]
        w = M.make_weights(p[1], p[3], p[2], *sh, c.wr_d, c.bias_d)
        y = torch.full((T, cfg.d), float("nan"), dtype=torch.float32, device=DEV)
        M.moe_layer_ep(c.dims, w, b, e, r == 0, c.x_d, c.tok_d, y, c.ws)
        assert M.moe_get_device_error() == 0
        yp = y.cpu().numpy()
        assert np.all(np.isfinite(yp))
        ref = oracle_partial(c, toks, b, e, r == 0)
        scale = max(np.abs(ref).max(), 1e-30)
        assert np.abs(yp[toks] - ref).max() <= TOL[cfg.act] * scale, f"rank {r} of {world}"
        total += yp
        del p, w
    f = full.cpu().numpy()
    assert np.abs(total - f).max() <= 1e-5 * np.abs(f).max()
    _, _, ref = oracle.layer_tokens(c.ora, c.x, toks, c.token_ids)
    assert np.abs(total[toks] - ref).max() <= TOL[cfg.act] * np.abs(ref).max()


def test_expert_parallel_arguments():
    dims = M.make_dims(8, 4096, 2048, 256, 8, d_ff_shared=2048)
    assert M.moe_ep_range(256, 0, 8) == (0, 32) and M.moe_ep_range(256, 7, 8) == (224, 256)
    assert M.moe_ep_range(10, 2, 3) == (6, 10)
    for bad in ((0, 0), (5, 3), (-1, 4), (0, 257)):
        with pytest.raises(M.MoeError):
            M.moe_layer_ep(dims, M.make_weights(0x100, 0x100, 0x100), bad[0], bad[1], 0, 0x100, None, 0x100, 0x100)

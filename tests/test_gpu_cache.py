"""Routed experts from pinned host memory through a cache of expert slots in HBM.

One wave (the cache holds every expert the batch touches) gives moe_layer's
result bit for bit, with a second batch finding some experts cached and copying
the rest; a cache smaller than the batch's expert set runs the batch in waves
and matches moe_layer up to the order of the fp32 sums, and the oracle within
the layer tolerance. Decode (bf16, MXFP4 and Q2_K) and the w4a8 tensor-core path.
"""
import numpy as np
import pytest

import oracle
import synth
from harness import Case, host_weights

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import routed_expert_ffn_05_b200 as M  # noqa: E402

DEV = torch.device("cuda:0")
TOL = {"bf16": 2e-3, "mxfp8": 1e-2}


def make_cache(c, slots):
    cfg = c.cfg
    host = [torch.empty(c.packed[w].numel(), dtype=torch.uint8).pin_memory() for w in (1, 3, 2)]
    for h, w in zip(host, (1, 3, 2)):
        h.copy_(c.packed[w].cpu())
    dl = M.make_dims(cfg.T, cfg.d, cfg.F, slots, cfg.k, c.dims.route, c.dims.act, c.dims.wfmt, 0)
    dev = [torch.empty(M.moe_packed_size(dl, w), dtype=torch.uint8, device=DEV) for w in (1, 3, 2)]
    return M.moe_cache_create(c.dims, slots, *host, *dev)


def run_both(c, cache, x_d, tok_d):
    cfg = c.cfg
    ref = torch.empty((cfg.T, cfg.d), dtype=torch.float32, device=DEV)
    got = torch.full((cfg.T, cfg.d), float("nan"), dtype=torch.float32, device=DEV)
    M.moe_layer(c.dims, c.weights, x_d, tok_d, ref, c.ws)
    cache.layer(c.dims, c.weights, x_d, tok_d, got, c.ws)
    torch.cuda.synchronize()
    assert M.moe_get_device_error() == 0
    return ref.cpu().numpy(), got.cpu().numpy()


def ensure_batches(cfg, batches):
    """The host weights must hold every expert the batches touch before the
    device copy is packed."""
    hw = host_weights(cfg)
    for b in batches:
        x = synth.make_x(cfg, 0, b)
        if cfg.route == "hash":
            idx, _, _ = oracle.hash_route(synth.make_token_ids(cfg, 0, b), cfg.E, cfg.k)
        else:
            idx, _ = oracle.topk_softmax(oracle.router_logits(x, synth.make_router(cfg), synth.make_bias(cfg)), cfg.k)
        hw.ensure(np.unique(idx))


@pytest.mark.parametrize("name,T,slots", [("decode", 8, 64), ("q2k", 1, 8)])
def test_cache_one_wave_is_moe_layer_bit_for_bit(name, T, slots):
    cfg = synth.CONFIGS[name].with_T(T)
    ensure_batches(cfg, (0, 1, 2))
    c = Case(cfg)
    cache = make_cache(c, slots)
    U = []
    for b in (0, 1, 2, 0):
        x = torch.from_numpy(synth.make_x(cfg, 0, b).astype(np.int16)).to(DEV)
        ref, got = run_both(c, cache, x, None)
        np.testing.assert_array_equal(got.view(np.uint32), ref.view(np.uint32))
        idx, _ = oracle.topk_softmax(oracle.router_logits(synth.make_x(cfg, 0, b), c.wr, c.bias), cfg.k)
        U.append(len(np.unique(idx)))
    st = cache.stats()
    assert st["calls"] == 4 and st["waves"] == 4
    assert st["hits"] + st["misses"] == sum(U)
    assert st["misses"] >= U[0] and st["hits"] > 0  # the first batch copies all; the repeat finds some cached
    per = sum(M.moe_packed_size(M.make_dims(1, cfg.d, cfg.F, 1, 1, wfmt=c.dims.wfmt), w) for w in (1, 3, 2))
    assert st["bytes_h2d"] <= st["misses"] * per


@pytest.mark.parametrize("name,T,slots", [("decode", 8, 16), ("prefill", 256, 64), ("hash", 256, 40)])
def test_cache_smaller_than_the_batch_runs_waves(name, T, slots):
    cfg = synth.CONFIGS[name].with_T(T)
    c = Case(cfg)
    cache = make_cache(c, slots)
    ref, got = run_both(c, cache, c.x_d, c.tok_d)
    U = len(np.unique(c.ora_idx))
    assert U > slots
    st = cache.stats()
    assert st["waves"] == -(-U // slots) and st["misses"] == U
    assert np.abs(got - ref).max() <= 1e-5 * np.abs(ref).max()
    toks = np.arange(min(T, 16), dtype=np.int32)
    _, _, ora = oracle.layer_tokens(c.ora, c.x, toks, c.token_ids)
    assert np.abs(got[toks] - ora).max() <= TOL[cfg.act] * np.abs(ora).max()


def test_cache_arguments():
    dims = M.make_dims(8, 4096, 2048, 256, 8, d_ff_shared=2048)
    with pytest.raises(M.MoeError):
        M.moe_cache_create(dims, 0, 0x100, 0x100, 0x100, 0x100, 0x100, 0x100)
    with pytest.raises(M.MoeError):
        M.moe_cache_create(dims, 257, 0x100, 0x100, 0x100, 0x100, 0x100, 0x100)
    with pytest.raises(M.MoeError):  # device buffers must be 256-byte aligned
        M.moe_cache_create(dims, 8, 0x100, 0x100, 0x100, 0x101, 0x100, 0x100)

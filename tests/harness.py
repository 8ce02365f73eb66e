"""Test harness: one layer instance on the host (oracle side) and the device.

Inputs come from ``synth`` (seeded); routed-expert weights are quantised on the
host by the oracle's encoder, uploaded in the canonical layout and packed on the
device by ``moe_pack_weights``. Nothing the oracle sees comes from the device.
Experts are generated lazily, so decode-sized tests only build the experts the
oracle's routing touches.
"""
from __future__ import annotations

import numpy as np

import oracle
import synth

_MATS = {synth.W1: 1, synth.W3: 3, synth.W2: 2}  # synth tensor id -> MOE_MAT_*


class HostWeights:
    """Canonical routed-expert weights of one config, filled expert by expert."""

    def __init__(self, cfg, seed=0):
        self.cfg, self.seed = cfg, seed
        self.filled = set()
        E, F, d = cfg.E, cfg.F, cfg.d
        self.arr = {}
        for t in (synth.W1, synth.W3, synth.W2):
            N, K = (F, d) if t != synth.W2 else (d, F)
            if cfg.wfmt == "q2k":
                self.arr[t] = (np.zeros((E, N, K // 256 * 84), np.uint8), None)
            else:
                self.arr[t] = (np.zeros((E, N, K // 2), np.uint8), np.zeros((E, N, K // 32), np.uint8))

    def ensure(self, experts):
        todo = sorted(set(int(e) for e in experts) - self.filled)
        for e in todo:
            for t in (synth.W1, synth.W3, synth.W2):
                w = synth.expert_weight_f32(self.cfg, self.seed, e, t)
                a, b = oracle.quantize_expert(self.cfg, w)
                self.arr[t][0][e] = a
                if b is not None:
                    self.arr[t][1][e] = b
            self.filled.add(e)

    def canonical_bytes(self, t) -> np.ndarray:
        a, b = self.arr[t]
        return np.concatenate([a.ravel(), b.ravel()]) if b is not None else a.ravel()

    def oracle_layer(self, cfg, wr=None, bias=None, shared=None) -> oracle.LayerWeights:
        (c1, s1), (c3, s3), (c2, s2) = (self.arr[t] for t in (synth.W1, synth.W3, synth.W2))
        kw = {}
        if shared is not None:
            kw = dict(sw1=shared[0], sw3=shared[1], sw2=shared[2])
        return oracle.LayerWeights(cfg, c1, s1, c3, s3, c2, s2, wr=wr, bias=bias, **kw)


_weights_cache = {}


def host_weights(cfg, seed=0) -> HostWeights:
    key = (cfg.d, cfg.F, cfg.E, cfg.wfmt, seed)
    if key not in _weights_cache:
        _weights_cache[key] = HostWeights(cfg, seed)
    return _weights_cache[key]


class Case:
    """A layer config with its seeded inputs on host and device."""

    def __init__(self, cfg, seed=0, batch=0, experts="routed", router_fn=None):
        import torch
        import routed_expert_ffn_05_b200 as M
        self.M, self.cfg, self.seed = M, cfg, seed
        self.x = synth.make_x(cfg, seed, batch)
        self.token_ids = synth.make_token_ids(cfg, seed, batch) if cfg.route == "hash" else None
        self.wr = synth.make_router(cfg, seed) if cfg.has_router else None
        if router_fn is not None:  # a test's edit of the router rows (ties and the like)
            router_fn(self.wr)
        self.bias = synth.make_bias(cfg, seed)
        self.shared = synth.shared_weights_bf16(cfg, seed)
        self.hw = host_weights(cfg, seed)
        # experts the layer touches, from the oracle's routing
        self.ora_idx, self.ora_w = self.oracle_route()
        self.hw.ensure(range(cfg.E) if experts == "all" else np.unique(self.ora_idx))
        self.ora = self.hw.oracle_layer(cfg, self.wr, self.bias, self.shared)
        self.dims = M.make_dims(cfg.T, cfg.d, cfg.F, cfg.E, cfg.k,
                                M.MOE_ROUTE_HASH if cfg.route == "hash" else M.MOE_ROUTE_SOFTMAX_TOPK,
                                {"mxfp8": M.MOE_A_MXFP8, "mxfp4": M.MOE_A_MXFP4}.get(cfg.act, M.MOE_A_BF16),
                                M.MOE_W_Q2K if cfg.wfmt == "q2k" else M.MOE_W_MXFP4,
                                cfg.Fs if self.shared is not None else 0)
        dev = torch.device("cuda:0")
        t16 = lambda a: torch.from_numpy(a.astype(np.int16)).to(dev) if a is not None else None
        self.x_d = t16(self.x)
        self.tok_d = torch.from_numpy(self.token_ids).to(dev) if self.token_ids is not None else None
        self.wr_d = t16(self.wr)
        self.bias_d = torch.from_numpy(self.bias).to(dev) if self.bias is not None else None
        self.sh_d = [t16(a) for a in self.shared] if self.shared is not None else [None] * 3
        self.packed = {}
        for t, which in _MATS.items():
            canon = torch.from_numpy(self.hw.canonical_bytes(t)).to(dev)
            out = torch.empty(M.moe_packed_size(self.dims, which), dtype=torch.uint8, device=dev)
            M.moe_pack_weights(self.dims, which, canon, out)
            self.packed[which] = out
            del canon
        self.weights = M.make_weights(self.packed[1], self.packed[3], self.packed[2], *self.sh_d,
                                      self.wr_d, self.bias_d)
        self.ws = torch.empty(max(M.moe_workspace_size(self.dims), 256), dtype=torch.uint8, device=dev)
        torch.cuda.synchronize()

    def oracle_route(self):
        cfg = self.cfg
        if cfg.route == "hash":
            idx, w, failed = oracle.hash_route(self.token_ids, cfg.E, cfg.k)
            assert failed == 0
            return idx, w
        return oracle.topk_softmax(oracle.router_logits(self.x, self.wr, self.bias), cfg.k)


def bf16_to_f32(a: np.ndarray) -> np.ndarray:
    return (a.astype(np.uint32) << 16).view(np.float32)

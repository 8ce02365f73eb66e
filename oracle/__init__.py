"""Oracle for the routed MoE FFN layer: ctypes binding to the plain C oracle.

TEST INFRASTRUCTURE. Only the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package; the CUDA library never
uses it and shares no code with it. Each C function cites the definition it
follows (see ``oracle.h`` and the ``*.c`` files).

Parity status: every function is pinned by a ``-m "not gpu"`` test against the
format definitions, brute force, closed forms, library routines or an
independently coded dense FFN; the SplitMix64 draws of hash routing are pinned
draw by draw against a library implementation of the generator.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRCS = ["formats.c", "route.c", "permute.c", "ffn.c"]
_SO = os.path.join(_HERE, "liboracle.so")

W_MXFP4, W_Q2K = 1, 2
A_BF16, A_MXFP8, A_MXFP4 = 0, 1, 2
ROUTE_SOFTMAX, ROUTE_HASH = 0, 1
Q2K_BLOCK, Q2K_BYTES = 256, 84
MAX_DRAWS = 1024


def build(force: bool = False) -> str:
    """Compile liboracle.so: gcc -O2, OpenMP, no FP contraction (fmaf is explicit)."""
    srcs = [os.path.join(_HERE, s) for s in _SRCS]
    deps = srcs + [os.path.join(_HERE, "oracle.h")]
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < max(map(os.path.getmtime, deps)):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                               "-ffp-contract=off", "-fno-fast-math", *srcs, "-o", tmp, "-lm"])
        os.replace(tmp, _SO)
    return _SO


class Layer(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("T", "d", "F", "E", "k", "wfmt", "act", "route", "Fs", "max_draws")] + \
               [(n, ctypes.c_void_p) for n in
                ("w1", "w1s", "w3", "w3s", "w2", "w2s", "sw1", "sw3", "sw2", "wr", "bias")]


_L = None


def lib():
    global _L
    if _L is None:
        build()
        L = ctypes.CDLL(_SO)
        vp, i32, i64, u8, u16, f64 = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                                      ctypes.c_uint8, ctypes.c_uint16, ctypes.c_double)
        sig = {
            "ora_e2m1_value": (f64, [u8]), "ora_e8m0_value": (f64, [u8]),
            "ora_e4m3_value": (f64, [u8]), "ora_e2m1_encode": (u8, [f64]),
            "ora_e2m1_encode_nearest": (u8, [f64]), "ora_e4m3_encode": (u8, [f64]),
            "ora_e4m3_encode_nearest": (u8, [f64]), "ora_floor_log2": (i32, [f64]),
            "ora_f32_to_f16": (u16, [ctypes.c_float]), "ora_f16_value": (f64, [u16]),
            "ora_f64_to_bf16": (u16, [f64]), "ora_bf16_value": (f64, [u16]),
            "ora_mxfp4_quantize": (None, [vp, i64, i64, vp, vp]),
            "ora_mxfp4_dequantize": (None, [vp, vp, i64, i64, vp]),
            "ora_mxfp4_quantize_f64": (None, [vp, i64, i64, vp, vp]),
            "ora_mxfp8_quantize_f64": (None, [vp, i64, i64, vp, vp]),
            "ora_mxfp8_quantize_bf16": (None, [vp, i64, i64, vp, vp]),
            "ora_mxfp8_dequantize": (None, [vp, vp, i64, i64, vp]),
            "ora_q2k_quantize": (None, [vp, i64, i64, vp]),
            "ora_q2k_dequantize": (None, [vp, i64, i64, vp]),
            "ora_router_logits": (None, [vp, vp, vp, i32, i32, i32, vp]),
            "ora_topk_softmax": (None, [vp, i32, i32, i32, vp, vp]),
            "ora_splitmix64_next": (ctypes.c_uint64, [vp]),
            "ora_hash_route": (i32, [vp, i32, i32, i32, i32, vp, vp]),
            "ora_permute": (i32, [vp, i32, i32, i32, vp, vp, vp, vp]),
            "ora_expert_ffn_token": (None, [vp, i32, vp, vp]),
            "ora_shared_ffn_token": (None, [vp, vp, vp]),
            "ora_expert_ffn_rows": (None, [vp, vp, vp, vp, i64, i64, vp]),
            "ora_combine": (None, [vp, vp, vp, vp, i32, i32, i32, vp]),
            "ora_layer_tokens": (i32, [vp, vp, vp, vp, i32, vp, vp, vp]),
            "ora_num_threads": (i32, []),
            "ora_set_num_threads": (i32, [i32]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _L = L
    return _L


def _p(a):
    if a is None:
        return None
    assert isinstance(a, np.ndarray) and a.flags["C_CONTIGUOUS"], "need a C-contiguous array"
    return a.ctypes.data


def num_threads() -> int:
    return int(lib().ora_num_threads())


def set_num_threads(n: int) -> int:
    """OpenMP threads for later calls (threading only; results do not depend
    on it). Returns the count in effect."""
    return int(lib().ora_set_num_threads(int(n)))


# ---- formats ---------------------------------------------------------------

def e2m1_value(code: int) -> float:
    return lib().ora_e2m1_value(code)


def e8m0_value(e: int) -> float:
    return lib().ora_e8m0_value(e)


def e4m3_value(code: int) -> float:
    return lib().ora_e4m3_value(code)


def e2m1_encode(y: float) -> int:
    return lib().ora_e2m1_encode(y)


def e2m1_encode_nearest(y: float) -> int:
    return lib().ora_e2m1_encode_nearest(y)


def e4m3_encode(y: float) -> int:
    return lib().ora_e4m3_encode(y)


def e4m3_encode_nearest(y: float) -> int:
    return lib().ora_e4m3_encode_nearest(y)


def f32_to_f16(v: float) -> int:
    return lib().ora_f32_to_f16(v)


def f16_value(h: int) -> float:
    return lib().ora_f16_value(h)


def f64_to_bf16(v: float) -> int:
    return lib().ora_f64_to_bf16(v)


def bf16_value(b: int) -> float:
    return lib().ora_bf16_value(b)


def mxfp4_quantize(w: np.ndarray):
    """fp32 [rows][K] -> (codes u8 [rows][K/2], scales u8 [rows][K/32])."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    rows, K = w.shape
    codes = np.empty((rows, K // 2), np.uint8)
    scales = np.empty((rows, K // 32), np.uint8)
    lib().ora_mxfp4_quantize(_p(w), rows, K, _p(codes), _p(scales))
    return codes, scales


def mxfp4_dequantize(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    rows, K = codes.shape[0], codes.shape[1] * 2
    out = np.empty((rows, K), np.float32)
    lib().ora_mxfp4_dequantize(_p(np.ascontiguousarray(codes)), _p(np.ascontiguousarray(scales)),
                               rows, K, _p(out))
    return out


def mxfp4_quantize_f64(v: np.ndarray):
    """fp64 [rows][K] -> (codes u8 [rows][K/2], scales u8 [rows][K/32]), the weights' MXFP4 rule."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    rows, K = v.shape
    codes = np.empty((rows, K // 2), np.uint8)
    scales = np.empty((rows, K // 32), np.uint8)
    lib().ora_mxfp4_quantize_f64(_p(v), rows, K, _p(codes), _p(scales))
    return codes, scales


def mxfp8_quantize_f64(v: np.ndarray):
    v = np.ascontiguousarray(v, dtype=np.float64)
    rows, K = v.shape
    codes = np.empty((rows, K), np.uint8)
    scales = np.empty((rows, K // 32), np.uint8)
    lib().ora_mxfp8_quantize_f64(_p(v), rows, K, _p(codes), _p(scales))
    return codes, scales


def mxfp8_quantize_bf16(x: np.ndarray):
    x = np.ascontiguousarray(x, dtype=np.uint16)
    rows, K = x.shape
    codes = np.empty((rows, K), np.uint8)
    scales = np.empty((rows, K // 32), np.uint8)
    lib().ora_mxfp8_quantize_bf16(_p(x), rows, K, _p(codes), _p(scales))
    return codes, scales


def mxfp8_dequantize(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    rows, K = codes.shape
    out = np.empty((rows, K), np.float64)
    lib().ora_mxfp8_dequantize(_p(np.ascontiguousarray(codes)), _p(np.ascontiguousarray(scales)),
                               rows, K, _p(out))
    return out


def q2k_quantize(w: np.ndarray) -> np.ndarray:
    """fp32 [rows][K] -> blocks u8 [rows][K/256*84]."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    rows, K = w.shape
    out = np.empty((rows, K // Q2K_BLOCK * Q2K_BYTES), np.uint8)
    lib().ora_q2k_quantize(_p(w), rows, K, _p(out))
    return out


def q2k_dequantize(blocks: np.ndarray, K: int) -> np.ndarray:
    rows = blocks.shape[0]
    out = np.empty((rows, K), np.float32)
    lib().ora_q2k_dequantize(_p(np.ascontiguousarray(blocks)), rows, K, _p(out))
    return out


# ---- routing / permute -----------------------------------------------------

def router_logits(x: np.ndarray, wr: np.ndarray, bias=None) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.uint16)
    wr = np.ascontiguousarray(wr, dtype=np.uint16)
    T, d = x.shape
    E = wr.shape[0]
    out = np.empty((T, E), np.float32)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    lib().ora_router_logits(_p(x), _p(wr), _p(b), T, d, E, _p(out))
    return out


def topk_softmax(logits: np.ndarray, k: int):
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = logits.shape
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    lib().ora_topk_softmax(_p(logits), T, E, k, _p(idx), _p(w))
    return idx, w


def splitmix64_outputs(seed: int, n: int):
    st = ctypes.c_uint64(seed)
    return [int(lib().ora_splitmix64_next(ctypes.addressof(st))) for _ in range(n)]


def hash_route(token_ids: np.ndarray, E: int, k: int, max_draws: int = MAX_DRAWS):
    tok = np.ascontiguousarray(token_ids, dtype=np.int32)
    T = tok.shape[0]
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    failed = lib().ora_hash_route(_p(tok), T, E, k, max_draws, _p(idx), _p(w))
    return idx, w, int(failed)


def permute(idx: np.ndarray, E: int):
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = idx.shape
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(T * k, np.int32)
    inv = np.empty(T * k, np.int32)
    rc = lib().ora_permute(_p(idx), T, k, E, _p(counts), _p(offsets), _p(perm), _p(inv))
    if rc != 0:
        raise ValueError("expert index out of range")
    return counts, offsets, perm, inv


# ---- layer -----------------------------------------------------------------

class LayerWeights:
    """Canonical weights of one layer, held as numpy arrays.

    MXFP4: w1/w3 codes [E][F][d/2] + scales [E][F][d/32]; w2 codes [E][d][F/2] +
    scales [E][d][F/32]. Q2_K: w1/w3 blocks [E][F][d/256*84], w2 [E][d][F/256*84].
    Shared expert bf16 bits: sw1/sw3 [Fs][d], sw2 [d][Fs]. Router bf16 [E][d].
    """

    def __init__(self, cfg, w1, w1s, w3, w3s, w2, w2s, sw1=None, sw3=None, sw2=None,
                 wr=None, bias=None):
        self.cfg = cfg
        self.w1, self.w1s, self.w3, self.w3s, self.w2, self.w2s = w1, w1s, w3, w3s, w2, w2s
        self.sw1, self.sw3, self.sw2, self.wr, self.bias = sw1, sw3, sw2, wr, bias

    def struct(self) -> Layer:
        c = self.cfg
        s = Layer()
        s.T, s.d, s.F, s.E, s.k = c.T, c.d, c.F, c.E, c.k
        s.wfmt = W_Q2K if c.wfmt == "q2k" else W_MXFP4
        s.act = {"mxfp8": A_MXFP8, "mxfp4": A_MXFP4}.get(c.act, A_BF16)
        s.route = ROUTE_HASH if c.route == "hash" else ROUTE_SOFTMAX
        s.Fs = c.Fs if self.sw1 is not None else 0
        s.max_draws = MAX_DRAWS
        for n in ("w1", "w1s", "w3", "w3s", "w2", "w2s", "sw1", "sw3", "sw2", "wr", "bias"):
            setattr(s, n, _p(getattr(self, n)))
        return s


def quantize_expert(cfg, w: np.ndarray):
    """Quantise one expert matrix in the config's format: (codes, scales) or (blocks, None)."""
    if cfg.wfmt == "q2k":
        return q2k_quantize(w), None
    return mxfp4_quantize(w)


def expert_ffn_token(weights: LayerWeights, e: int, x_t: np.ndarray) -> np.ndarray:
    s = weights.struct()
    x_t = np.ascontiguousarray(x_t, dtype=np.uint16)
    o = np.empty(weights.cfg.d, np.float64)
    lib().ora_expert_ffn_token(ctypes.byref(s), e, _p(x_t), _p(o))
    return o


def shared_ffn_token(weights: LayerWeights, x_t: np.ndarray) -> np.ndarray:
    s = weights.struct()
    x_t = np.ascontiguousarray(x_t, dtype=np.uint16)
    o = np.empty(weights.cfg.d, np.float64)
    lib().ora_shared_ffn_token(ctypes.byref(s), _p(x_t), _p(o))
    return o


def expert_ffn_rows(weights: LayerWeights, x: np.ndarray, offsets, perm, row_begin=0, row_end=None):
    s = weights.struct()
    x = np.ascontiguousarray(x, dtype=np.uint16)
    if row_end is None:
        row_end = int(offsets[-1])
    out = np.empty((row_end - row_begin, weights.cfg.d), np.float32)
    lib().ora_expert_ffn_rows(ctypes.byref(s), _p(x), _p(np.ascontiguousarray(offsets, np.int32)),
                              _p(np.ascontiguousarray(perm, np.int32)), row_begin, row_end, _p(out))
    return out


def combine(out_rows, inv_perm, topk_w, shared=None):
    out_rows = np.ascontiguousarray(out_rows, np.float32)
    topk_w = np.ascontiguousarray(topk_w, np.float32)
    T, k = topk_w.shape
    d = out_rows.shape[1]
    y = np.empty((T, d), np.float32)
    sh = None if shared is None else np.ascontiguousarray(shared, np.float32)
    lib().ora_combine(_p(out_rows), _p(np.ascontiguousarray(inv_perm, np.int32)), _p(topk_w),
                      _p(sh), T, d, k, _p(y))
    return y


def layer_tokens(weights: LayerWeights, x: np.ndarray, tokens, token_ids=None):
    """Whole layer for the chosen token indices: returns (idx, w, y)."""
    s = weights.struct()
    c = weights.cfg
    x = np.ascontiguousarray(x, dtype=np.uint16)
    tokens = np.ascontiguousarray(tokens, dtype=np.int32)
    n = tokens.shape[0]
    idx = np.empty((n, c.k), np.int32)
    w = np.empty((n, c.k), np.float32)
    y = np.empty((n, c.d), np.float32)
    tid = None if token_ids is None else np.ascontiguousarray(token_ids, np.int32)
    failed = lib().ora_layer_tokens(ctypes.byref(s), _p(x), _p(tid), _p(tokens), n, _p(idx), _p(w), _p(y))
    if failed:
        raise RuntimeError(f"{failed} tokens hit the hash-routing draw cap")
    return idx, w, y

"""Seeded synthetic inputs for the routed expert FFN layer.

Test and benchmark infrastructure. The oracle side and the CUDA side both take
their inputs from here; this module draws random numbers (Philox4x32-10, see
``synth.c``) and shapes them into the workloads' distributions. It holds none of
the layer's arithmetic: weights come out as fp32 normals and are quantised by
whoever consumes them.

Workload recipes (one per layer configuration):

* ``tiny``    T=4, d=256, F=512, E=8, k=2, softmax top-k, MXFP4, bf16 activations.
* ``decode``  T in {1,2,4,8}, d=4096, F=2048, E=256, k=8, MXFP4, bf16
              activations, plus one bf16 shared expert of d_ff 2048.
* ``prefill`` T=4096, same dims, router bias giving a Zipf(1.1) expert
              popularity, MXFP4 weights, MXFP8 activations.
* ``q2k``     T in {1,8}, same dims, Q2_K-style 2-bit experts, bf16 shared expert.
* ``hash``    T=16384, token ids uniform in [0, 129280), hash routing, MXFP4,
              MXFP8 activations.

Distributions: router and expert weights N(0, 0.02); activations N(0, 1) rounded
to bf16; shared-expert weights N(0, 0.02) rounded to bf16.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, replace

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_SO = os.path.join(_HERE, "libsynth.so")
_GPU_SRC = os.path.join(_HERE, "synth_gpu.cu")
_GPU_SO = os.path.join(_HERE, "libsynth_gpu.so")

# Tensor ids: each tensor of a workload draws from its own Philox key.
X, WR, W1, W3, W2, S1, S3, S2, TOK, ZIPF = range(1, 11)


def build(force: bool = False) -> str:
    """Compile libsynth.so next to its source (gcc, OpenMP)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                               "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _SO)
    if force or not os.path.exists(_GPU_SO) or os.path.getmtime(_GPU_SO) < os.path.getmtime(_GPU_SRC):
        tmp = _GPU_SO + f".tmp{os.getpid()}"
        subprocess.check_call(["nvcc", "-O3", "-gencode", "arch=compute_100a,code=sm_100a", "-Xcompiler",
                               "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-shared", _GPU_SRC, "-o", tmp])
        os.replace(tmp, _GPU_SO)
    return _SO


_lib_handle = None


def _lib():
    global _lib_handle
    if _lib_handle is None:
        build()
        L = ctypes.CDLL(_SO)
        u64, u32, i64, i32, f64, vp = (ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int64,
                                       ctypes.c_int32, ctypes.c_double, ctypes.c_void_p)
        L.synth_normal_f32.argtypes = [u64, u32, u32, u64, i64, f64, f64, vp]
        L.synth_normal_bf16.argtypes = [u64, u32, u32, u64, i64, f64, f64, vp]
        L.synth_uniform_f64.argtypes = [u64, u32, u32, u64, i64, vp]
        L.synth_uniform_int.argtypes = [u64, u32, u32, u64, i64, i64, i64, vp]
        L.synth_permutation.argtypes = [u64, u32, u32, i32, vp]
        L.synth_philox4x32_10.argtypes = [vp, u32, u32, vp]
        L.synth_num_threads.restype = ctypes.c_int
        for f in ("synth_normal_f32", "synth_normal_bf16", "synth_uniform_f64",
                  "synth_uniform_int", "synth_permutation", "synth_philox4x32_10"):
            getattr(L, f).restype = None
        _lib_handle = L
    return _lib_handle


_gpu_handle = None


def normal_f32_device(seed, tensor, sub, n, mean=0.0, std=1.0, first=0, out=None, stream=None):
    """Fill a float32 CUDA tensor with the same normal stream as normal_f32 (device copy of
    the generator; bench-sized tensors only)."""
    import torch
    global _gpu_handle
    if _gpu_handle is None:
        build()
        L = ctypes.CDLL(_GPU_SO)
        L.synth_gpu_normal_f32.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint64,
                                           ctypes.c_int64, ctypes.c_double, ctypes.c_double, ctypes.c_void_p,
                                           ctypes.c_void_p]
        L.synth_gpu_normal_f32.restype = ctypes.c_int
        _gpu_handle = L
    if out is None:
        out = torch.empty(n, dtype=torch.float32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream if stream is None else stream
    rc = _gpu_handle.synth_gpu_normal_f32(seed, tensor, sub, first, n, mean, std, out.data_ptr(), s)
    if rc != 0:
        raise RuntimeError(f"synth_gpu_normal_f32 failed: cuda error {rc}")
    return out


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def philox4x32_10(ctr, key) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(ctr, dtype=np.uint32))
    out = np.zeros(4, dtype=np.uint32)
    _lib().synth_philox4x32_10(_ptr(c), int(key[0]), int(key[1]), _ptr(out))
    return out


def normal_f32(seed, tensor, sub, n, mean=0.0, std=1.0, first=0, out=None) -> np.ndarray:
    if out is None:
        out = np.empty(n, dtype=np.float32)
    _lib().synth_normal_f32(seed, tensor, sub, first, n, mean, std, _ptr(out))
    return out


def normal_bf16(seed, tensor, sub, n, mean=0.0, std=1.0, first=0, out=None) -> np.ndarray:
    """bf16 bit patterns (uint16) of N(mean, std) draws rounded to nearest even."""
    if out is None:
        out = np.empty(n, dtype=np.uint16)
    _lib().synth_normal_bf16(seed, tensor, sub, first, n, mean, std, _ptr(out))
    return out


def uniform_f64(seed, tensor, sub, n, first=0) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    _lib().synth_uniform_f64(seed, tensor, sub, first, n, _ptr(out))
    return out


def uniform_int(seed, tensor, sub, n, lo, hi, first=0) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    _lib().synth_uniform_int(seed, tensor, sub, first, n, lo, hi, _ptr(out))
    return out


def permutation(seed, tensor, sub, n) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    _lib().synth_permutation(seed, tensor, sub, n, _ptr(out))
    return out


def num_threads() -> int:
    return int(_lib().synth_num_threads())


@dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int
    d: int = 4096
    F: int = 2048
    E: int = 256
    k: int = 8
    route: str = "softmax"      # "softmax" (top-k softmax) | "hash"
    act: str = "bf16"           # "bf16" (w4a16) | "mxfp8" (w4a8) | "mxfp4" (w4a4)
    wfmt: str = "mxfp4"         # "mxfp4" | "q2k"
    Fs: int = 0                 # shared-expert d_ff; 0 = no shared expert
    zipf_s: float = 0.0         # >0: router bias gives Zipf(zipf_s) expert popularity
    vocab: int = 129280         # token-id range for hash routing
    w_std: float = 0.02

    def with_T(self, T: int) -> "LayerConfig":
        return replace(self, T=T)

    @property
    def has_router(self) -> bool:
        return self.route == "softmax"


CONFIGS = {
    "tiny": LayerConfig("tiny", T=4, d=256, F=512, E=8, k=2),
    "decode": LayerConfig("decode", T=8, Fs=2048),
    "prefill": LayerConfig("prefill", T=4096, act="mxfp8", zipf_s=1.1),
    "q2k": LayerConfig("q2k", T=8, wfmt="q2k", Fs=2048),
    "hash": LayerConfig("hash", T=16384, route="hash", act="mxfp8"),
}
DECODE_TS = (1, 2, 4, 8)
Q2K_TS = (1, 8)


def make_x(cfg: LayerConfig, seed: int = 0, batch: int = 0) -> np.ndarray:
    """Activations x[T][d], bf16 bits, N(0, 1). ``batch`` selects an independent batch."""
    return normal_bf16(seed, X, batch, cfg.T * cfg.d).reshape(cfg.T, cfg.d)


def make_router(cfg: LayerConfig, seed: int = 0) -> np.ndarray:
    """Router weight W_r[E][d], bf16 bits, N(0, 0.02)."""
    return normal_bf16(seed, WR, 0, cfg.E * cfg.d, 0.0, cfg.w_std).reshape(cfg.E, cfg.d)


def make_bias(cfg: LayerConfig, seed: int = 0):
    """Router logit bias giving a Zipf(s) expert popularity, or None.

    bias_e = -sigma * s * ln(1 + pi(e)), sigma = w_std * sqrt(d) (the standard
    deviation of an unbiased logit), pi a seeded permutation of the experts, so
    the expert of rank r is favoured by -sigma * s * ln(r).
    """
    if cfg.zipf_s <= 0:
        return None
    pi = permutation(seed, ZIPF, 0, cfg.E).astype(np.float64)
    sigma = cfg.w_std * math.sqrt(cfg.d)
    return (-sigma * cfg.zipf_s * np.log1p(pi)).astype(np.float32)


def make_token_ids(cfg: LayerConfig, seed: int = 0, batch: int = 0) -> np.ndarray:
    return uniform_int(seed, TOK, batch, cfg.T, 0, cfg.vocab)


def expert_weight_f32(cfg: LayerConfig, seed: int, e: int, which: int, out=None) -> np.ndarray:
    """fp32 N(0, w_std) weights of routed expert e: which = W1, W3 ([F][d]) or W2 ([d][F])."""
    assert which in (W1, W3, W2)
    rows, K = (cfg.F, cfg.d) if which != W2 else (cfg.d, cfg.F)
    a = normal_f32(seed, which, e, rows * K, 0.0, cfg.w_std, out=out)
    return a.reshape(rows, K)


def shared_weights_bf16(cfg: LayerConfig, seed: int = 0):
    """bf16 shared expert (W1s [Fs][d], W3s [Fs][d], W2s [d][Fs]) or None."""
    if cfg.Fs <= 0:
        return None
    s1 = normal_bf16(seed, S1, 0, cfg.Fs * cfg.d, 0.0, cfg.w_std).reshape(cfg.Fs, cfg.d)
    s3 = normal_bf16(seed, S3, 0, cfg.Fs * cfg.d, 0.0, cfg.w_std).reshape(cfg.Fs, cfg.d)
    s2 = normal_bf16(seed, S2, 0, cfg.d * cfg.Fs, 0.0, cfg.w_std).reshape(cfg.d, cfg.Fs)
    return s1, s3, s2

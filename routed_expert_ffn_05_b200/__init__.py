"""Python binding of libmoe.so, the routed MoE FFN layer for B200 (sm_100a).

Argument marshalling only: every function here has the name of a C entry
point in ``include/moe.h`` and forwards device pointers (torch CUDA tensors or
raw integers), sizes and the current CUDA stream. All computation runs in the
library's CUDA kernels; there is no fallback. The library must have been built
(``python -m routed_expert_ffn_05_b200.build``); importing fails loudly when it
is missing.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe.so")

# moe_status
MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA, MOE_ERR_DEVICE, MOE_ERR_TIMEOUT = range(6)
# formats and modes
MOE_W_MXFP4, MOE_W_Q2K = 1, 2
MOE_A_BF16, MOE_A_MXFP8, MOE_A_MXFP4 = 0, 1, 2
MOE_ROUTE_SOFTMAX_TOPK, MOE_ROUTE_HASH = 0, 1
MOE_MAT_W1, MOE_MAT_W2, MOE_MAT_W3 = 1, 2, 3
MOE_DEVERR_NONE, MOE_DEVERR_EXPERT_RANGE, MOE_DEVERR_HASH_CAP, MOE_DEVERR_TIMEOUT, MOE_DEVERR_PERM = range(5)


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class moe_dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("T", "d_model", "d_ff", "E", "k", "route", "act", "wfmt", "d_ff_shared")]


class moe_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("w1", "w3", "w2", "sw1", "sw3", "sw2", "w_router", "router_bias")]


class moe_cache_stats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_uint64) for n in ("calls", "waves", "hits", "misses", "bytes_h2d")]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python routed_expert_ffn_05_b200/build.py`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    D, W = ctypes.POINTER(moe_dims), ctypes.POINTER(moe_weights)
    sigs = {
        "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "moe_workspace_size": (ctypes.c_int, [D, ctypes.POINTER(sz)]),
        "moe_quantize_weights": (ctypes.c_int, [D, i32, vp, vp, vp]),
        "moe_packed_size": (ctypes.c_int, [D, i32, ctypes.POINTER(sz)]),
        "moe_pack_weights": (ctypes.c_int, [D, i32, vp, vp, vp]),
        "moe_route": (ctypes.c_int, [D, vp, W, vp, vp, vp, vp, vp]),
        "moe_permute": (ctypes.c_int, [D, vp, vp, vp, vp, vp, vp, vp]),
        "moe_expert_ffn": (ctypes.c_int, [D, W, vp, vp, vp, vp, vp, vp]),
        "moe_shared_ffn": (ctypes.c_int, [D, W, vp, vp, vp, vp]),
        "moe_combine": (ctypes.c_int, [D, vp, vp, vp, vp, vp, vp]),
        "moe_layer": (ctypes.c_int, [D, W, vp, vp, vp, vp, vp]),
        "moe_get_device_error": (ctypes.c_int, [vp, ctypes.POINTER(i32)]),
        "moe_debug_dequant": (ctypes.c_int, [D, i32, vp, i32, vp, vp]),
        "moe_debug_quant_act": (ctypes.c_int, [vp, i32, i32, vp, vp, vp]),
        "moe_layer_static_ws": (ctypes.c_int, [D, W, vp, vp, vp, vp]),
        "moe_ep_range": (ctypes.c_int, [i32, i32, i32, ctypes.POINTER(i32), ctypes.POINTER(i32)]),
        "moe_layer_ep": (ctypes.c_int, [D, W, i32, i32, i32, vp, vp, vp, vp, vp]),
        "moe_cache_create": (ctypes.c_int, [D, i32, vp, vp, vp, vp, vp, vp, ctypes.POINTER(vp)]),
        "moe_cache_destroy": (ctypes.c_int, [vp]),
        "moe_cache_get_stats": (ctypes.c_int, [vp, ctypes.POINTER(moe_cache_stats)]),
        "moe_layer_cached": (ctypes.c_int, [vp, D, W, vp, vp, vp, vp, vp]),
        "moe_debug_hash_route": (ctypes.c_int, [D, vp, i32, vp, vp, vp]),
        "moe_debug_tc_gather": (ctypes.c_int, [D, vp, vp, vp, vp, vp, vp, vp, vp]),
        "moe_debug_set_wait": (ctypes.c_int, [ctypes.c_uint64, ctypes.c_uint32]),
        "moe_debug_router_approx": (ctypes.c_int, [D, vp, W, vp, vp, vp]),
        "moe_debug_launch_count": (ctypes.c_uint64, []),
        "moe_debug_set_ffn_events": (ctypes.c_int, [vp, vp]),
    }
    for name, (res, args) in sigs.items():
        f = getattr(L, name)
        f.restype, f.argtypes = res, args
    return L


lib = _load()


def _p(x):
    """Device pointer of a torch tensor, an int address, or None (NULL)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _check(st: int, where: str):
    if st != MOE_OK:
        raise MoeError(st, where)


def status_string(st: int) -> str:
    return lib.moe_status_string(st).decode()


moe_status_string = status_string


def make_dims(T, d_model, d_ff, E, k, route=MOE_ROUTE_SOFTMAX_TOPK, act=MOE_A_BF16, wfmt=MOE_W_MXFP4,
              d_ff_shared=0) -> moe_dims:
    return moe_dims(T, d_model, d_ff, E, k, route, act, wfmt, d_ff_shared)


def make_weights(w1, w3, w2, sw1=None, sw3=None, sw2=None, w_router=None, router_bias=None) -> moe_weights:
    args = (w1, w3, w2, sw1, sw3, sw2, w_router, router_bias)
    w = moe_weights(*(_p(a) for a in args))
    w._keep = args  # the struct holds raw pointers: keep the tensors alive with it
    return w


def moe_workspace_size(dims: moe_dims) -> int:
    n = ctypes.c_size_t()
    _check(lib.moe_workspace_size(ctypes.byref(dims), ctypes.byref(n)), "moe_workspace_size")
    return n.value


def moe_packed_size(dims: moe_dims, which: int) -> int:
    n = ctypes.c_size_t()
    _check(lib.moe_packed_size(ctypes.byref(dims), which, ctypes.byref(n)), "moe_packed_size")
    return n.value


def moe_quantize_weights(dims, which, w, canonical, stream=None):
    _check(lib.moe_quantize_weights(ctypes.byref(dims), which, _p(w), _p(canonical), _stream(stream)),
           "moe_quantize_weights")


def moe_pack_weights(dims, which, canonical, packed, stream=None):
    _check(lib.moe_pack_weights(ctypes.byref(dims), which, _p(canonical), _p(packed), _stream(stream)),
           "moe_pack_weights")


def moe_route(dims, x, weights, token_ids, topk_idx, topk_w, ws, stream=None):
    _check(lib.moe_route(ctypes.byref(dims), _p(x), ctypes.byref(weights), _p(token_ids), _p(topk_idx),
                         _p(topk_w), _p(ws), _stream(stream)), "moe_route")


def moe_permute(dims, topk_idx, counts, offsets, perm, inv_perm, ws, stream=None):
    _check(lib.moe_permute(ctypes.byref(dims), _p(topk_idx), _p(counts), _p(offsets), _p(perm), _p(inv_perm),
                           _p(ws), _stream(stream)), "moe_permute")


def moe_expert_ffn(dims, weights, x, offsets, perm, out_rows, ws, stream=None):
    _check(lib.moe_expert_ffn(ctypes.byref(dims), ctypes.byref(weights), _p(x), _p(offsets), _p(perm),
                              _p(out_rows), _p(ws), _stream(stream)), "moe_expert_ffn")


def moe_shared_ffn(dims, weights, x, shared_out, ws, stream=None):
    _check(lib.moe_shared_ffn(ctypes.byref(dims), ctypes.byref(weights), _p(x), _p(shared_out), _p(ws),
                              _stream(stream)), "moe_shared_ffn")


def moe_combine(dims, out_rows, inv_perm, topk_w, shared_out, y, stream=None):
    _check(lib.moe_combine(ctypes.byref(dims), _p(out_rows), _p(inv_perm), _p(topk_w), _p(shared_out), _p(y),
                           _stream(stream)), "moe_combine")


def moe_layer(dims, weights, x, token_ids, y, ws, stream=None):
    _check(lib.moe_layer(ctypes.byref(dims), ctypes.byref(weights), _p(x), _p(token_ids), _p(y), _p(ws),
                         _stream(stream)), "moe_layer")


def moe_ep_range(E, rank, world):
    """(begin, end): the contiguous routed experts rank `rank` of `world` owns."""
    b, e = ctypes.c_int32(), ctypes.c_int32()
    _check(lib.moe_ep_range(E, rank, world, ctypes.byref(b), ctypes.byref(e)), "moe_ep_range")
    return b.value, e.value


def moe_layer_ep(dims, weights, expert_begin, expert_end, add_shared, x, token_ids, y, ws, stream=None):
    _check(lib.moe_layer_ep(ctypes.byref(dims), ctypes.byref(weights), expert_begin, expert_end, int(add_shared),
                            _p(x), _p(token_ids), _p(y), _p(ws), _stream(stream)), "moe_layer_ep")


def moe_layer_ep_allreduce(dims, weights, rank, world, x, token_ids, y, ws, group=None, stream=None):
    """One rank of the expert-parallel layer: this rank's part (its experts,
    plus the shared expert on rank 0) into y, then the sum over ranks in place
    (torch.distributed all-reduce; NCCL on GPUs). Every rank ends with the
    whole layer's y. ``weights`` holds this rank's experts (moe_ep_range)."""
    import torch.distributed as dist
    b, e = moe_ep_range(dims.E, rank, world)
    moe_layer_ep(dims, weights, b, e, rank == 0, x, token_ids, y, ws, stream)
    dist.all_reduce(y, op=dist.ReduceOp.SUM, group=group)
    return y


class ExpertCache:
    """moe_cache_create / moe_layer_cached / moe_cache_destroy: ``slots`` routed
    experts in HBM (dev_w1/3/2), all of them in pinned host memory (host_w1/3/2,
    packed layout). Keeps the buffers it was given alive."""

    def __init__(self, dims, slots, host_w1, host_w3, host_w2, dev_w1, dev_w3, dev_w2):
        self.handle = None
        self._keep = (host_w1, host_w3, host_w2, dev_w1, dev_w3, dev_w2)
        self.dims = dims
        h = ctypes.c_void_p()
        _check(lib.moe_cache_create(ctypes.byref(dims), slots, _p(host_w1), _p(host_w3), _p(host_w2), _p(dev_w1),
                                    _p(dev_w3), _p(dev_w2), ctypes.byref(h)), "moe_cache_create")
        self.handle = h.value

    def layer(self, dims, weights, x, token_ids, y, ws, stream=None):
        _check(lib.moe_layer_cached(self.handle, ctypes.byref(dims), ctypes.byref(weights), _p(x), _p(token_ids),
                                    _p(y), _p(ws), _stream(stream)), "moe_layer_cached")

    def stats(self) -> dict:
        st = moe_cache_stats()
        _check(lib.moe_cache_get_stats(self.handle, ctypes.byref(st)), "moe_cache_get_stats")
        return {n: getattr(st, n) for n, _ in st._fields_}

    def close(self):
        if self.handle:
            lib.moe_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        self.close()


def moe_cache_create(dims, slots, host_w1, host_w3, host_w2, dev_w1, dev_w3, dev_w2) -> ExpertCache:
    return ExpertCache(dims, slots, host_w1, host_w3, host_w2, dev_w1, dev_w3, dev_w2)


def moe_cache_destroy(cache: ExpertCache):
    cache.close()


def moe_cache_get_stats(cache: ExpertCache) -> dict:
    return cache.stats()


def moe_layer_cached(cache: ExpertCache, dims, weights, x, token_ids, y, ws, stream=None):
    cache.layer(dims, weights, x, token_ids, y, ws, stream)


MOE_STATIC_WS_BYTES = 32 << 20


def moe_layer_static_ws(dims, weights, x, token_ids, y, stream=None):
    """moe_layer for callers that cannot allocate device memory: scratch comes from an
    array built into the library (MOE_STATIC_WS_BYTES per GPU); see include/moe.h."""
    _check(lib.moe_layer_static_ws(ctypes.byref(dims), ctypes.byref(weights), _p(x), _p(token_ids), _p(y),
                                   _stream(stream)), "moe_layer_static_ws")


def moe_get_device_error(stream=None) -> int:
    code = ctypes.c_int32()
    st = lib.moe_get_device_error(_stream(stream), ctypes.byref(code))
    if st not in (MOE_OK, MOE_ERR_DEVICE):
        raise MoeError(st, "moe_get_device_error")
    return code.value


def moe_debug_dequant(dims, which, packed, expert, out, stream=None):
    _check(lib.moe_debug_dequant(ctypes.byref(dims), which, _p(packed), expert, _p(out), _stream(stream)),
           "moe_debug_dequant")


def moe_debug_quant_act(x, rows, K, codes, scales, stream=None):
    _check(lib.moe_debug_quant_act(_p(x), rows, K, _p(codes), _p(scales), _stream(stream)),
           "moe_debug_quant_act")


def moe_debug_hash_route(dims, token_ids, max_draws, topk_idx, topk_w, stream=None):
    _check(lib.moe_debug_hash_route(ctypes.byref(dims), _p(token_ids), max_draws, _p(topk_idx), _p(topk_w),
                                    _stream(stream)), "moe_debug_hash_route")


def moe_debug_tc_gather(dims, x, offsets, perm, codes, atoms, ustart, ws, stream=None):
    _check(lib.moe_debug_tc_gather(ctypes.byref(dims), _p(x), _p(offsets), _p(perm), _p(codes), _p(atoms),
                                   _p(ustart), _p(ws), _stream(stream)), "moe_debug_tc_gather")


def moe_debug_router_approx(dims, x, weights, approx, wnorm, stream=None):
    _check(lib.moe_debug_router_approx(ctypes.byref(dims), _p(x), ctypes.byref(weights), _p(approx), _p(wnorm),
                                       _stream(stream)), "moe_debug_router_approx")


def moe_debug_set_wait(limit_ns=0, extra_tiles=0):
    _check(lib.moe_debug_set_wait(limit_ns, extra_tiles), "moe_debug_set_wait")


def moe_debug_launch_count() -> int:
    return int(lib.moe_debug_launch_count())


def moe_debug_set_ffn_events(before=None, after=None):
    """``before``/``after``: torch.cuda.Event (or raw cudaEvent_t ints), or None to turn off."""
    h = lambda ev: None if ev is None else (ev if isinstance(ev, int) else ev.cuda_event)
    _check(lib.moe_debug_set_ffn_events(h(before), h(after)), "moe_debug_set_ffn_events")

"""Thin Python binding of libftmoe.so (include/ftmoe.h): argument marshalling only.

Every function has the name of its C entry point and the same arguments; tensors may
be passed as torch tensors (their data_ptr() is used), plain integer addresses, or
None (NULL).  `stream=None` means torch's current CUDA stream.  A non-OK status raises
FtError carrying the status code and ft_last_error().  No arithmetic of the layer
happens here: every step runs in the library's CUDA kernels.  If the library has not
been built, the first call raises: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
import re

PKG = os.path.dirname(os.path.abspath(__file__))
# FTMOE_LIB selects another build of the same library (e.g. libftmoe_debug.so, the
# debug-bounds build); default: the in-tree libftmoe.so
LIB_PATH = os.environ.get("FTMOE_LIB") or os.path.join(PKG, "libftmoe.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "ftmoe.h")

FT_OK, FT_ERR_INVALID_ARG, FT_ERR_UNSUPPORTED, FT_ERR_CUDA, FT_ERR_WORKSPACE, FT_ERR_NOT_PINNED, \
    FT_ERR_TIMEOUT, FT_ERR_DEVICE_CHECK = range(8)
FT_W_BF16, FT_W_MXFP4 = 0, 1
FT_CACHE_PER_LAYER, FT_CACHE_GLOBAL = 0, 1

c_i32, c_i64, c_u64, c_sz, c_vp, c_f32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t, \
    ctypes.c_void_p, ctypes.c_float


class ft_moe_shape(ctypes.Structure):
    _fields_ = [("hidden", c_i32), ("ffn", c_i32), ("num_experts", c_i32), ("top_k", c_i32),
                ("num_shared", c_i32), ("wdtype", c_i32)]


class ft_moe_weights(ctypes.Structure):
    _fields_ = [("w13", c_vp), ("w13_scale", c_vp), ("w2", c_vp), ("w2_scale", c_vp), ("expert_ptrs", c_vp),
                ("shared_w13", c_vp), ("shared_w13_scale", c_vp), ("shared_w2", c_vp), ("shared_w2_scale", c_vp)]


class ft_stream_cfg(ctypes.Structure):
    _fields_ = [("num_layers", c_i32), ("slots_per_layer", c_i32), ("shape", ft_moe_shape),
                ("host_layers", ctypes.POINTER(ft_moe_weights)), ("hbm_arena", c_vp), ("hbm_arena_bytes", c_sz),
                ("host_wait_timeout_ms", c_i64), ("cache_policy", c_i32)]


class FtError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"ftmoe status {status}: {msg}")
        self.status = status


_lib = None

_SIGS = {
    "ft_last_error": (ctypes.c_char_p, []),
    "ft_version": (ctypes.c_char_p, []),
    "ft_set_decode_max_tokens": (c_i32, [c_i32]),
    "ft_get_decode_max_tokens": (c_i32, []),
    "ft_set_pipeline_wait_limit_ns": (c_u64, [c_u64]),
    "ft_set_block_scaled_decode": (c_i32, [c_i32]),
    "ft_moe_decode_kernels": (c_i32, [ctypes.POINTER(ft_moe_shape), c_i32]),
    "ft_hbm_read_probe": (c_i32, [c_vp, c_sz, c_vp, c_i32, c_vp]),
    "ft_tma_read_probe": (c_i32, [c_i32, c_vp, c_sz, c_sz, c_vp, c_vp]),
    "ft_moe_workspace_bytes": (c_sz, [ctypes.POINTER(ft_moe_shape), c_i32]),
    "ft_moe_workspace_init": (c_i32, [c_vp, c_sz, c_vp]),
    "ft_moe_check": (c_i32, [c_vp, c_vp]),
    "ft_moe_route": (c_i32, [ctypes.POINTER(ft_moe_shape), c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "ft_moe_permute": (c_i32, [ctypes.POINTER(ft_moe_shape), c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "ft_moe_permute_noalloc": (c_i32, [ctypes.POINTER(ft_moe_shape), c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp]),
    "ft_moe_experts": (c_i32, [ctypes.POINTER(ft_moe_shape), c_i32, ctypes.POINTER(ft_moe_weights), c_vp, c_vp, c_vp,
                               c_vp, c_vp, c_vp, c_sz, c_vp]),
    "ft_moe_experts_gateup": (c_i32, [ctypes.POINTER(ft_moe_shape), c_i32, ctypes.POINTER(ft_moe_weights), c_vp, c_vp,
                                      c_vp, c_vp, c_sz, c_vp]),
    "ft_moe_experts_down": (c_i32, [ctypes.POINTER(ft_moe_shape), c_i32, ctypes.POINTER(ft_moe_weights), c_vp, c_vp,
                                    c_vp, c_vp, c_sz, c_vp]),
    "ft_moe_combine": (c_i32, [ctypes.POINTER(ft_moe_shape), c_i32, c_vp, c_vp, c_vp, c_vp, c_vp]),
    "ft_moe_layer_forward": (c_i32, [ctypes.POINTER(ft_moe_shape), c_i32, c_vp, c_vp, c_vp, ctypes.POINTER(ft_moe_weights),
                                     c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "ft_moe_unit_rms": (c_i32, [c_i32, c_i32, c_vp, c_vp, c_f32, c_vp]),
    "ft_expert_stream_arena_bytes": (c_sz, [ctypes.POINTER(ft_stream_cfg)]),
    "ft_expert_stream_create": (c_i32, [ctypes.POINTER(ft_stream_cfg), ctypes.POINTER(c_vp)]),
    "ft_expert_stream_prefill": (c_i32, [c_vp, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp, c_vp]),
    "ft_expert_stream_prefill_routed": (c_i32, [c_vp, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp, c_vp]),
    "ft_expert_stream_decode_step": (c_i32, [c_vp, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp, c_vp]),
    "ft_expert_stream_stats": (c_i32, [c_vp, c_i32, ctypes.POINTER(c_u64)]),
    "ft_expert_stream_slots": (c_i32, [c_vp, c_i32, ctypes.POINTER(c_i32)]),
    "ft_expert_stream_reset_cache": (c_i32, [c_vp]),
    "ft_expert_stream_set_slots": (c_i32, [c_vp, c_i32, c_vp, c_vp]),
    "ft_expert_stream_destroy": (None, [c_vp]),
    "ft_expert_stream_inject_copy_failure": (c_i32, [c_vp, c_i64]),
    "ft_lru_step": (c_i32, [c_i32, c_i32, c_vp, c_vp, c_vp, c_i64, c_vp, c_i32, c_vp, c_vp]),
    "ft_lru_resize": (c_i32, [c_i32, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp]),
}


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with `python -m expert_offload_serving_router_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of every function declared in include/ftmoe.h."""
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(ft_[a-z0-9_]+)\s*\(", txt)))


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if hasattr(t, "data_ptr"):
        return t.data_ptr()
    if isinstance(t, ctypes.Array):
        return ctypes.addressof(t)
    raise TypeError(f"cannot pass {type(t)} as a pointer")


def _s(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(st: int):
    if st != FT_OK:
        raise FtError(st, lib().ft_last_error().decode())


def _nbytes(ws, ws_bytes):
    if ws_bytes is not None:
        return ws_bytes
    return ws.numel() * ws.element_size()


# ---------------------------------------------------------------- structures
def make_shape(hidden, ffn, num_experts, top_k, num_shared=0, wdtype=FT_W_BF16) -> ft_moe_shape:
    return ft_moe_shape(hidden, ffn, num_experts, top_k, num_shared, wdtype)


def make_weights(w13=None, w13_scale=None, w2=None, w2_scale=None, expert_ptrs=None, shared_w13=None,
                 shared_w13_scale=None, shared_w2=None, shared_w2_scale=None) -> ft_moe_weights:
    return ft_moe_weights(_p(w13), _p(w13_scale), _p(w2), _p(w2_scale), _p(expert_ptrs), _p(shared_w13),
                          _p(shared_w13_scale), _p(shared_w2), _p(shared_w2_scale))


# ---------------------------------------------------------------- entry points
def ft_last_error() -> str:
    return lib().ft_last_error().decode()


def ft_version() -> str:
    return lib().ft_version().decode()


def ft_set_decode_max_tokens(t: int) -> int:
    return lib().ft_set_decode_max_tokens(t)


def ft_get_decode_max_tokens() -> int:
    return lib().ft_get_decode_max_tokens()


def ft_set_pipeline_wait_limit_ns(ns: int) -> int:
    return lib().ft_set_pipeline_wait_limit_ns(ns)


def ft_set_block_scaled_decode(mode: int) -> int:
    return lib().ft_set_block_scaled_decode(mode)


def ft_moe_decode_kernels(shape: ft_moe_shape, T: int) -> int:
    return lib().ft_moe_decode_kernels(ctypes.byref(shape), T)


def ft_hbm_read_probe(buf, nbytes: int, sink, ctas_per_sm: int, stream=None) -> None:
    _check(lib().ft_hbm_read_probe(_p(buf), nbytes, _p(sink), ctas_per_sm, _s(stream)))


def ft_tma_read_probe(mode: int, buf, nbytes: int, region_bytes: int, status, stream=None) -> None:
    _check(lib().ft_tma_read_probe(mode, _p(buf), nbytes, region_bytes, _p(status), _s(stream)))


def ft_moe_workspace_bytes(shape: ft_moe_shape, max_tokens: int) -> int:
    return lib().ft_moe_workspace_bytes(ctypes.byref(shape), max_tokens)


def ft_moe_workspace_init(ws, ws_bytes=None, stream=None):
    _check(lib().ft_moe_workspace_init(_p(ws), _nbytes(ws, ws_bytes), _s(stream)))


def ft_moe_check(ws, stream=None):
    _check(lib().ft_moe_check(_p(ws), _s(stream)))


def ft_moe_route(shape, T, x, w_router, bias, topk_idx, topk_w, logits, ws, ws_bytes=None, stream=None):
    _check(lib().ft_moe_route(ctypes.byref(shape), T, _p(x), _p(w_router), _p(bias), _p(topk_idx), _p(topk_w),
                              _p(logits), _p(ws), _nbytes(ws, ws_bytes), _s(stream)))


def ft_moe_permute(shape, T, topk_idx, x, offsets, sorted_flat, inv_pos, x_sorted, ws, ws_bytes=None, stream=None):
    _check(lib().ft_moe_permute(ctypes.byref(shape), T, _p(topk_idx), _p(x), _p(offsets), _p(sorted_flat),
                                _p(inv_pos), _p(x_sorted), _p(ws), _nbytes(ws, ws_bytes), _s(stream)))


def ft_moe_permute_noalloc(shape, T, topk_idx, x, offsets, sorted_flat, inv_pos, x_sorted, stream=None):
    """Permutation without a workspace (static device scratch); for callers that cannot allocate."""
    _check(lib().ft_moe_permute_noalloc(ctypes.byref(shape), T, _p(topk_idx), _p(x), _p(offsets), _p(sorted_flat),
                                        _p(inv_pos), _p(x_sorted), _s(stream)))


def ft_moe_experts(shape, T, weights, x, x_sorted, offsets, sorted_flat, o_sorted, ws, ws_bytes=None, stream=None):
    _check(lib().ft_moe_experts(ctypes.byref(shape), T, ctypes.byref(weights), _p(x), _p(x_sorted), _p(offsets),
                                _p(sorted_flat), _p(o_sorted), _p(ws), _nbytes(ws, ws_bytes), _s(stream)))


def ft_moe_experts_gateup(shape, T, weights, x_sorted, offsets, h, ws, ws_bytes=None, stream=None):
    _check(lib().ft_moe_experts_gateup(ctypes.byref(shape), T, ctypes.byref(weights), _p(x_sorted), _p(offsets), _p(h),
                                       _p(ws), _nbytes(ws, ws_bytes), _s(stream)))


def ft_moe_experts_down(shape, T, weights, h, offsets, o_sorted, ws, ws_bytes=None, stream=None):
    _check(lib().ft_moe_experts_down(ctypes.byref(shape), T, ctypes.byref(weights), _p(h), _p(offsets), _p(o_sorted),
                                     _p(ws), _nbytes(ws, ws_bytes), _s(stream)))


def ft_moe_combine(shape, T, o_sorted, inv_pos, topk_w, y, stream=None):
    _check(lib().ft_moe_combine(ctypes.byref(shape), T, _p(o_sorted), _p(inv_pos), _p(topk_w), _p(y), _s(stream)))


def ft_moe_layer_forward(shape, T, x, w_router, bias, weights, y, topk_idx_out, logits_out, ws, ws_bytes=None,
                         stream=None):
    _check(lib().ft_moe_layer_forward(ctypes.byref(shape), T, _p(x), _p(w_router), _p(bias), ctypes.byref(weights),
                                      _p(y), _p(topk_idx_out), _p(logits_out), _p(ws), _nbytes(ws, ws_bytes),
                                      _s(stream)))


def ft_moe_unit_rms(T, H, x_in, x_out, eps=1e-6, stream=None):
    _check(lib().ft_moe_unit_rms(T, H, _p(x_in), _p(x_out), eps, _s(stream)))


def ft_lru_step(E, n_slots, content, stamp, where, step, ids, out_slot, out_hit):
    """Host-only LRU policy step on numpy arrays (int32 content/where/ids/out_slot, int64 stamp, uint8 out_hit)."""
    P = lambda a: a.ctypes.data_as(c_vp) if a is not None else None
    _check(lib().ft_lru_step(E, n_slots, P(content), P(stamp), P(where), step, P(ids), len(ids), P(out_slot), P(out_hit)))


def ft_lru_resize(E, n_old, n_new, content, stamp, where):
    """Host-only resize of one LRU state (numpy int32 content/where, int64 stamp, each with room
    for max(n_old, n_new) slots).  Returns the list of (from, to) slot moves."""
    P = lambda a: a.ctypes.data_as(c_vp)
    mf = (c_i32 * max(1, n_old))()
    mt = (c_i32 * max(1, n_old))()
    nm = c_i32()
    _check(lib().ft_lru_resize(E, n_old, n_new, P(content), P(stamp), P(where), mf, mt, ctypes.byref(nm)))
    return [(mf[i], mt[i]) for i in range(nm.value)]


# ---------------------------------------------------------------- expert stream
def ft_expert_stream_arena_bytes(cfg: ft_stream_cfg) -> int:
    return lib().ft_expert_stream_arena_bytes(ctypes.byref(cfg))


def ft_expert_stream_create(cfg: ft_stream_cfg) -> int:
    h = c_vp()
    _check(lib().ft_expert_stream_create(ctypes.byref(cfg), ctypes.byref(h)))
    return h.value


def _ptr_array(items):
    arr = (c_vp * len(items))(*[_p(t) for t in items])
    return arr


def ft_expert_stream_prefill(handle, T, x, w_router, bias, y_layers, x_layers, ws, ws_bytes=None, compute_stream=None,
                             copy_stream=None):
    wr = _ptr_array(w_router)
    bs = _ptr_array(bias) if bias is not None else None
    _check(lib().ft_expert_stream_prefill(handle, T, _p(x), ctypes.addressof(wr), ctypes.addressof(bs) if bs else None,
                                          _p(y_layers), _p(x_layers), _p(ws), _nbytes(ws, ws_bytes),
                                          _s(compute_stream), _s(copy_stream)))


def ft_expert_stream_prefill_routed(handle, T, x, w_router, bias, y_layers, x_layers, ws, ws_bytes=None,
                                    compute_stream=None, copy_stream=None):
    wr = _ptr_array(w_router)
    bs = _ptr_array(bias) if bias is not None else None
    _check(lib().ft_expert_stream_prefill_routed(handle, T, _p(x), ctypes.addressof(wr),
                                                 ctypes.addressof(bs) if bs else None, _p(y_layers), _p(x_layers),
                                                 _p(ws), _nbytes(ws, ws_bytes), _s(compute_stream), _s(copy_stream)))


def ft_expert_stream_decode_step(handle, T, x, w_router, bias, y_layers, x_layers, ws, ws_bytes=None,
                                 compute_stream=None, copy_stream=None):
    wr = _ptr_array(w_router)
    bs = _ptr_array(bias) if bias is not None else None
    _check(lib().ft_expert_stream_decode_step(handle, T, _p(x), ctypes.addressof(wr),
                                              ctypes.addressof(bs) if bs else None, _p(y_layers), _p(x_layers), _p(ws),
                                              _nbytes(ws, ws_bytes), _s(compute_stream), _s(copy_stream)))


def ft_expert_stream_stats(handle, layer: int = -1) -> list[int]:
    out = (c_u64 * 6)()
    _check(lib().ft_expert_stream_stats(handle, layer, out))
    return list(out)


def ft_expert_stream_slots(handle, layer: int, n_slots: int) -> list[int]:
    out = (c_i32 * n_slots)()
    _check(lib().ft_expert_stream_slots(handle, layer, out))
    return list(out)


def ft_expert_stream_reset_cache(handle):
    _check(lib().ft_expert_stream_reset_cache(handle))


def ft_expert_stream_set_slots(handle, slots_per_layer: int, compute_stream=None, copy_stream=None):
    _check(lib().ft_expert_stream_set_slots(handle, slots_per_layer, _s(compute_stream), _s(copy_stream)))


def ft_expert_stream_destroy(handle):
    lib().ft_expert_stream_destroy(handle)


def ft_expert_stream_inject_copy_failure(handle, n: int):
    _check(lib().ft_expert_stream_inject_copy_failure(handle, n))

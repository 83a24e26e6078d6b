"""fp64 CPU oracle for the sparse-MoE FFN layer and the decode LRU expert cache.

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
CPU-baseline leg of bench.py, never by the product library.  The arithmetic
lives in moe_oracle.c (plain loops, fp64); this module only builds it with
gcc and marshals numpy arrays.  Every function cites, in moe_oracle.c, the
passage of the source pages (or the OCP MX v1.0 spec) it follows.

Parity pins: every function here is pinned by tests/test_oracle_pins.py
against something other than itself (spec tables, brute force, numpy float64
matmul, closed forms and invariants); none is "parity unpinned" except the
pages' claim that the CPU/GPU merge is exact, which prints no number.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile moe_oracle.c -> liboracle.so (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i32, i64, dbl = ctypes.c_int, ctypes.c_long, ctypes.c_double
        L.oracle_bf16_to_f64.restype = dbl
        L.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        L.oracle_e2m1_to_f64.restype = dbl
        L.oracle_e2m1_to_f64.argtypes = [ctypes.c_uint8]
        L.oracle_e8m0_to_f64.restype = dbl
        L.oracle_e8m0_to_f64.argtypes = [ctypes.c_uint8]
        L.oracle_decode_matrix.argtypes = [i32, P, P, i64, i64, P]
        L.oracle_e4m3_to_f64.restype = dbl
        L.oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        L.oracle_decode_nvfp4.argtypes = [P, P, ctypes.c_float, i64, i64, P]
        L.oracle_router_logits.argtypes = [i32, i32, i32, P, P, P, P, P]
        L.oracle_topk.argtypes = [i32, i32, i32, P, P, P]
        L.oracle_permute.argtypes = [i32, i32, i32, i32, P, P, P, P]
        L.oracle_expert_ffn.argtypes = [i32, i32, i32, P, P, P, P, P, P]
        L.oracle_moe_layer.restype = i32
        L.oracle_moe_layer.argtypes = [i32] * 7 + [P, i32, P, P, P] + [P] * 8 + [P, i32]
        L.oracle_unit_rms.argtypes = [i32, i32, P, dbl, P]
        L.oracle_lru_sim.restype = i32
        L.oracle_lru_sim.argtypes = [i32, i32, i32, P, P, P, P, P, P, P]
        L.oracle_e4m3_round.restype = dbl
        L.oracle_e4m3_round.argtypes = [dbl]
        L.oracle_mxfp8_qdq.argtypes = [i64, P, P]
        L.oracle_expert_ffn_mxfp8_act.argtypes = [i32, i32, i32, P, P, P, P, P, P]
        L.oracle_mxfp8x2_qdq.argtypes = [i64, P, P]
        L.oracle_expert_ffn_mxfp8_planes.argtypes = [i32, i32, i32, i32, P, P, P, P, P, P]
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- decodes
def bf16_to_f64(bits) -> float:
    return lib().oracle_bf16_to_f64(int(bits))


def e2m1_to_f64(code) -> float:
    return lib().oracle_e2m1_to_f64(int(code))


def e8m0_to_f64(b) -> float:
    return lib().oracle_e8m0_to_f64(int(b))


def e4m3_to_f64(b) -> float:
    return lib().oracle_e4m3_to_f64(int(b))


def decode_nvfp4(codes, scales, tensor_scale: float, rows: int, cols: int) -> np.ndarray:
    """NVFP4 [rows, cols] to fp64: E2M1 codes (two per byte), E4M3 scale per 16, fp32 tensor scale."""
    codes, scales = _c(codes, np.uint8), _c(scales, np.uint8)
    out = np.empty((rows, cols), dtype=np.float64)
    lib().oracle_decode_nvfp4(_p(codes), _p(scales), float(tensor_scale), rows, cols, _p(out))
    return out


def decode_matrix(wdtype: int, w, scale, rows: int, cols: int) -> np.ndarray:
    w = np.ascontiguousarray(w)
    scale = _c(scale, np.uint8)
    out = np.empty((rows, cols), dtype=np.float64)
    lib().oracle_decode_matrix(wdtype, _p(w), _p(scale), rows, cols, _p(out))
    return out


# ---------------------------------------------------------------- steps
def router_logits(x_bits, w_router, bias=None, with_absdot=False):
    x = _c(x_bits, np.uint16)
    w = _c(w_router, np.float32)
    b = _c(bias, np.float32)
    T, H = x.shape
    E = w.shape[0]
    out = np.empty((T, E), dtype=np.float64)
    ad = np.empty((T, E), dtype=np.float64) if with_absdot else None
    lib().oracle_router_logits(T, H, E, _p(x), _p(w), _p(b), _p(out), _p(ad))
    return (out, ad) if with_absdot else out


def topk(logits32, k: int):
    l32 = _c(logits32, np.float32)
    T, E = l32.shape
    idx = np.empty((T, k), dtype=np.int32)
    g = np.empty((T, k), dtype=np.float64)
    lib().oracle_topk(T, E, k, _p(l32), _p(idx), _p(g))
    return idx, g


def permute(idx, num_experts: int, num_shared: int = 0):
    idx = _c(idx, np.int32)
    T, k = idx.shape
    G = num_experts + (1 if num_shared else 0)
    n = T * k + (T if num_shared else 0)
    offsets = np.empty(G + 1, dtype=np.int32)
    sf = np.empty(n, dtype=np.int32)
    inv = np.empty(n, dtype=np.int32)
    lib().oracle_permute(T, k, num_experts, 1 if num_shared else 0, _p(idx), _p(offsets), _p(sf), _p(inv))
    return offsets, sf, inv


def expert_ffn(wdtype: int, hidden: int, ffn: int, w13, w13_scale, w2, w2_scale, x64) -> np.ndarray:
    """One token (fp64 vector) through one expert whose weights are passed unstacked."""
    w13 = np.ascontiguousarray(w13)
    w2 = np.ascontiguousarray(w2)
    x = _c(x64, np.float64)
    o = np.empty(hidden, dtype=np.float64)
    lib().oracle_expert_ffn(hidden, ffn, wdtype, _p(w13), _p(_c(w13_scale, np.uint8)), _p(w2),
                            _p(_c(w2_scale, np.uint8)), _p(x), _p(o))
    return o


def moe_layer(shape: dict, x_bits, idx, g, weights: dict, tokens=None, n_threads: int = 0) -> np.ndarray:
    """y[n, H] in fp64 for the listed tokens (all if None), given routing (idx, g)."""
    H, F, E, k, S, wd = (shape[n] for n in ("hidden", "ffn", "num_experts", "top_k", "num_shared", "wdtype"))
    x = _c(x_bits, np.uint16)
    T = x.shape[0]
    idx = _c(idx, np.int32)
    g = _c(g, np.float64)
    tok = _c(tokens, np.int32)
    n = T if tok is None else len(tok)
    y = np.empty((n, H), dtype=np.float64)
    keep = [np.ascontiguousarray(weights[key]) if weights.get(key) is not None else None
            for key in ("w13", "w13_scale", "w2", "w2_scale", "shared_w13", "shared_w13_scale", "shared_w2", "shared_w2_scale")]
    rc = lib().oracle_moe_layer(T, H, F, E, k, S, wd, _p(tok), n, _p(x), _p(idx), _p(g),
                                *[_p(a) for a in keep], _p(y), int(n_threads))
    if rc != 0:
        raise ValueError("oracle_moe_layer: token index out of range")
    return y


def unit_rms(y64, eps: float = 1e-6) -> np.ndarray:
    y = _c(y64, np.float64)
    T, H = y.shape
    out = np.empty_like(y)
    lib().oracle_unit_rms(T, H, _p(y), eps, _p(out))
    return out


def lru_sim(num_experts: int, n_slots: int, steps):
    """steps: list of per-step expert-id lists.  Returns (slot, hit, slot_expert, hits, misses);
    slot/hit are lists aligned with sorted(set(step))."""
    uniq = [sorted(set(int(i) for i in s)) for s in steps]
    counts = np.array([len(u) for u in uniq], dtype=np.int32)
    ids = np.array([i for u in uniq for i in u], dtype=np.int32)
    slot = np.empty(len(ids), dtype=np.int32)
    hit = np.empty(len(ids), dtype=np.uint8)
    se = np.empty((len(uniq), n_slots), dtype=np.int32)
    h = ctypes.c_int64()
    m = ctypes.c_int64()
    rc = lib().oracle_lru_sim(num_experts, n_slots, len(uniq), _p(counts), _p(ids), _p(slot), _p(hit), _p(se),
                              ctypes.byref(h), ctypes.byref(m))
    if rc != 0:
        raise ValueError("oracle_lru_sim: step larger than the slot count or id out of range")
    out_slot, out_hit, b = [], [], 0
    for u in uniq:
        out_slot.append(slot[b:b + len(u)].tolist())
        out_hit.append(hit[b:b + len(u)].astype(bool).tolist())
        b += len(u)
    return out_slot, out_hit, se, h.value, m.value


def lru_sim_global(num_layers: int, num_experts: int, n_slots: int, routed):
    """One LRU cache of n_slots slots shared by all layers, keyed by layer * E + expert
    (global LRU at equal capacity: FreeToken article, dothoosh.com, "Benchmarks and real
    performance").  routed[l][s]: expert ids of layer l at decode step s.  Policy steps run
    in execution order (step 0 layers 0..L-1, step 1 ...), each the same policy as
    lru_sim.  Returns (per-layer hits, per-layer misses, final slot contents)."""
    L, E = num_layers, num_experts
    n_steps = len(routed[0])
    flat = [[l * E + int(e) for e in routed[l][s]] for s in range(n_steps) for l in range(L)]
    _, hit, se, _, _ = lru_sim(L * E, n_slots, flat)
    hits, misses = [0] * L, [0] * L
    for i, h in enumerate(hit):
        hits[i % L] += sum(h)
        misses[i % L] += len(h) - sum(h)
    return hits, misses, (se[-1].tolist() if len(flat) else [-1] * n_slots)


def lru_resize(content, stamp, where, n_new):
    """Slot budget change of one LRU cache state (lists content/stamp, dict where), in place.
    Growing appends empty slots.  Shrinking keeps the n_new occupied slots used most recently
    (largest stamps), empties the rest, then moves each kept expert that sits at slot >= n_new,
    in ascending slot order, to the lowest empty slot below n_new.  Returns the moves
    [(from, to)].  (Elastic expert cache rebuilt under a new VRAM budget at a safe point:
    FreeToken article, dothoosh.com, "FreeToken architecture", mechanism 3.)"""
    n_old = len(content)
    if n_new >= n_old:
        content.extend([-1] * (n_new - n_old))
        stamp.extend([-1] * (n_new - n_old))
        return []
    occupied = [i for i in range(n_old) if content[i] >= 0]
    occupied.sort(key=lambda i: -stamp[i])
    for i in occupied[n_new:]:
        del where[content[i]]
        content[i], stamp[i] = -1, -1
    moves = []
    for i in range(n_new, n_old):
        if content[i] < 0:
            continue
        j = content.index(-1)
        content[j], stamp[j] = content[i], stamp[i]
        where[content[j]] = j
        content[i], stamp[i] = -1, -1
        moves.append((i, j))
    del content[n_new:]
    del stamp[n_new:]
    return moves


def _lru_run(num_keys: int, n_slots: int, steps, resize_before):
    """The decode LRU policy (as lru_sim) in plain Python over policy steps, with slot-budget
    changes {policy step: new slot count} applied before the given steps."""
    content, stamp, where = [-1] * n_slots, [-1] * n_slots, {}
    slots_out, hits_out = [], []
    for s, step in enumerate(steps):
        if s in resize_before:
            lru_resize(content, stamp, where, resize_before[s])
        ids = sorted(set(int(i) for i in step))
        if len(ids) > len(content) or any(u < 0 or u >= num_keys for u in ids):
            raise ValueError("step larger than the slot count or id out of range")
        touched, sl, hit = set(), [None] * len(ids), [False] * len(ids)
        for r, u in enumerate(ids):
            if u in where:
                touched.add(where[u])
                stamp[where[u]] = s * num_keys + r
                sl[r], hit[r] = where[u], True
        for r, u in enumerate(ids):
            if hit[r]:
                continue
            if -1 in content:
                v = content.index(-1)
            else:
                v = min((i for i in range(len(content)) if i not in touched), key=lambda i: stamp[i])
                del where[content[v]]
            content[v], stamp[v], where[u] = u, s * num_keys + r, v
            touched.add(v)
            sl[r] = v
        slots_out.append(sl)
        hits_out.append(hit)
    return slots_out, hits_out, content


def lru_sim_resizable(num_experts: int, n_slots: int, steps, resize_before=None):
    """Per-layer cache with slot-budget changes {decode step: new slots} before those steps.
    Returns (slot, hit, final content, hits, misses)."""
    sl, hit, content = _lru_run(num_experts, n_slots, steps, dict(resize_before or {}))
    h = sum(sum(x) for x in hit)
    return sl, hit, content, h, sum(len(x) for x in hit) - h


def lru_sim_global_resizable(num_layers: int, num_experts: int, slots_per_layer: int, routed, resize_before=None):
    """Global cache (num_layers * slots_per_layer slots, keys layer * E + expert) with budget
    changes {decode step: new slots per layer} before layer 0 of those steps.  Returns
    (per-layer hits, per-layer misses, final content)."""
    L, E = num_layers, num_experts
    n_steps = len(routed[0])
    flat = [[l * E + int(e) for e in routed[l][s]] for s in range(n_steps) for l in range(L)]
    rb = {s * L: L * n for s, n in (resize_before or {}).items()}
    _, hit, content = _lru_run(L * E, L * slots_per_layer, flat, rb)
    hits, misses = [0] * L, [0] * L
    for i, h in enumerate(hit):
        hits[i % L] += sum(h)
        misses[i % L] += len(h) - sum(h)
    return hits, misses, content


def e4m3_round(v: float) -> float:
    return lib().oracle_e4m3_round(float(v))


def mxfp8_qdq(v) -> np.ndarray:
    """Block-scaled E4M3 quantise-dequantise (blocks of 32 along the last axis)."""
    a = _c(v, np.float64)
    out = np.empty_like(a)
    lib().oracle_mxfp8_qdq(a.size, _p(a), _p(out))
    return out


def expert_ffn_mxfp8_act(wdtype: int, hidden: int, ffn: int, w13, w13_scale, w2, w2_scale, x64) -> np.ndarray:
    """expert_ffn with x and h quantised to MXFP8 (E4M3 + E8M0 per 32), for error studies of a
    block-scaled MMA path; not the method's arithmetic."""
    w13 = np.ascontiguousarray(w13)
    w2 = np.ascontiguousarray(w2)
    x = _c(x64, np.float64)
    o = np.empty(hidden, dtype=np.float64)
    lib().oracle_expert_ffn_mxfp8_act(hidden, ffn, wdtype, _p(w13), _p(_c(w13_scale, np.uint8)), _p(w2),
                                      _p(_c(w2_scale, np.uint8)), _p(x), _p(o))
    return o


def mxfp8x2_qdq(v) -> np.ndarray:
    """Two-plane block-scaled E4M3 split: high plane = mxfp8_qdq(v), low plane = mxfp8_qdq of
    the remainder; returns high + low (blocks of 32 along the last axis)."""
    a = _c(v, np.float64)
    out = np.empty_like(a)
    lib().oracle_mxfp8x2_qdq(a.size, _p(a), _p(out))
    return out


def expert_ffn_mxfp8_planes(planes: int, wdtype: int, hidden: int, ffn: int, w13, w13_scale, w2, w2_scale,
                            x64) -> np.ndarray:
    """expert_ffn with x and h quantised to `planes` MXFP8 planes (1 or 2), for error studies
    of a block-scaled MMA path; not the method's arithmetic."""
    w13 = np.ascontiguousarray(w13)
    w2 = np.ascontiguousarray(w2)
    x = _c(x64, np.float64)
    o = np.empty(hidden, dtype=np.float64)
    lib().oracle_expert_ffn_mxfp8_planes(planes, hidden, ffn, wdtype, _p(w13), _p(_c(w13_scale, np.uint8)), _p(w2),
                                         _p(_c(w2_scale, np.uint8)), _p(x), _p(o))
    return o


def full_layer(shape: dict, x_bits, w_router, bias, weights: dict, logits32=None, tokens=None, n_threads: int = 0):
    """Convenience: logits (fp64) -> top-k on the given fp32 logits (or on the fp64 logits
    rounded to fp32 when none are given) -> y for the listed tokens."""
    l64 = router_logits(x_bits, w_router, bias)
    l32 = l64.astype(np.float32) if logits32 is None else np.asarray(logits32, dtype=np.float32)
    idx, g = topk(l32, shape["top_k"])
    y = moe_layer(shape, x_bits, idx, g, weights, tokens, n_threads)
    return dict(logits64=l64, idx=idx, g=g, y=y)

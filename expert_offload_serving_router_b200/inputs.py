"""Seeded synthetic inputs for the sparse-MoE layer (shared by tests, bench and smoke).

This module holds only random-number recipes and dtype packing.  It contains
none of the layer's arithmetic (no routing, no FFN, no combine), so both the
CUDA path and the fp64 oracle can be fed from it without sharing method code.

The source pages measure real checkpoints on agent traces; none of those are
available, so seeded tensors with the pages' layer shapes stand in for them:
DeepSeek-V4-Flash routes 6 of 256 experts per layer (FreeToken write-up,
aihot.vn, "The gap it targets"), Gemma-4-26B-A4B activates 8 routed experts
plus one shared expert per token (TurboFieldfare article, dothoosh.com,
"Background: Gemma 4 26B A4B"), Qwen3.6-35B-A3B is served in BF16 and
DeepSeek-V4-Flash in MXFP4 (FreeToken write-up, dothoosh.com, "Benchmarks").

Recipe (every tensor):
  * generator = numpy PCG64(SeedSequence([seed, config_id, tensor_id, layer]));
    expert weights draw each expert's slice from its own stream
    SeedSequence([seed, config_id, tensor_id, layer, expert]) (so experts can be
    generated in parallel threads);
  * normals are drawn in float32 (numpy's float32 ziggurat), scaled in
    float32, and for bf16 tensors rounded to bf16 (RNE on the float32 bit
    pattern); the router weights stay float32;
  * MXFP4 codes are uniform random bytes (the raw 64-bit PCG64 output viewed
    as bytes: each nibble uniform over the 16 E2M1 codes, -0 included); E8M0
    scale bytes are integers uniform on 119..123, i.e. scales 2^-8 .. 2^-4;
  * the skewed-routing bias is b_e = -s * ln(r_e) with r = 1 + a seeded
    permutation of 0..E-1 and s = 1.0, so exp(b_e) follows Zipf(s) over a
    scattered rank order.
"""
from __future__ import annotations

import concurrent.futures as _cf
import dataclasses
import os

import numpy as np

# tensor ids inside the seed sequence
TID_X, TID_WR, TID_BIAS, TID_W13, TID_W2, TID_W13S, TID_W2S, TID_SW13, TID_SW2, TID_SW13S, TID_SW2S = range(11)

WDTYPE_BF16 = 0
WDTYPE_MXFP4 = 1


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    config_id: int
    hidden: int
    ffn: int
    num_experts: int
    top_k: int
    num_shared: int
    wdtype: int
    zipf_bias: bool
    decode_tokens: tuple
    prefill_tokens: tuple


CONFIGS = {
    "tiny": LayerConfig("tiny", 1, 256, 512, 8, 2, 0, WDTYPE_BF16, False, (), (64,)),
    "qwen3_a3b": LayerConfig("qwen3_a3b", 2, 2048, 768, 128, 8, 0, WDTYPE_BF16, True, (1, 4, 16), (4096,)),
    "dsv4_flash": LayerConfig("dsv4_flash", 3, 4096, 2048, 256, 6, 0, WDTYPE_MXFP4, False, (1, 8), (8192,)),
    "gemma4_26b_a4b": LayerConfig("gemma4_26b_a4b", 4, 2816, 704, 128, 8, 1, WDTYPE_BF16, False, (1,), (2048,)),
}

# Expert-offload stack: 8 DeepSeek-V4-Flash-shaped MXFP4 layers, Zipf-skewed routing,
# 32 HBM expert slots per layer, 8192-token prefill then 256 single-token decode steps.
STACK = dict(layer="dsv4_flash", config_id=5, num_layers=8, slots_per_layer=32,
             prefill_tokens=8192, decode_steps=256, decode_tokens=1, zipf_bias=True)


def rng(seed: int, config_id: int, tensor_id: int, layer: int = 0, *sub: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, config_id, tensor_id, layer, *sub])))


def _per_expert(fn, n_experts: int):
    """Run fn(e) for every expert in a thread pool (numpy's generators release the GIL)."""
    with _cf.ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
        return list(ex.map(fn, range(n_experts)))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round-to-nearest-even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = (u >> 16) & np.uint32(1)
    r += np.uint32(0x7FFF)
    r += u
    r >>= 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _normal_bf16(g: np.random.Generator, shape, std: float, chunk_rows: int | None = None) -> np.ndarray:
    """bf16 N(0, std^2) tensor, drawn slice by slice along axis 0 to bound host memory."""
    out = np.empty(shape, dtype=np.uint16)
    n0 = shape[0]
    step = chunk_rows or n0
    for s in range(0, n0, step):
        v = g.standard_normal((min(step, n0 - s),) + tuple(shape[1:]), dtype=np.float32)
        v *= np.float32(std)
        out[s:s + step] = f32_to_bf16_bits(v)
    return out


def zipf_bias(seed: int, config_id: int, num_experts: int, layer: int = 0, s: float = 1.0) -> np.ndarray:
    r = 1 + rng(seed, config_id, TID_BIAS, layer).permutation(num_experts)
    return (-s * np.log(r.astype(np.float64))).astype(np.float32)


def make_tokens(cfg: LayerConfig, T: int, seed: int = 0, stream: int = 0) -> np.ndarray:
    """x[T, H] as bf16 bits, N(0, 1).  `stream` separates independent batches (e.g. decode steps)."""
    return _normal_bf16(rng(seed, cfg.config_id, TID_X, 1000 + stream), (T, cfg.hidden), 1.0)


def make_router(cfg: LayerConfig, seed: int = 0, layer: int = 0, zipf: bool | None = None):
    w_r = rng(seed, cfg.config_id, TID_WR, layer).standard_normal((cfg.num_experts, cfg.hidden), dtype=np.float32)
    w_r *= np.float32(0.02)
    use_bias = cfg.zipf_bias if zipf is None else zipf
    bias = zipf_bias(seed, cfg.config_id, cfg.num_experts, layer) if use_bias else None
    return w_r, bias


def _stacked_bf16(seed, cid, tid, layer, shape, std):
    """[E, rows, cols] bf16 N(0, std^2); expert e from stream (seed, cid, tid, layer, e)."""
    out = np.empty(shape, dtype=np.uint16)

    def one(e):
        out[e] = _normal_bf16(rng(seed, cid, tid, layer, e), shape[1:], std)
    _per_expert(one, shape[0])
    return out


def _stacked_mxfp4(seed, cid, tid_codes, tid_scales, layer, n_experts, rows, k):
    """codes [E, rows, k/2] (uniform bytes) + E8M0 scales [E, rows, k/32] (uniform 119..123)."""
    codes = np.empty((n_experts, rows, k // 2), dtype=np.uint8)
    scales = np.empty((n_experts, rows, k // 32), dtype=np.uint8)

    def one(e):
        raw = rng(seed, cid, tid_codes, layer, e).bit_generator.random_raw(rows * (k // 2) // 8)
        codes[e] = raw.view(np.uint8).reshape(rows, k // 2)
        scales[e] = rng(seed, cid, tid_scales, layer, e).integers(119, 124, size=(rows, k // 32), dtype=np.uint8)
    _per_expert(one, n_experts)
    return codes, scales


def make_experts(cfg: LayerConfig, seed: int = 0, layer: int = 0, config_id: int | None = None) -> dict:
    """Expert weights of one layer.

    BF16:  w13[E, 2F, H] (rows 0..F-1 gate, F..2F-1 up), w2[E, H, F]; both K-contiguous.
    MXFP4: w13 codes [E, 2F, H/2] + E8M0 scales [E, 2F, H/32]; w2 codes [E, H, F/2] + scales
           [E, H, F/32].  Low nibble = even K index.
    Shared expert (if any) has the same layout with a leading dimension of 1.
    """
    cid = cfg.config_id if config_id is None else config_id
    E, H, F = cfg.num_experts, cfg.hidden, cfg.ffn
    out = {}
    if cfg.wdtype == WDTYPE_BF16:
        out["w13"] = _stacked_bf16(seed, cid, TID_W13, layer, (E, 2 * F, H), 0.02)
        out["w2"] = _stacked_bf16(seed, cid, TID_W2, layer, (E, H, F), 0.02)
        out["w13_scale"] = None
        out["w2_scale"] = None
        if cfg.num_shared:
            out["shared_w13"] = _stacked_bf16(seed, cid, TID_SW13, layer, (1, 2 * F, H), 0.02)
            out["shared_w2"] = _stacked_bf16(seed, cid, TID_SW2, layer, (1, H, F), 0.02)
    else:
        out["w13"], out["w13_scale"] = _stacked_mxfp4(seed, cid, TID_W13, TID_W13S, layer, E, 2 * F, H)
        out["w2"], out["w2_scale"] = _stacked_mxfp4(seed, cid, TID_W2, TID_W2S, layer, E, H, F)
        if cfg.num_shared:
            out["shared_w13"], out["shared_w13_scale"] = _stacked_mxfp4(seed, cid, TID_SW13, TID_SW13S, layer, 1, 2 * F, H)
            out["shared_w2"], out["shared_w2_scale"] = _stacked_mxfp4(seed, cid, TID_SW2, TID_SW2S, layer, 1, H, F)
    return out


def make_layer(cfg: LayerConfig, seed: int = 0, layer: int = 0, zipf: bool | None = None, config_id: int | None = None) -> dict:
    w_r, bias = make_router(cfg, seed, layer, zipf)
    d = make_experts(cfg, seed, layer, config_id)
    d["w_router"] = w_r
    d["bias"] = bias
    return d


def custom_config(name="custom", hidden=256, ffn=512, num_experts=8, top_k=2, num_shared=0,
                  wdtype=WDTYPE_BF16, zipf_bias=False, config_id=99) -> LayerConfig:
    return LayerConfig(name, config_id, hidden, ffn, num_experts, top_k, num_shared, wdtype, zipf_bias, (), ())

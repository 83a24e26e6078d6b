// Internal helpers shared by the libftmoe kernels and host code (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>
#include <stddef.h>

#include "../../include/ftmoe.h"

namespace ftmoe {

constexpr int kMaxExperts = 256;
constexpr int kMaxTopK = 8;
constexpr int kGemmBN = 256;        // token rows per grouped-GEMM tile (max MMA N)
constexpr int kPermChunk = 1024;    // flat pairs per counting-sort chunk
constexpr int kSmallRoute = 32;     // T <= this: split-expert router + fused permute

// ------------------------------------------------------------------ device scalar helpers
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ float bf16f(uint16_t b) { return __uint_as_float(uint32_t(b) << 16); }
__device__ __forceinline__ uint16_t f2bf(float f) {
    __nv_bfloat16 h = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t*>(&h);
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    return uint32_t(f2bf(lo)) | (uint32_t(f2bf(hi)) << 16);
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Transpose-reduce step: n per-lane values -> n/2, pairing lanes across `off`; lanes with
// (lane & off) keep the upper half.  After log2(n) steps plus plain butterfly steps each
// lane holds one complete warp sum (n-1 + 5 - log2 n shuffles instead of 5 n).
__device__ __forceinline__ void tr_step(float* v, int n, int off, int lane) {
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < n / 2; ++i) {
        const float send = up ? v[i] : v[i + n / 2];
        const float recv = __shfl_xor_sync(0xffffffffu, send, off);
        v[i] = (up ? v[i + n / 2] : v[i]) + recv;
    }
}

// silu(a) * b, silu(a) = a * sigmoid(a) = h + h * tanh(h) with h = a/2 (tanh.approx: one MUFU op,
// relative error ~2^-11, below the bf16 rounding of the result)
__device__ __forceinline__ float tanh_approx(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float silu_mul(float a, float b) {
    const float h = 0.5f * a;
    return fmaf(h, tanh_approx(h), h) * b;
}

// ------------------------------------------------------------------ workspace layout
// One layout serves every entry point: a region is only touched by the steps that need it.
struct WsLayout {
    size_t logits, topk_idx, topk_w, offsets, sorted_flat, inv_pos;
    size_t chunk_cnt, chunk_base, local_rank, sched, err;
    size_t x_sorted, h, o_sorted;
    size_t wr_planes;   // router weights as three bf16 planes (prefill-sized batches only)
    size_t route_part;  // partial logits of the prefill router, one slab per K split
    size_t mx_decode;   // activation planes of the block-scaled MXFP4 decode (decode-sized batches)
    size_t total;
    int T, P, R, G, C;
};

__host__ __device__ inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Workspace header (cleared by ft_moe_workspace_init): word 0 device error flag, word 1 the
// decode router's ticket (left at zero by every launch), words kWsReady.. the tensor-core
// decode's per-group counters (2 x (E + S) words, left at zero by every launch and zeroed by
// the decode permutation); the rest is reserved.
constexpr size_t kWsHeaderBytes = 4096;
constexpr int kWsReady = 64;            // word index; 2 x 257 counters fit
constexpr int kRouteTok = 128;          // tokens per router CTA
constexpr int kRouteTargetCtas = 148;   // split K until the router grid covers about one wave
constexpr int kRouteMaxSplit = 8;

// K splits of the prefill router for T tokens, H hidden (each split keeps >= 1 K stage of 64)
__host__ __device__ inline int route_splits(int T, int H) {
    const int tiles = (T + kRouteTok - 1) / kRouteTok;
    if (tiles <= 0) return 1;
    int ks = kRouteTargetCtas / tiles;
    if (ks > kRouteMaxSplit) ks = kRouteMaxSplit;
    if (ks > H / 64) ks = H / 64;
    return ks < 1 ? 1 : ks;
}

// sched region: [0] total GEMM tiles for BN, [1] n_active groups, [2..] ntile_off[G+1], then active[G]
inline WsLayout make_layout(const ft_moe_shape& s, int T) {
    WsLayout L{};
    L.T = T;
    L.P = T * s.top_k;
    L.G = s.num_experts + (s.num_shared ? 1 : 0);
    L.R = L.P + (s.num_shared ? T : 0);
    L.C = (L.R + kPermChunk - 1) / kPermChunk;
    if (L.C < 1) L.C = 1;
    size_t o = 0;
    auto take = [&](size_t bytes) { size_t r = o; o = align256(o + bytes); return r; };
    L.err = take(kWsHeaderBytes);   // first: [0] device error flag, [1] decode-router ticket, down tickets
    L.logits = take(sizeof(float) * size_t(T) * s.num_experts);
    L.topk_idx = take(sizeof(int32_t) * size_t(L.P));
    L.topk_w = take(sizeof(float) * size_t(L.P));
    L.offsets = take(sizeof(int32_t) * size_t(L.G + 1));
    L.sorted_flat = take(sizeof(int32_t) * size_t(L.R));
    L.inv_pos = take(sizeof(int32_t) * size_t(L.R));
    L.chunk_cnt = take(sizeof(int32_t) * size_t(L.C) * L.G);
    L.chunk_base = take(sizeof(int32_t) * size_t(L.C) * L.G);
    L.local_rank = take(sizeof(int32_t) * size_t(L.R));
    L.sched = take(sizeof(int32_t) * size_t(2 + 2 * (L.G + 1)));
    L.x_sorted = take(sizeof(uint16_t) * size_t(L.R) * s.hidden);
    L.h = take(sizeof(uint16_t) * size_t(L.R) * s.ffn);
    L.o_sorted = take(sizeof(uint16_t) * size_t(L.R) * s.hidden);
    L.wr_planes = take(T > kSmallRoute ? size_t(3) * size_t((s.num_experts + 15) & ~15) * s.hidden * 2 : 0);
    L.route_part = take(T > kSmallRoute ? size_t(route_splits(T, s.hidden)) * ((T + kRouteTok - 1) / kRouteTok) *
                                              kRouteTok * ((s.num_experts + 15) & ~15) * sizeof(float) : 0);
    // two E4M3 planes + E8M0 scales of x (32 rows) and of h (R rows): decode-sized MXFP4 batches
    L.mx_decode = take(T <= kSmallRoute && s.wdtype == FT_W_MXFP4
                           ? 2 * (32 * size_t(s.hidden) + size_t(s.hidden)) + 2 * (size_t(L.R) * s.ffn + size_t(L.R) * s.ffn / 32) + 2048
                           : 0);
    L.total = o;
    return L;
}

// device error codes written into ws err[0]
enum : uint32_t { kDevErrNone = 0, kDevErrBadExpert = 1, kDevErrTimeout = 2, kDevErrShape = 3, kDevErrBounds = 4 };

#ifndef FT_DEBUG_BOUNDS
#define FT_DEBUG_BOUNDS 0
#endif

}  // namespace ftmoe

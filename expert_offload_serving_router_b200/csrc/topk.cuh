// Top-k of one token's router logits, shared by the decode and the prefill routers:
// experts ordered by logit descending, the lower index first on equal logits; gates =
// softmax over the kept logits (fp32, summed in slot order).
//
// The prefill router keeps a Top8 list sorted in registers per thread: offering a candidate
// costs a fixed, branch-free sequence (8 compares, 16 selects per array) so a warp of tokens
// never diverges on it, and a group of lanes merges its lists with a bitonic butterfly.  The
// decode router's last CTA gives each token a warp and selects by warp reductions instead.
#pragma once
#include "common.cuh"

namespace ftmoe {

// Order-preserving 32-bit key of an fp32 logit (larger logit -> larger key); -0 is folded
// onto +0 first so that they compare equal, as floats do.  Key 0 sorts below every logit.
__device__ __forceinline__ uint32_t logit_key(float v) {
    uint32_t u = __float_as_uint(v);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_logit(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

struct Top8 {
    uint32_t key[kMaxTopK];
    int32_t idx[kMaxTopK];

    __device__ __forceinline__ void init() {
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) { key[j] = 0u; idx[j] = 0; }
    }
    // Offer expert e with key kv.  Experts must be offered in ascending index order: an
    // equal key already in the list then has the lower index and stays ahead (>=).
    __device__ __forceinline__ void offer(uint32_t kv, int32_t e) {
        bool ge[kMaxTopK];
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) ge[j] = key[j] >= kv;
#pragma unroll
        for (int j = kMaxTopK - 1; j > 0; --j) {
            key[j] = ge[j] ? key[j] : (ge[j - 1] ? kv : key[j - 1]);
            idx[j] = ge[j] ? idx[j] : (ge[j - 1] ? e : idx[j - 1]);
        }
        key[0] = ge[0] ? key[0] : kv;
        idx[0] = ge[0] ? idx[0] : e;
    }
};

// (key desc, index asc) as one unsigned 64-bit order: key high, complemented index low.
__device__ __forceinline__ uint64_t top_pack(uint32_t k, int32_t e) {
    return (uint64_t(k) << 32) | uint64_t(~uint32_t(e));
}

// Merge the lists of a group of `width` lanes (a power of two <= 32, aligned; each list
// sorted, over disjoint expert sets) into the group's top 8; every lane of the group ends
// with the same list.  All 32 lanes must call it.  Each butterfly step: c[j] = max(c[j],
// partner[7-j]) holds the top 8 of both lists as a bitonic sequence, three compare-exchange
// stages sort it.
__device__ __forceinline__ void group_merge_top8(Top8& t, int width) {
    uint64_t c[kMaxTopK];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) c[j] = top_pack(t.key[j], t.idx[j]);
#pragma unroll 1
    for (int off = width >> 1; off >= 1; off >>= 1) {
        uint64_t o[kMaxTopK];
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) o[j] = __shfl_xor_sync(0xffffffffu, c[j], off);
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) c[j] = c[j] > o[kMaxTopK - 1 - j] ? c[j] : o[kMaxTopK - 1 - j];
#pragma unroll
        for (int d = kMaxTopK / 2; d >= 1; d >>= 1) {
#pragma unroll
            for (int j = 0; j < kMaxTopK; ++j) {
                if ((j & d) == 0) {
                    const uint64_t a = c[j], b = c[j + d];
                    c[j] = a > b ? a : b;
                    c[j + d] = a > b ? b : a;
                }
            }
        }
    }
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
        t.key[j] = uint32_t(c[j] >> 32);
        t.idx[j] = int32_t(~uint32_t(c[j]));
    }
}

// Gate of slot j of the first k: exp(l_j - l_0) / sum_{i<k} exp(l_i - l_0).
__device__ __forceinline__ float top_den(const Top8& t, int k) {
    const float l0 = key_logit(t.key[0]);
    float den = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j)
        if (j < k) den += expf(key_logit(t.key[j]) - l0);
    return den;
}

// Slot j of the list and its gate (j is a runtime lane index: selected, not indexed).
__device__ __forceinline__ void top_slot(const Top8& t, int k, int j, int32_t* e_out, float* w_out) {
    const float l0 = key_logit(t.key[0]);
    const float den = top_den(t, k);
    uint32_t kk = 0u;
    int32_t ee = 0;
#pragma unroll
    for (int i = 0; i < kMaxTopK; ++i)
        if (i == j) { kk = t.key[i]; ee = t.idx[i]; }
    *e_out = ee;
    *w_out = expf(key_logit(kk) - l0) / den;
}

// Warp-wide top-k over the E <= 256 logits of one token.  warp_topk_keys reads the row from
// global memory `row` (L2: other CTAs wrote it) into registers -- lane l holds the keys of
// experts l, l+32, ... -- so a caller can have the next token's loads in flight while it selects
// this one.  warp_topk_select takes k rounds: each takes the warp's largest key (one
// max-reduction) and, among the lanes holding it, the lowest expert (one min-reduction), then
// the owning lane drops it.  Same order as Top8 (logit desc, index asc; key 0 never chosen) and
// the same gates; lanes 0..k-1 write slot = lane.
constexpr int kTopkPer = kMaxExperts / 32;
__device__ __forceinline__ void warp_topk_keys(const float* row, int E, uint32_t (&key)[kTopkPer]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int s = 0; s < kTopkPer; ++s) {
        const int e = lane + 32 * s;
        key[s] = e < E ? logit_key(__ldcg(row + e)) : 0u;
    }
}
__device__ inline void warp_topk_select(uint32_t (&key)[kTopkPer], int k, int32_t* idx_out, float* w_out,
                                        int32_t* idx_smem) {
    const int lane = threadIdx.x & 31;
    Top8 t;
    t.init();
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
        if (j >= k) break;
        uint32_t bk = 0u, be = 0xffffffffu;        // this lane's best: experts ascend with s
#pragma unroll
        for (int s = 0; s < kTopkPer; ++s) {
            const bool better = key[s] > bk;
            bk = better ? key[s] : bk;
            be = better ? uint32_t(lane + 32 * s) : be;
        }
        const uint32_t mk = __reduce_max_sync(0xffffffffu, bk);
        if (mk == 0u) break;                       // only key-0 experts left: slots stay (0, 0)
        const uint32_t me = __reduce_min_sync(0xffffffffu, bk == mk ? be : 0xffffffffu);
#pragma unroll
        for (int s = 0; s < kTopkPer; ++s)
            if (uint32_t(lane + 32 * s) == me) key[s] = 0u;
        t.key[j] = mk;
        t.idx[j] = int32_t(me);
    }
    if (lane < k) {
        int32_t ee;
        float ww;
        top_slot(t, k, lane, &ee, &ww);
        idx_out[lane] = ee;
        w_out[lane] = ww;
        if (idx_smem) idx_smem[lane] = ee;
    }
}

}  // namespace ftmoe

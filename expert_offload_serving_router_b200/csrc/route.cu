// Step 1 -- router: fp32 logits l = x Wr^T + b, top-k by (logit desc, index asc),
// gates = softmax over the k kept logits.
//
// Two launch shapes:
//  * T > 32 (prefill): the tensor-core router of route_sm100.cu (router weights split
//    exactly into three bf16 planes, tcgen05 MMAs, per-thread top-k from TMEM).
//  * route_small_kernel (T <= 32): decode batches, fp32 SIMT.  One CTA per expert streams
//    that expert's router row once for all T tokens (spreads the Wr read over E CTAs), and
//    the last CTA to finish (atomic ticket, no waiting) does the top-k for every token
//    and, optionally, the counting-sort permutation of the routed pairs.
#include "kernels.h"
#include "permute_small.cuh"
#include "topk.cuh"

namespace ftmoe {

// ------------------------------------------------------------------ T <= 32
struct SmallRouteArgs {
    int T, H, E, k, S;
    const uint16_t* x;
    const float* wr;
    const float* bias;
    int32_t* topk_idx;
    float* topk_w;
    float* logits;          // [T,E] (always written: the last CTA reads it back)
    uint32_t* ticket;       // zero before launch; the last CTA resets it
    int do_permute;
    PermOut perm;
};

// TOK tokens per pass, NI float4s of the router row per thread and pass of the row: every x load
// of a pass is issued before any is used (TOK x NI 8-byte loads in flight per thread), so a pass
// costs one L2 round trip rather than one per token.
template <int TOK, int NI>
__global__ void __launch_bounds__(256) route_small_kernel(SmallRouteArgs a) {
    __shared__ float red[kSmallRoute][8];
    __shared__ int last;
    const int e = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nq = a.H >> 2;      // float4s per row
    const float* wrow = a.wr + size_t(e) * a.H;
    for (int t = tid; t < kSmallRoute * 8; t += 256) (&red[0][0])[t] = 0.f;
    __syncthreads();
    for (int base = 0; base < nq; base += 256 * NI) {
        float4 w[NI];
#pragma unroll
        for (int i = 0; i < NI; ++i) {
            int q = base + tid + 256 * i;
            w[i] = q < nq ? __ldg(reinterpret_cast<const float4*>(wrow) + q) : make_float4(0, 0, 0, 0);
        }
        // weights do not depend on the preceding kernel: wait for it only before reading x.
        // Only then let the expert kernels that follow (programmatic dependents) be scheduled:
        // they stage x before their own wait, so x must be final by the time they start.
        if (base == 0) {
            asm volatile("griddepcontrol.wait;" ::: "memory");
            asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
        }
        for (int t0 = 0; t0 < a.T; t0 += TOK) {
            // loads with clamped indices (rows past T re-read the last token, vectors past the
            // row's end its last vector): no branch between them; both kinds are dropped below
            uint2 u[TOK][NI];
#pragma unroll
            for (int j = 0; j < TOK; ++j) {
                const uint2* xr = reinterpret_cast<const uint2*>(a.x + size_t(min(t0 + j, a.T - 1)) * a.H);
#pragma unroll
                for (int i = 0; i < NI; ++i) u[j][i] = __ldg(xr + min(base + tid + 256 * i, nq - 1));
            }
            float s[TOK];
#pragma unroll
            for (int j = 0; j < TOK; ++j) {
                s[j] = 0.f;
#pragma unroll
                for (int i = 0; i < NI; ++i) {
                    if (base + tid + 256 * i < nq) {
                        s[j] = fmaf(bf16lo(u[j][i].x), w[i].x, s[j]);
                        s[j] = fmaf(bf16hi(u[j][i].x), w[i].y, s[j]);
                        s[j] = fmaf(bf16lo(u[j][i].y), w[i].z, s[j]);
                        s[j] = fmaf(bf16hi(u[j][i].y), w[i].w, s[j]);
                    }
                }
            }
            // transpose-reduce: lane l ends with the warp sum of token t0 + (its TOK-slot from
            // bits 4, 3 (and 2) of l)
            int t;
            if (TOK == 1) {
#pragma unroll
                for (int o = 16; o; o >>= 1) s[0] += __shfl_xor_sync(0xffffffffu, s[0], o);
                t = lane == 0 ? t0 : a.T;
            } else if (TOK == 8) {
                tr_step(s, 8, 16, lane);
                tr_step(s, 4, 8, lane);
                tr_step(s, 2, 4, lane);
                s[0] += __shfl_xor_sync(0xffffffffu, s[0], 2);
                s[0] += __shfl_xor_sync(0xffffffffu, s[0], 1);
                t = (lane & 3) == 0 ? t0 + ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1) : a.T;
            } else {   // TOK == 4
                tr_step(s, 4, 16, lane);
                tr_step(s, 2, 8, lane);
                s[0] += __shfl_xor_sync(0xffffffffu, s[0], 4);
                s[0] += __shfl_xor_sync(0xffffffffu, s[0], 2);
                s[0] += __shfl_xor_sync(0xffffffffu, s[0], 1);
                t = (lane & 7) == 0 ? t0 + ((lane >> 4) & 1) * 2 + ((lane >> 3) & 1) : a.T;
            }
            if (t < a.T) red[t][warp] += s[0];
        }
    }
    __syncthreads();
    if (tid < a.T) {
        float l = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) l += red[tid][w];
        if (a.bias) l += a.bias[e];
        a.logits[size_t(tid) * a.E + e] = l;
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) last = (atomicAdd(a.ticket, 1u) == gridDim.x - 1);
    __syncthreads();
    if (!last) return;
    __threadfence();
    // ---- last CTA: top-k for every token (+ permutation), a warp per token; the next token's
    // logits load while this one's are selected
    __shared__ int32_t sidx[kSmallRoute * kMaxTopK];
    uint32_t key[kTopkPer], nkey[kTopkPer];
    if (warp < a.T) warp_topk_keys(a.logits + size_t(warp) * a.E, a.E, key);
    for (int t = warp; t < a.T; t += 8) {
        if (t + 8 < a.T) warp_topk_keys(a.logits + size_t(t + 8) * a.E, a.E, nkey);
        warp_topk_select(key, a.k, a.topk_idx + size_t(t) * a.k, a.topk_w + size_t(t) * a.k, sidx + t * a.k);
#pragma unroll
        for (int s = 0; s < kTopkPer; ++s) key[s] = nkey[s];
    }
    if (tid == 0) *a.ticket = 0u;
    __syncthreads();
    if (!a.do_permute) return;
    __shared__ int cnt[kMaxExperts + 2];
    if (warp == 0) warp_permute_small(sidx, a.T, a.k, a.E, a.S, cnt, a.perm);
}

// ------------------------------------------------------------------ host launchers
cudaError_t launch_route(int T, int H, int E, int k, int S, const uint16_t* x, const float* wr, const float* bias,
                         int32_t* topk_idx, float* topk_w, float* logits, uint32_t* err, uint16_t* planes,
                         float* part, const PermOut* perm, cudaStream_t st) {
    if (T <= 0) return cudaSuccess;
    if (T <= kSmallRoute) {
        SmallRouteArgs a{T, H, E, k, S, x, wr, bias, topk_idx, topk_w, logits, err + 1, perm != nullptr, {}};
        if (perm) a.perm = *perm;
        // programmatic dependent launch: the router rows stream while the preceding kernel
        // (the previous layer's down GEMV) finishes
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(E);
        cfg.blockDim = dim3(256);
        cfg.stream = st;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        at[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        // hidden <= 2048: two row vectors per thread, eight tokens a pass; wider rows: four and
        // four; a single token: one a pass
        const bool narrow = H / 4 <= 512;
        cudaError_t e = T == 1 ? (narrow ? cudaLaunchKernelEx(&cfg, route_small_kernel<1, 2>, a)
                                         : cudaLaunchKernelEx(&cfg, route_small_kernel<1, 4>, a))
                               : (narrow ? cudaLaunchKernelEx(&cfg, route_small_kernel<8, 2>, a)
                                         : cudaLaunchKernelEx(&cfg, route_small_kernel<4, 4>, a));
        if (e != cudaSuccess || !perm) return e;
        return launch_perm_check(topk_idx, T, k, E, S, *perm, st);
    }
    if (perm) return cudaErrorInvalidValue;   // the fused permutation exists only for decode-sized batches
    return launch_route_tc(T, H, E, k, x, wr, bias, topk_idx, topk_w, logits, planes, part, err, st);
}

}  // namespace ftmoe

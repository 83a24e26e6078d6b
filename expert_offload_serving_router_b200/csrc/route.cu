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

__global__ void __launch_bounds__(256) route_small_kernel(SmallRouteArgs a) {
    __shared__ float red[kSmallRoute][8];
    __shared__ int last;
    const int e = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nq = a.H >> 2;      // float4s per row
    const float* wrow = a.wr + size_t(e) * a.H;
    for (int t = tid; t < kSmallRoute * 8; t += 256) (&red[0][0])[t] = 0.f;
    __syncthreads();
    for (int base = 0; base < nq; base += 256 * 4) {
        float4 w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
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
        // eight tokens per pass: all their x loads in flight together, then one transpose-
        // reduce leaves token t0 + 4*bit4(lane) + 2*bit3(lane) + bit2(lane) on lane
        for (int t0 = 0; t0 < a.T; t0 += 8) {
            float s[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                s[j] = 0.f;
                if (t0 + j < a.T) {
                    const uint2* xr = reinterpret_cast<const uint2*>(a.x + size_t(t0 + j) * a.H);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        int q = base + tid + 256 * i;
                        if (q < nq) {
                            uint2 u = __ldg(xr + q);
                            s[j] = fmaf(bf16lo(u.x), w[i].x, s[j]);
                            s[j] = fmaf(bf16hi(u.x), w[i].y, s[j]);
                            s[j] = fmaf(bf16lo(u.y), w[i].z, s[j]);
                            s[j] = fmaf(bf16hi(u.y), w[i].w, s[j]);
                        }
                    }
                }
            }
            tr_step(s, 8, 16, lane);
            tr_step(s, 4, 8, lane);
            tr_step(s, 2, 4, lane);
            s[0] += __shfl_xor_sync(0xffffffffu, s[0], 2);
            s[0] += __shfl_xor_sync(0xffffffffu, s[0], 1);
            const int t = t0 + ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1);
            if ((lane & 3) == 0 && t < a.T) red[t][warp] += s[0];
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
    // ---- last CTA: top-k for every token (+ permutation), a warp per token
    __shared__ int32_t sidx[kSmallRoute * kMaxTopK];
    for (int t = warp; t < a.T; t += 8)
        warp_topk_row(a.logits + size_t(t) * a.E, a.E, a.k, a.topk_idx + size_t(t) * a.k, a.topk_w + size_t(t) * a.k,
                      sidx + t * a.k);
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
        cudaError_t e = cudaLaunchKernelEx(&cfg, route_small_kernel, a);
        if (e != cudaSuccess || !perm) return e;
        return launch_perm_check(topk_idx, T, k, E, S, *perm, st);
    }
    if (perm) return cudaErrorInvalidValue;   // the fused permutation exists only for decode-sized batches
    return launch_route_tc(T, H, E, k, x, wr, bias, topk_idx, topk_w, logits, planes, part, err, st);
}

}  // namespace ftmoe

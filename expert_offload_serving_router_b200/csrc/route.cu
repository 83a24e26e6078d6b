// Step 1 -- router: fp32 logits l = x Wr^T + b, top-k by (logit desc, index asc),
// gates = softmax over the k kept logits.  No tensor cores: the router is fp32 SIMT.
//
// Two launch shapes:
//  * route_tile_kernel (T > 32): one CTA owns 32 tokens x all E experts (E <= 256),
//    a register-blocked SIMT GEMM (8 tokens x 8 experts per thread, K staged through
//    shared memory), then one warp per token does the register top-k from shared memory.
//  * route_small_kernel (T <= 32): decode batches.  One CTA per expert streams that
//    expert's router row once for all T tokens (spreads the Wr read over E CTAs), and
//    the last CTA to finish (atomic ticket, no waiting) does the top-k for every token
//    and, optionally, the counting-sort permutation of the routed pairs.
#include "kernels.h"
#include "permute_small.cuh"

namespace ftmoe {

// Warp-wide top-k over the E logits of one token held in `row` (shared memory).
// Lane l owns experts l, l+32, ...  Ties resolve to the lower index; -0 == +0 as floats.
__device__ inline void warp_topk_row(const float* row, int E, int k, int32_t* idx_out, float* w_out,
                                     int32_t* idx_smem) {
    const int lane = threadIdx.x & 31;
    float v[kMaxExperts / 32];
    uint32_t taken = 0;
#pragma unroll
    for (int i = 0; i < kMaxExperts / 32; ++i) {
        int e = lane + 32 * i;
        v[i] = e < E ? row[e] : -INFINITY;
    }
    float sel_v[kMaxTopK];
    int sel_e[kMaxTopK];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
        if (j >= k) break;
        float bv = -INFINITY;
        int be = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < kMaxExperts / 32; ++i) {
            int e = lane + 32 * i;
            bool ok = e < E && !((taken >> i) & 1u);
            if (ok && (v[i] > bv || (v[i] == bv && e < be))) { bv = v[i]; be = e; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            int oe = __shfl_xor_sync(0xffffffffu, be, o);
            if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        sel_v[j] = bv;
        sel_e[j] = be;
    }
    // gates: softmax over the kept logits, fp32, summed in slot order
    float den = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j)
        if (j < k) den += expf(sel_v[j] - sel_v[0]);
    if (lane < k) {
        float num = 0.f;
        int ee = 0;
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j)
            if (j == lane) { num = expf(sel_v[j] - sel_v[0]); ee = sel_e[j]; }
        idx_out[lane] = ee;
        w_out[lane] = num / den;
        if (idx_smem) idx_smem[lane] = ee;
    }
}

// ------------------------------------------------------------------ T > 32
constexpr int kRtTok = 32;    // tokens per CTA
constexpr int kRtBK = 32;     // K slice staged per iteration
constexpr int kRtLd = kRtBK + 4;

__global__ void __launch_bounds__(128)
route_tile_kernel(int T, int H, int E, int k, const uint16_t* __restrict__ x, const float* __restrict__ wr,
                  const float* __restrict__ bias, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                  float* __restrict__ logits) {
    extern __shared__ float4 smem4[];
    float* ws = reinterpret_cast<float*>(smem4);            // [256][kRtLd]  (reused as logit tile)
    float* xs = ws + kMaxExperts * kRtLd;                   // [32][kRtLd]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t0 = blockIdx.x * kRtTok;
    float acc[8][8];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;

    for (int k0 = 0; k0 < H; k0 += kRtBK) {
        // W slice: E rows x 32 floats, 8 float4 per row, 8 consecutive threads per row
        for (int f = tid; f < E * 8; f += 128) {
            int e = f >> 3, q = f & 7;
            float4 w4 = *reinterpret_cast<const float4*>(wr + size_t(e) * H + k0 + q * 4);
            *reinterpret_cast<float4*>(ws + e * kRtLd + q * 4) = w4;
        }
        // x slice: 32 tokens x 32 bf16 (4 x 16 B per token)
        {
            int t = tid >> 2, q = tid & 3;
            uint4 u = make_uint4(0, 0, 0, 0);
            if (t0 + t < T) u = *reinterpret_cast<const uint4*>(x + size_t(t0 + t) * H + k0 + q * 8);
            float* d = xs + t * kRtLd + q * 8;
            d[0] = bf16lo(u.x); d[1] = bf16hi(u.x); d[2] = bf16lo(u.y); d[3] = bf16hi(u.y);
            d[4] = bf16lo(u.z); d[5] = bf16hi(u.z); d[6] = bf16lo(u.w); d[7] = bf16hi(u.w);
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kRtBK; kk += 4) {
            float4 xv[8], wv[8];
#pragma unroll
            for (int a = 0; a < 8; ++a) xv[a] = *reinterpret_cast<const float4*>(xs + (warp * 8 + a) * kRtLd + kk);
#pragma unroll
            for (int b = 0; b < 8; ++b) wv[b] = *reinterpret_cast<const float4*>(ws + (lane + 32 * b) * kRtLd + kk);
#pragma unroll
            for (int a = 0; a < 8; ++a)
#pragma unroll
                for (int b = 0; b < 8; ++b) {
                    acc[a][b] = fmaf(xv[a].x, wv[b].x, acc[a][b]);
                    acc[a][b] = fmaf(xv[a].y, wv[b].y, acc[a][b]);
                    acc[a][b] = fmaf(xv[a].z, wv[b].z, acc[a][b]);
                    acc[a][b] = fmaf(xv[a].w, wv[b].w, acc[a][b]);
                }
        }
        __syncthreads();
    }
    // logits -> shared tile [32][E] (+ global when requested)
    float* lt = ws;
#pragma unroll
    for (int b = 0; b < 8; ++b) {
        int e = lane + 32 * b;
        if (e >= E) continue;
        float bb = bias ? bias[e] : 0.f;
#pragma unroll
        for (int a = 0; a < 8; ++a) {
            int t = warp * 8 + a;
            float l = acc[a][b] + bb;
            lt[t * kMaxExperts + e] = l;
            if (logits && t0 + t < T) logits[size_t(t0 + t) * E + e] = l;
        }
    }
    __syncwarp();
    // each warp handles its own 8 tokens
    for (int a = 0; a < 8; ++a) {
        int t = t0 + warp * 8 + a;
        if (t >= T) break;
        warp_topk_row(lt + (warp * 8 + a) * kMaxExperts, E, k, topk_idx + size_t(t) * k, topk_w + size_t(t) * k,
                      nullptr);
    }
}

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
        for (int t = 0; t < a.T; ++t) {
            const uint2* xr = reinterpret_cast<const uint2*>(a.x + size_t(t) * a.H);
            float s = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                int q = base + tid + 256 * i;
                if (q < nq) {
                    uint2 u = __ldg(xr + q);
                    s = fmaf(bf16lo(u.x), w[i].x, s);
                    s = fmaf(bf16hi(u.x), w[i].y, s);
                    s = fmaf(bf16lo(u.y), w[i].z, s);
                    s = fmaf(bf16hi(u.y), w[i].w, s);
                }
            }
            s = warp_sum(s);
            if (lane == 0) red[t][warp] += s;
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
    // ---- last CTA: top-k for every token (+ permutation)
    __shared__ float lrow[8][kMaxExperts];
    __shared__ int32_t sidx[kSmallRoute * kMaxTopK];
    for (int t = warp; t < a.T; t += 8) {
        for (int i = lane; i < a.E; i += 32) lrow[warp][i] = __ldcg(a.logits + size_t(t) * a.E + i);
        __syncwarp();
        warp_topk_row(lrow[warp], a.E, a.k, a.topk_idx + size_t(t) * a.k, a.topk_w + size_t(t) * a.k,
                      sidx + t * a.k);
        __syncwarp();
    }
    if (tid == 0) *a.ticket = 0u;
    __syncthreads();
    if (!a.do_permute) return;
    __shared__ int grp[kSmallRoute * (kMaxTopK + 1)];
    __shared__ int cnt[kMaxExperts + 2];
    __shared__ int flag[kMaxExperts + 2];
    __shared__ int tmp[33];
    block_permute_small(sidx, a.T, a.k, a.E, a.S, grp, cnt, flag, tmp, a.perm);
}

// ------------------------------------------------------------------ host launchers
cudaError_t launch_route(int T, int H, int E, int k, int S, const uint16_t* x, const float* wr, const float* bias,
                         int32_t* topk_idx, float* topk_w, float* logits, uint32_t* ticket, const PermOut* perm,
                         cudaStream_t st) {
    if (T <= 0) return cudaSuccess;
    if (T <= kSmallRoute) {
        SmallRouteArgs a{T, H, E, k, S, x, wr, bias, topk_idx, topk_w, logits, ticket, perm != nullptr, {}};
        if (perm) a.perm = *perm;
        route_small_kernel<<<E, 256, 0, st>>>(a);
        return cudaGetLastError();
    }
    size_t smem = sizeof(float) * (kMaxExperts * kRtLd + kRtTok * kRtLd);
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(route_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    int grid = (T + kRtTok - 1) / kRtTok;
    route_tile_kernel<<<grid, 128, smem, st>>>(T, H, E, k, x, wr, bias, topk_idx, topk_w, logits);
    return cudaGetLastError();
}

}  // namespace ftmoe

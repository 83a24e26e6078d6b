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
constexpr int kRtTok = 32;          // tokens per CTA (8 per warp)
constexpr int kRtBK = 32;           // K slice staged per pipeline stage
constexpr int kRtStages = 4;        // cp.async pipeline depth
constexpr int kRtLdW = kRtBK + 4;   // floats per staged router row (conflict-free float4 reads)
constexpr int kRtLdX = kRtBK + 8;   // bf16 per staged token row

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(uint32_t(__cvta_generic_to_shared(smem))),
                 "l"(gmem), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// NE = router rows per lane for all E (E <= 32*NE).  256 threads: warp w owns tokens
// 8*(w&3) .. +7 and expert half w>>2 (NEH = ceil(NE/2) rows per lane), so two warps share
// each scheduler for latency hiding.  K slices of the router rows and token rows stream
// through a 4-stage cp.async ring (one barrier per slice).
template <int NE>
__global__ void __launch_bounds__(256)
route_tile_kernel(int T, int H, int E, int k, const uint16_t* __restrict__ x, const float* __restrict__ wr,
                  const float* __restrict__ bias, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                  float* __restrict__ logits) {
    extern __shared__ float4 smem4[];
    constexpr int kRows = 32 * NE;
    constexpr int NEH = NE >= 2 ? NE / 2 : 1;
    float* wbuf = reinterpret_cast<float*>(smem4);                                   // [S][kRows][kRtLdW]
    uint16_t* xbuf = reinterpret_cast<uint16_t*>(wbuf + kRtStages * kRows * kRtLdW); // [S][32][kRtLdX]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tg = warp & 3, eh = warp >> 2;
    const int ebase = eh * 32 * NEH;
    const int t0 = blockIdx.x * kRtTok;
    const int nk = H / kRtBK;

    auto stage = [&](int s, int k0) {
        float* wd = wbuf + s * kRows * kRtLdW;
        for (int f = tid; f < E * 8; f += 256) {
            const int e = f >> 3, q = f & 7;
            cp_async16(wd + e * kRtLdW + q * 4, wr + size_t(e) * H + k0 + q * 4, 16);
        }
        if (tid < 128) {
            const int t = tid >> 2, q = tid & 3;
            const bool ok = t0 + t < T;
            cp_async16(xbuf + (s * kRtTok + t) * kRtLdX + q * 8, x + size_t(ok ? t0 + t : 0) * H + k0 + q * 8,
                       ok ? 16 : 0);
        }
        cp_async_commit();
    };

    float acc[8][NEH];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < NEH; ++b) acc[a][b] = 0.f;

#pragma unroll
    for (int s = 0; s < kRtStages - 1; ++s) {
        if (s < nk) stage(s, s * kRtBK);
        else cp_async_commit();
    }
    for (int kb = 0; kb < nk; ++kb) {
        cp_async_wait<kRtStages - 2>();     // slice kb has landed (this thread's copies)
        __syncthreads();                    // ... and everyone's; slice kb-1 is no longer read
        const int nxt = kb + kRtStages - 1;
        if (nxt < nk) stage(nxt % kRtStages, nxt * kRtBK);
        else cp_async_commit();
        const float* wsm = wbuf + (kb % kRtStages) * kRows * kRtLdW;
        const uint16_t* xsm = xbuf + (kb % kRtStages) * kRtTok * kRtLdX;
#pragma unroll
        for (int kk = 0; kk < kRtBK; kk += 4) {
            float4 wv[NEH];
#pragma unroll
            for (int b = 0; b < NEH; ++b)
                wv[b] = *reinterpret_cast<const float4*>(wsm + (ebase + lane + 32 * b) * kRtLdW + kk);
#pragma unroll
            for (int a = 0; a < 8; ++a) {
                const uint2 u = *reinterpret_cast<const uint2*>(xsm + (tg * 8 + a) * kRtLdX + kk);
                const float x0 = bf16lo(u.x), x1 = bf16hi(u.x), x2 = bf16lo(u.y), x3 = bf16hi(u.y);
#pragma unroll
                for (int b = 0; b < NEH; ++b) {
                    acc[a][b] = fmaf(x0, wv[b].x, acc[a][b]);
                    acc[a][b] = fmaf(x1, wv[b].y, acc[a][b]);
                    acc[a][b] = fmaf(x2, wv[b].z, acc[a][b]);
                    acc[a][b] = fmaf(x3, wv[b].w, acc[a][b]);
                }
            }
        }
    }
    cp_async_wait<0>();
    __syncthreads();
    // logits -> shared tile [32][E] (+ global when requested)
    float* lt = wbuf;
#pragma unroll
    for (int b = 0; b < NEH; ++b) {
        const int e = ebase + lane + 32 * b;
        if (e >= E) continue;
        const float bb = bias ? bias[e] : 0.f;
#pragma unroll
        for (int a = 0; a < 8; ++a) {
            const int t = tg * 8 + a;
            const float l = acc[a][b] + bb;
            lt[t * E + e] = l;
            if (logits && t0 + t < T) logits[size_t(t0 + t) * E + e] = l;
        }
    }
    __syncthreads();
    for (int a = 0; a < 4; ++a) {     // warp w ranks tokens 4w .. 4w+3
        const int tl = warp * 4 + a;
        const int t = t0 + tl;
        if (t >= T) break;
        warp_topk_row(lt + tl * E, E, k, topk_idx + size_t(t) * k, topk_w + size_t(t) * k, nullptr);
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
    const int grid = (T + kRtTok - 1) / kRtTok;
    const int ne = (E + 31) / 32;
#define FT_RT(NEV)                                                                                          \
    do {                                                                                                    \
        const size_t smem = sizeof(float) * kRtStages * 32 * NEV * kRtLdW + sizeof(uint16_t) * kRtStages * kRtTok * kRtLdX; \
        static bool set = false;                                                                            \
        if (!set) {                                                                                         \
            cudaError_t e = cudaFuncSetAttribute(route_tile_kernel<NEV>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)); \
            if (e != cudaSuccess) return e;                                                                 \
            set = true;                                                                                     \
        }                                                                                                   \
        route_tile_kernel<NEV><<<grid, 256, smem, st>>>(T, H, E, k, x, wr, bias, topk_idx, topk_w, logits); \
    } while (0)
    if (ne <= 1) FT_RT(1);
    else if (ne <= 2) FT_RT(2);
    else if (ne <= 4) FT_RT(4);
    else FT_RT(8);
#undef FT_RT
    return cudaGetLastError();
}

}  // namespace ftmoe

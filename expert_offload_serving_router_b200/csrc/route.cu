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

// Order-preserving 32-bit key of an fp32 logit (larger logit -> larger key); -0 is folded
// onto +0 first so that they compare equal, as floats do.
__device__ __forceinline__ uint32_t logit_key(float v) {
    uint32_t u = __float_as_uint(v);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Warp-wide top-k over the E logits of one token held in `row` (shared memory).
// Lane l owns experts l, l+32, ...; each round: the lane's best (largest key, lowest index)
// candidate, a warp max of the key and a warp min of the index among the lanes holding that
// key (two redux.sync).  Ties therefore resolve to the lower expert index.
__device__ inline void warp_topk_row(const float* row, int E, int k, int32_t* idx_out, float* w_out,
                                     int32_t* idx_smem) {
    const int lane = threadIdx.x & 31;
    constexpr int NV = kMaxExperts / 32;
    uint32_t key[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int e = lane + 32 * i;
        key[i] = e < E ? logit_key(row[e]) : 0u;   // key 0 sorts below every finite logit
    }
    uint32_t taken = 0;
    float sel_v[kMaxTopK];
    int sel_e[kMaxTopK];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
        if (j >= k) break;
        uint32_t bk = 0u;
        int bi = 0;
        bool have = false;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const bool ok = (lane + 32 * i) < E && !((taken >> i) & 1u);
            if (ok && (!have || key[i] > bk)) { bk = key[i]; bi = i; have = true; }
        }
        const uint32_t kmax = __reduce_max_sync(0xffffffffu, have ? bk : 0u);
        const uint32_t cand = (have && bk == kmax) ? uint32_t(lane + 32 * bi) : 0xffffffffu;
        const uint32_t e = __reduce_min_sync(0xffffffffu, cand);
        if (int(e & 31) == lane) taken |= 1u << (e >> 5);
        sel_e[j] = int(e);
        sel_v[j] = row[e];
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
constexpr int kRtLdX = kRtBK + 4;   // floats per staged token row (fp32, converted once per slice)

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
    float* xbuf = wbuf + kRtStages * kRows * kRtLdW;                                  // [2][32][kRtLdX] fp32
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tg = warp & 3, eh = warp >> 2;
    const int ebase = eh * 32 * NEH;
    const int t0 = blockIdx.x * kRtTok;
    const int nk = H / kRtBK;

    auto stage = [&](int s, int k0) {        // router rows of one K slice: cp.async
        float* wd = wbuf + s * kRows * kRtLdW;
        for (int f = tid; f < E * 8; f += 256) {
            const int e = f >> 3, q = f & 7;
            cp_async16(wd + e * kRtLdW + q * 4, wr + size_t(e) * H + k0 + q * 4, 16);
        }
        cp_async_commit();
    };
    // token rows of one K slice go through registers and are stored as fp32, so the inner
    // loop does no bf16 unpacking: thread tid < 128 owns token tid/4, 8 values at (tid%4)*8
    const int xt = tid >> 2, xq = tid & 3;
    uint4 xr = make_uint4(0, 0, 0, 0);
    auto xload = [&](int k0) {
        xr = make_uint4(0, 0, 0, 0);
        if (tid < 128 && t0 + xt < T) xr = __ldg(reinterpret_cast<const uint4*>(x + size_t(t0 + xt) * H + k0 + xq * 8));
    };
    auto xstore = [&](int b) {
        if (tid < 128) {
            float* d = xbuf + (b * kRtTok + xt) * kRtLdX + xq * 8;
            *reinterpret_cast<float4*>(d) = make_float4(bf16lo(xr.x), bf16hi(xr.x), bf16lo(xr.y), bf16hi(xr.y));
            *reinterpret_cast<float4*>(d + 4) = make_float4(bf16lo(xr.z), bf16hi(xr.z), bf16lo(xr.w), bf16hi(xr.w));
        }
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
    xload(0);
    xstore(0);
    if (nk > 1) xload(kRtBK);
    for (int kb = 0; kb < nk; ++kb) {
        cp_async_wait<kRtStages - 2>();     // slice kb has landed (this thread's copies)
        __syncthreads();                    // ... and everyone's; slice kb-1 is no longer read
        const int nxt = kb + kRtStages - 1;
        if (nxt < nk) stage(nxt % kRtStages, nxt * kRtBK);
        else cp_async_commit();
        if (kb + 1 < nk) xstore((kb + 1) & 1);   // buffer of slice kb-1, free after the barrier
        if (kb + 2 < nk) xload((kb + 2) * kRtBK);
        const float* wsm = wbuf + (kb % kRtStages) * kRows * kRtLdW;
        const float* xsm = xbuf + (kb & 1) * kRtTok * kRtLdX;
#pragma unroll
        for (int kk = 0; kk < kRtBK; kk += 4) {
            float4 wv[NEH];
#pragma unroll
            for (int b = 0; b < NEH; ++b)
                wv[b] = *reinterpret_cast<const float4*>(wsm + (ebase + lane + 32 * b) * kRtLdW + kk);
#pragma unroll
            for (int a = 0; a < 8; ++a) {
                const float4 xv = *reinterpret_cast<const float4*>(xsm + (tg * 8 + a) * kRtLdX + kk);
                const float x0 = xv.x, x1 = xv.y, x2 = xv.z, x3 = xv.w;
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
    // the expert kernels that follow are launched as programmatic dependents: let them be
    // scheduled (and stage their token rows) while this grid runs
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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
    __shared__ int cnt[kMaxExperts + 2];
    if (warp == 0) warp_permute_small(sidx, a.T, a.k, a.E, a.S, cnt, a.perm);
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
        const size_t smem = sizeof(float) * (kRtStages * 32 * NEV * kRtLdW + 2 * kRtTok * kRtLdX);             \
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

// Step 1 for prefill batches -- the router GEMM on the tensor cores, with fp32-exact weights.
//
// The router weights are fp32 and the tokens bf16.  Every fp32 weight w splits exactly into
// three bf16 pieces w = hi + mid + lo (hi = bf16(w), mid = bf16(w - hi), lo = w - hi - mid:
// each difference is exact in fp32, and after two 8-bit pieces at most 8 significant bits
// are left, which bf16 holds).  A bf16 token value times a bf16 piece is exact in fp32, so
// l = sum_h x_h hi_h + sum_h x_h mid_h + sum_h x_h lo_h is the fp32 dot product with all
// products exact and only the accumulation rounded -- the same class of result as an
// fp32 FMA loop, with the same error bound (H + 1 roundings of partial sums at most).
//
//   split_router_kernel  fp32 W_r[E, H] -> planes[3][E16, H] bf16 (rows >= E are zero)
//   route_tc_kernel      one CTA per 128 tokens: D[128 tokens, E16] accumulated in TMEM by
//                        tcgen05.mma over K = H (3 MMAs per 16-wide K step, one per
//                        plane); while the grid is under one wave the K range is split
//                        across CTAs and the last CTA of a token tile (per-tile ticket)
//                        adds the partial sums in split order.  The logits + bias are
//                        staged in shared memory; then eight lanes per token store the
//                        row and keep the top k (logit descending, lower index first on
//                        ties; gates = softmax over the kept logits).
//
// Warp roles: warp 0 TMA producer (token tile + the three weight planes per K stage),
// warp 1 TMEM allocator + single-thread MMA issuer, warps 2-5 epilogue (warp w reads TMEM
// lanes 32(w%4) .. +31); all six warps run the per-token top-k.  All waits are bounded; on timeout the kernel raises the device
// error flag, drains its copies and MMAs, frees TMEM and returns.
#include "sm100.cuh"
#include "topk.cuh"

namespace ftmoe {

constexpr int kRcTok = kRouteTok;               // tokens per CTA (MMA M)
constexpr int kRcBK = 64;                       // K per stage
constexpr int kRcABytes = kRcTok * kRcBK * 2;   // 16 KB token tile
constexpr int kRcMaxStages = 4;
constexpr int kRcSmemCap = 227 * 1024;

__global__ void split_router_kernel(const float* __restrict__ wr, int E, int E16, int H, uint16_t* __restrict__ planes) {
    const size_t per_plane = size_t(E16) * H;
    const size_t n4 = per_plane / 4;
    for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += size_t(gridDim.x) * blockDim.x) {
        const size_t e = (i * 4) / size_t(H);
        float w[4] = {0.f, 0.f, 0.f, 0.f};
        if (e < size_t(E)) {
            const uint4 u = ldg_nc_v4(wr + i * 4);
            w[0] = __uint_as_float(u.x); w[1] = __uint_as_float(u.y);
            w[2] = __uint_as_float(u.z); w[3] = __uint_as_float(u.w);
        }
        uint16_t hi[4], mid[4], lo[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const __nv_bfloat16 h = __float2bfloat16_rn(w[j]);
            const float r1 = w[j] - __bfloat162float(h);
            const __nv_bfloat16 m = __float2bfloat16_rn(r1);
            const float r2 = r1 - __bfloat162float(m);
            const __nv_bfloat16 l = __float2bfloat16_rn(r2);
            hi[j] = __bfloat16_as_ushort(h);
            mid[j] = __bfloat16_as_ushort(m);
            lo[j] = __bfloat16_as_ushort(l);
        }
        uint2* p0 = reinterpret_cast<uint2*>(planes + i * 4);
        uint2* p1 = reinterpret_cast<uint2*>(planes + per_plane + i * 4);
        uint2* p2 = reinterpret_cast<uint2*>(planes + 2 * per_plane + i * 4);
        *p0 = make_uint2(hi[0] | (uint32_t(hi[1]) << 16), hi[2] | (uint32_t(hi[3]) << 16));
        *p1 = make_uint2(mid[0] | (uint32_t(mid[1]) << 16), mid[2] | (uint32_t(mid[3]) << 16));
        *p2 = make_uint2(lo[0] | (uint32_t(lo[1]) << 16), lo[2] | (uint32_t(lo[3]) << 16));
    }
}

struct RcParams {
    int T, Tpad, H, NP, stages, tmem_cols, KS;
    float* part;     // [KS][Tpad][NP] partial logits, one slab per K split
    uint32_t* err;
};

__global__ void __launch_bounds__(192, 1)
route_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w, RcParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int S = p.stages;
    const int bbytes = 3 * p.NP * kRcBK * 2;
    const int stage_bytes = kRcABytes + bbytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * stage_bytes);
    uint64_t* empty = full + kRcMaxStages;
    uint64_t* done = empty + kRcMaxStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    // the top-k kernel that follows is a programmatic dependent: let it be scheduled now
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tile0 = blockIdx.x * kRcTok;
    const int split = blockIdx.y;
    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(tmem_slot)),
                     "r"(p.tmem_cols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int nkt = p.H / kRcBK;                       // K stages of the whole contraction
    const int kb0 = split * nkt / p.KS, kb1 = (split + 1) * nkt / p.KS;
    const int nk = kb1 - kb0;                           // this CTA's stages

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int issued[kRcMaxStages];
            uint32_t issued_par[kRcMaxStages];
            for (int s = 0; s < kRcMaxStages; ++s) issued[s] = 0;
            bool ok = true;
            for (int kb = 0; kb < nk; ++kb) {
                if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
                uint8_t* a = smem + stage * stage_bytes;
                mbar_expect_tx(&full[stage], uint32_t(stage_bytes));
                tma_2d(&tm_x, &full[stage], a, (kb0 + kb) * kRcBK, tile0);
                tma_3d(&tm_w, &full[stage], a + kRcABytes, (kb0 + kb) * kRcBK, 0, 0);
                issued[stage] = 1;
                issued_par[stage] = phase;
                if (++stage == S) { stage = 0; phase ^= 1; }
            }
            if (!ok) { *abort_flag = 1; atomicExch(p.err, kDevErrTimeout); }
            for (int s = 0; s < S; ++s)
                if (issued[s]) mbar_wait(&full[s], issued_par[s], nullptr);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            const uint32_t idesc = idesc_bf16(kRcTok, p.NP);
            const int pbytes = p.NP * kRcBK * 2;
            for (int kb = 0; kb < nk; ++kb) {
                if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint8_t* a = smem + stage * stage_bytes;
                const uint64_t ad = sdesc_sw128(su32(a));
#pragma unroll
                for (int kk = 0; kk < kRcBK / 16; ++kk) {
#pragma unroll
                    for (int pl = 0; pl < 3; ++pl) {
                        const uint64_t bd = sdesc_sw128(su32(a + kRcABytes + pl * pbytes));
                        umma_bf16(tmem_base, ad + uint64_t(kk * 2), bd + uint64_t(kk * 2), idesc, (kb | kk | pl) != 0);
                    }
                }
                umma_commit(&empty[stage]);
                if (++stage == S) { stage = 0; phase ^= 1; }
            }
            if (!ok) { *abort_flag = 1; atomicExch(p.err, kDevErrTimeout); }
            umma_commit(done);   // arrives once every MMA issued above has completed
            mbar_wait(done, 0, nullptr);   // no MMA may still run when TMEM is freed
        }
    } else {
        // ------------------------------------------------ epilogue: one thread per token row,
        // TMEM -> this split's partial logits row (fp32, no bias), full 32-byte sectors
        const int q = warp & 3;
        const int r = 32 * q + lane;
        const int nch = (p.NP + 31) >> 5;
        const bool ok = mbar_wait(done, 0, abort_flag);
        if (!ok) {
            *abort_flag = 1;
            if (lane == 0) atomicExch(p.err, kDevErrTimeout);
        }
        if (ok && !*abort_flag) {
            tc_fence_after();
            float* dst = p.part + (size_t(split) * p.Tpad + tile0 + r) * p.NP;
            for (int c = 0; c < nch; ++c) {
                float v[32], dummy[32];
                tmem_ld32_nowait(tmem_base + (uint32_t(32 * q) << 16) + uint32_t(32 * c), v);
#pragma unroll
                for (int i = 0; i < 32; ++i) dummy[i] = 0.f;
                tmem_wait_ld(v, dummy);
                const int ncol = p.NP - 32 * c < 32 ? p.NP - 32 * c : 32;   // 16 or 32
#pragma unroll
                for (int i = 0; i < 32; i += 4)
                    if (i < ncol) *reinterpret_cast<float4*>(dst + 32 * c + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(p.tmem_cols));
    }
}

// Per token: l_e = (sum over splits in order of the partial dots) + b_e, stored as the logits
// row, and the top k of l.  16 lanes per token (lane g takes experts g, g+16, ...), lists
// merged by a 4-step butterfly: many short latency chains, which is what a full grid of
// small CTAs hides best.
constexpr int kTkLanes = 16;
constexpr int kTkThreads = 256;

__global__ void __launch_bounds__(kTkThreads)
route_topk_kernel(int T, int Tpad, int E, int NP, int k, int KS, const float* __restrict__ part,
                  const float* __restrict__ bias, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                  float* __restrict__ logits) {
    asm volatile("griddepcontrol.wait;" ::: "memory");   // partial logits of the router GEMM
    const int g = threadIdx.x % kTkLanes;
    const int t = blockIdx.x * (kTkThreads / kTkLanes) + threadIdx.x / kTkLanes;
    const bool live = t < T;
    const int tt = live ? t : T - 1;
    const float* row = part + size_t(tt) * NP;
    const size_t slab = size_t(Tpad) * NP;
    // all of this lane's partial values of one split are loaded before any is added, so a
    // lane waits for KS round trips, not KS x E/16
    constexpr int kPer = kMaxExperts / kTkLanes;
    float l[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) l[i] = 0.f;
    for (int sp = 0; sp < KS; ++sp) {
        float v[kPer];
#pragma unroll
        for (int i = 0; i < kPer; ++i) v[i] = g + kTkLanes * i < E ? __ldcg(row + sp * slab + g + kTkLanes * i) : 0.f;
#pragma unroll
        for (int i = 0; i < kPer; ++i) l[i] = sp == 0 ? v[i] : l[i] + v[i];
    }
    Top8 tk;
    tk.init();
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int e = g + kTkLanes * i;
        if (e < E) {
            const float le = bias ? l[i] + bias[e] : l[i];
            if (live && logits) logits[size_t(t) * E + e] = le;
            tk.offer(logit_key(le), e);
        }
    }
    group_merge_top8(tk, kTkLanes);
    if (live && g < k) {
        int32_t ee;
        float ww;
        top_slot(tk, k, g, &ee, &ww);
        topk_idx[size_t(t) * k + g] = ee;
        topk_w[size_t(t) * k + g] = ww;
    }
}

static size_t rc_smem(int stages, int NP) {
    return 1024 + size_t(stages) * (kRcABytes + 3 * NP * kRcBK * 2) + 2 * kRcMaxStages * 8 + 8 + 16;
}

cudaError_t launch_route_tc(int T, int H, int E, int k, const uint16_t* x, const float* wr, const float* bias,
                            int32_t* topk_idx, float* topk_w, float* logits, uint16_t* planes, float* part,
                            uint32_t* err, cudaStream_t st) {
    const int NP = (E + 15) & ~15;
    const int grid_split = num_sms() * 4;
    const size_t n4 = size_t(NP) * H / 4;
    int gs = int((n4 + 255) / 256);
    if (gs > grid_split) gs = grid_split;
    split_router_kernel<<<gs, 256, 0, st>>>(wr, E, NP, H, planes);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    CUtensorMap tx{}, tw{};
    {
        uint64_t dims[2] = {uint64_t(H), uint64_t(T)};
        uint64_t str[1] = {uint64_t(H) * 2};
        uint32_t box[2] = {kRcBK, kRcTok};
        if (!make_map(&tx, x, 2, dims, str, box)) return cudaErrorInvalidValue;
    }
    {
        uint64_t dims[3] = {uint64_t(H), uint64_t(NP), 3};
        uint64_t str[2] = {uint64_t(H) * 2, uint64_t(H) * NP * 2};
        uint32_t box[3] = {kRcBK, uint32_t(NP), 3};
        if (!make_map(&tw, planes, 3, dims, str, box)) return cudaErrorInvalidValue;
    }
    int stages = kRcMaxStages;
    while (stages > 1 && rc_smem(stages, NP) > size_t(kRcSmemCap)) --stages;
    const size_t smem = rc_smem(stages, NP);
    if (smem > size_t(kRcSmemCap)) return cudaErrorInvalidConfiguration;
    static PerDeviceOnce attr;
    e = attr([&] { return cudaFuncSetAttribute(route_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kRcSmemCap); });
    if (e != cudaSuccess) return e;
    const int tiles = (T + kRcTok - 1) / kRcTok;
    RcParams p{};
    p.T = T; p.Tpad = tiles * kRcTok; p.H = H; p.NP = NP; p.stages = stages;
    p.tmem_cols = NP <= 32 ? 32 : NP <= 64 ? 64 : NP <= 128 ? 128 : 256;
    p.part = part; p.err = err;
    p.KS = route_splits(T, H);
    route_tc_kernel<<<dim3(tiles, p.KS), 192, smem, st>>>(tx, tw, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((T + kTkThreads / kTkLanes - 1) / (kTkThreads / kTkLanes));
    cfg.blockDim = dim3(kTkThreads);
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, route_topk_kernel, T, p.Tpad, E, NP, k, p.KS, static_cast<const float*>(part), bias,
                              topk_idx, topk_w, logits);
}

}  // namespace ftmoe

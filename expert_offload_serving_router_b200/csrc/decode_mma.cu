// Steps 3/4 (decode, BF16 weights) on the tensor cores.  A decode batch (T <= 32 tokens) is a
// stream over the routed experts' weights; with several tokens per expert the SIMT GEMV spends
// as long on its FMAs and shared-memory reads of x as on the stream.  Here every MMA has the
// weights as A (M = 128 rows, TMA-fed through a three-stage ring) and the tokens as B (N =
// T rounded up to 16), so the arithmetic is the tensor cores' and each CTA is a weight stream.
//
// One persistent launch does both projections.  Its items are all gate/up items, then all down
// items:
//   gate/up: (active group, 128 interleaved gate/up rows = 64 f).  B = x itself ([T, H], every
//       token): the MMA computes all T columns and the epilogue keeps the columns of the group's
//       tokens, h[row, f] = silu(gate) * up -> bf16.  No gather of x, no x_sorted.  Each epilogue
//       warp then raises the group's readiness counter (after a fence).
//   down:    (active group, 128 hidden rows).  B = the group's contiguous h rows
//       [offsets[g], offsets[g+1]) (rows past the group belong to other groups and are
//       ignored), o[row, hidden] -> bf16.  Its producer waits (bounded) until every gate/up
//       item of the group has raised the counter before it loads h; the weights need no wait.
//       The last down item of a group to pass that wait returns the group's counters to zero.
// So a group's down items start as soon as its own h is written, while other groups' gate/up
// items are still streaming, and there is no second launch.  The gate-weighted combine back to
// token order follows as its own small kernel (programmatic dependent launch).
// Persistent CTAs (three per SM, never more than fit at once, so every gate/up item a down
// item waits for is running or done) walk the items with one TMA ring; accumulators are double
// buffered.  Warp roles: 0 TMA producer, 1 TMEM allocation + MMA issuer, 2-5 epilogue (TMEM lane
// quarter warp & 3).  Every wait is bounded (the grouped GEMMs' limit).
#include "gemm_common.cuh"
#include "decode_common.cuh"

namespace ftmoe {

constexpr int kDmSt = 3;                           // stages of one 64-deep K step (three CTAs per SM)
constexpr int kDmATile = 128 * kBK * 2;            // 16 KB
constexpr int kDmBTile = 32 * kBK * 2;             // 4 KB: up to 32 token rows
constexpr int kDmThreads = 192;

struct DecMmaParams {
    int T, k, E, S, H, F, G, NB;      // NB = MMA N (T rounded up to 16)
    int gu_blocks;                     // 128-row gate/up blocks per expert (F / 64)
    int dn_blocks;                     // 128-row down blocks per expert (H / 128)
    const int32_t* offsets;
    const int32_t* sorted_flat;
    const int32_t* sched;              // [1] n_active, active groups at [2 + G + 1 ...]
    uint16_t* h;                       // [R, F]
    uint16_t* o;                       // [R, H]
    uint32_t* ready;                   // [G] gate/up epilogue warps done per group, [G .. 2G) down items past the wait
    uint32_t* err;
    unsigned long long wait_ns;
};

__host__ __device__ constexpr size_t dec_mma_smem() {
    return 1024 + size_t(kDmSt) * (kDmATile + kDmBTile) + 512;
}

// token of the group's i-th row
__device__ __forceinline__ int group_token(const DecMmaParams& p, int g, int i) {
    const int P = p.T * p.k;
    const int fl = p.sorted_flat[p.offsets[g] + i];
    return fl < P ? fl / p.k : fl - P;
}

struct DmItem { int g, e, rg, r0, n; bool shared, down; };
__device__ __forceinline__ DmItem dm_item(const DecMmaParams& p, int it, int n_gu) {
    DmItem d;
    d.down = it >= n_gu;
    const int blocks = d.down ? p.dn_blocks : p.gu_blocks;
    const int j = d.down ? it - n_gu : it;
    const int slot = j / blocks;
    d.rg = j - slot * blocks;
    d.g = p.sched[2 + (p.G + 1) + slot];
    d.r0 = p.offsets[d.g];
    d.n = p.offsets[d.g + 1] - d.r0;
    d.shared = d.g >= p.E;
    d.e = d.shared ? 0 : d.g;
    return d;
}

// Persistent: CTA b takes items b, b + gridDim.x, ... (gate/up items first); one TMA ring runs
// across items and the accumulators are double buffered (2 x 32 TMEM columns), so an item's
// epilogue overlaps the next item's weight stream.
__global__ void __launch_bounds__(kDmThreads, 3)
decode_mma_kernel(const __grid_constant__ CUtensorMap tm_w13, const __grid_constant__ CUtensorMap tm_sw13,
                  const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w2,
                  const __grid_constant__ CUtensorMap tm_sw2, const __grid_constant__ CUtensorMap tm_h,
                  DecMmaParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = sA + kDmSt * kDmATile;
    uint64_t* full = reinterpret_cast<uint64_t*>(sB + kDmSt * kDmBTile);
    uint64_t* empty = full + kDmSt;
    uint64_t* tfull = empty + kDmSt;
    uint64_t* tempty = tfull + 2;
    uint64_t* mma_done = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    pdl_wait();          // routing (offsets, schedule) comes from the preceding kernels
    pdl_trigger();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_active = p.sched[1];
    const int n_gu = n_active * p.gu_blocks;
    const int n_items = n_gu + n_active * p.dn_blocks;
    if (int(blockIdx.x) >= n_items) return;            // uniform across the CTA
    const int nk_gu = p.H / kBK, nk_dn = p.F / kBK;
    if (tid == 0) {
        for (int s = 0; s < kDmSt; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        for (int b = 0; b < 2; ++b) { mbar_init(&tfull[b], 1); mbar_init(&tempty[b], 4); }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(tmem_slot)), "r"(64));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint32_t bbytes = uint32_t(p.NB) * kBK * 2;
            const uint32_t h_target = 4u * uint32_t(p.gu_blocks);     // four epilogue warps per gate/up item
            int step = 0;
            bool ok = true;
            for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
                const DmItem d = dm_item(p, it, n_gu);
                if (d.down) {
                    // the group's h rows must all be written before the first B load
                    const unsigned long long t0 = gtimer();
                    while (ld_acquire_u32(p.ready + d.g) < h_target) {
                        if (*abort_flag || gtimer() - t0 > p.wait_ns) { ok = false; break; }
                        __nanosleep(64);
                    }
                    if (!ok) break;
                    asm volatile("fence.proxy.async.global;" ::: "memory");   // h (generic writes) -> TMA reads
                    // the last down item of the group past this point leaves both counters at zero
                    if (atomicAdd(p.ready + p.G + d.g, 1u) == uint32_t(p.dn_blocks - 1)) {
                        p.ready[d.g] = 0u;
                        p.ready[p.G + d.g] = 0u;
                    }
                }
                const int nk = d.down ? nk_dn : nk_gu;
                for (int kb = 0; kb < nk; ++kb, ++step) {
                    const int s = step % kDmSt;
                    if (!mbar_wait(&empty[s], (uint32_t(step / kDmSt) & 1u) ^ 1u, abort_flag, p.wait_ns)) { ok = false; break; }
                    mbar_expect_tx(&full[s], uint32_t(kDmATile) + bbytes);
                    if (!d.down) {
                        tma_5d(d.shared ? &tm_sw13 : &tm_w13, &full[s], sA + s * kDmATile, kb * kBK, 0, 0, d.rg * 4, d.e);
                        tma_2d(&tm_x, &full[s], sB + s * kDmBTile, kb * kBK, 0);
                    } else {
                        tma_3d(d.shared ? &tm_sw2 : &tm_w2, &full[s], sA + s * kDmATile, kb * kBK, d.rg * 128, d.e);
                        tma_2d(&tm_h, &full[s], sB + s * kDmBTile, kb * kBK, d.r0);
                    }
                }
            }
            if (!ok) { *abort_flag = 1; atomicExch(p.err, kDevErrTimeout); }
            for (int st = step - kDmSt > 0 ? step - kDmSt : 0; st < step; ++st)   // drain
                mbar_wait(&full[st % kDmSt], uint32_t(st / kDmSt) & 1u, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, p.NB);
            int step = 0, buf = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
                const int nk = it >= n_gu ? nk_dn : nk_gu;
                if (!mbar_wait(&tempty[buf], acc_phase ^ 1u, abort_flag, p.wait_ns)) { ok = false; break; }
                tc_fence_after();
                for (int kb = 0; kb < nk; ++kb, ++step) {
                    const int s = step % kDmSt;
                    if (!mbar_wait(&full[s], uint32_t(step / kDmSt) & 1u, abort_flag, p.wait_ns)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t ad = sdesc_sw128(su32(sA + s * kDmATile));
                    const uint64_t bd = sdesc_sw128(su32(sB + s * kDmBTile));
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        umma_bf16(tmem + uint32_t(32 * buf), ad + uint64_t(kk * 2), bd + uint64_t(kk * 2), idesc,
                                  (kb | kk) != 0);
                    umma_commit(&empty[s]);
                }
                if (!ok) break;
                umma_commit(&tfull[buf]);
                if (++buf == 2) { buf = 0; acc_phase ^= 1; }
            }
            if (!ok) { *abort_flag = 1; atomicExch(p.err, kDevErrTimeout); }
            umma_commit(mma_done);                 // completion of every MMA issued above
            mbar_wait(mma_done, 0, nullptr);       // none may still run when TMEM is freed
        }
    } else {
        // ------------------------------------------------ epilogue: TMEM lanes 32q.., one column per routed row
        const int q = warp & 3;
        int buf = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
            const DmItem d = dm_item(p, it, n_gu);
            // lane l < n stands for row r0 + l of the group; gate/up: its token
            const int my_tok = (!d.down && lane < d.n) ? group_token(p, d.g, lane) : -1;
            if (!mbar_wait(&tfull[buf], acc_phase, abort_flag, p.wait_ns)) { ok = false; break; }
            tc_fence_after();
            float v[32];
            tmem_ld32_nowait(tmem + (uint32_t(q * 32) << 16) + uint32_t(32 * buf), v);
            tmem_wait_16(v);
            tmem_fence_regs(v + 16);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[buf]);          // the accumulator is free for the item after next
            if (!d.down) {
                // rows 32q..32q+15: gate of f = 64 rg + 16 q + (lane & 15); rows +16: up of the same f
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    if (c >= p.NB) break;
                    const unsigned hit = __ballot_sync(0xffffffffu, my_tok == c);
                    if (!hit) continue;                                  // token c is not routed here
                    const int r = d.r0 + __ffs(hit) - 1;
                    const float other = __shfl_xor_sync(0xffffffffu, v[c], 16);
                    const float hv = silu_mul(lane < 16 ? v[c] : other, lane < 16 ? other : v[c]);
                    const uint32_t b = f2bf(hv);
                    const uint32_t pair = b | (__shfl_down_sync(0xffffffffu, b, 1) << 16);
                    if (lane < 16 && !(lane & 1))
                        *reinterpret_cast<uint32_t*>(p.h + size_t(r) * p.F + 64 * d.rg + 16 * q + lane) = pair;
                }
                // these h columns are written: one count towards the group's down items
                __threadfence();
                __syncwarp();
                if (lane == 0) atomicAdd(p.ready + d.g, 1u);
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (i < d.n) p.o[size_t(d.r0 + i) * p.H + 128 * d.rg + 32 * q + lane] = f2bf(v[i]);
            }
            if (++buf == 2) { buf = 0; acc_phase ^= 1; }
        }
        if (!ok) { *abort_flag = 1; if (lane == 0) atomicExch(p.err, kDevErrTimeout); }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(64));
    }
}

// ------------------------------------------------------------------ host side
bool decode_mma_eligible(const DecodeArgs& a) {
    return a.wdtype == FT_W_BF16 && !a.eptr && a.T >= 1 && a.T <= 32 && a.H % 128 == 0 && a.F % 64 == 0;
}

cudaError_t launch_decode_mma(const DecodeArgs& a, cudaStream_t st) {
    const int T = a.T, H = a.H, F = a.F, E = a.E, k = a.k, S = a.S;
    const int P = T * k, R = P + (S ? T : 0), G = E + (S ? 1 : 0);
    const int na_max = R < G ? R : G;
    const int NB = T <= 16 ? 16 : 32;
    DecMmaParams p{};
    p.T = T; p.k = k; p.E = E; p.S = S; p.H = H; p.F = F; p.G = G; p.NB = NB;
    p.gu_blocks = F / 64;
    p.dn_blocks = H / 128;
    p.offsets = a.offsets;
    p.sorted_flat = a.sorted_flat;
    p.sched = a.sched;
    p.h = a.h;
    p.o = a.y ? a.o_ws : a.o_sorted;
    p.ready = a.err + kWsReady;
    p.err = a.err;
    p.wait_ns = gemm_wait_ns();
    CUtensorMap gw{}, gsw{}, gb{}, dw{}, dsw{}, db{};
    {   // gate/up: w13 [E][2][F][H] as (H, 16, 2, F/16, E), one (64, 16, 2, 4, 1) box = 128 interleaved rows
        uint64_t str[4] = {uint64_t(H) * 2, uint64_t(F) * H * 2, uint64_t(16) * H * 2, uint64_t(2) * F * H * 2};
        uint32_t box[5] = {kBK, 16, 2, 4, 1};
        uint64_t dims[5] = {uint64_t(H), 16, 2, uint64_t(F / 16), uint64_t(E)};
        if (!make_map(&gw, a.w13, 5, dims, str, box)) return cudaErrorInvalidValue;
        dims[4] = 1;
        if (S && !make_map(&gsw, a.sw13, 5, dims, str, box)) return cudaErrorInvalidValue;
        uint64_t xd[2] = {uint64_t(H), uint64_t(T)}, xs[1] = {uint64_t(H) * 2};
        uint32_t xb[2] = {kBK, uint32_t(NB)};
        if (!make_map(&gb, a.x, 2, xd, xs, xb)) return cudaErrorInvalidValue;
    }
    {   // down: w2 [E][H][F] as (F, H, E), (64, 128, 1) boxes; B = h rows [R, F]
        uint64_t dims[3] = {uint64_t(F), uint64_t(H), uint64_t(E)};
        uint64_t str[2] = {uint64_t(F) * 2, uint64_t(H) * F * 2};
        uint32_t box[3] = {kBK, 128, 1};
        if (!make_map(&dw, a.w2, 3, dims, str, box)) return cudaErrorInvalidValue;
        dims[2] = 1;
        if (S && !make_map(&dsw, a.sw2, 3, dims, str, box)) return cudaErrorInvalidValue;
        uint64_t hd[2] = {uint64_t(F), uint64_t(R)}, hs[1] = {uint64_t(F) * 2};   // rows past R read as zero
        uint32_t hb[2] = {kBK, uint32_t(NB)};
        if (!make_map(&db, a.h, 2, hd, hs, hb)) return cudaErrorInvalidValue;
    }
    if (!S) { gsw = gw; dsw = dw; }
    constexpr size_t smem = dec_mma_smem();
    // Down items wait for gate/up items of other CTAs, so every CTA must be resident at once: the
    // grid is three per SM (what fits at this shared-memory size: 3 x 62 KB; all of them enter
    // within a few microseconds, measured) and never more than the items a batch can have.  Were
    // a CTA ever kept from running by other work, a waiting down item gives up after the bounded
    // wait and the call reports a timeout.
    static PerDeviceOnce attrs;
    {
        const cudaError_t e = attrs([&] {
            cudaError_t r = cudaFuncSetAttribute(decode_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
            if (r == cudaSuccess)   // the whole unified L1 / shared array as shared memory
                r = cudaFuncSetAttribute(decode_mma_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                         int(cudaSharedmemCarveoutMaxShared));
            return r;
        });
        if (e != cudaSuccess) return e;
    }
    const int cap = 3 * num_sms();
    const int max_items = na_max * (p.gu_blocks + p.dn_blocks);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(max_items < cap ? max_items : cap);
    cfg.blockDim = dim3(kDmThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, decode_mma_kernel, gw, gsw, gb, dw, dsw, db, p);
    if (e != cudaSuccess) return e;
    if (a.y) e = launch_combine_dependent(T, H, k, S, R, a.o_ws, a.inv_pos, a.topk_w, a.y, st);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace ftmoe

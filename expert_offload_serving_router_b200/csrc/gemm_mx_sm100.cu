// Step 3 (prefill) over MXFP4 expert weights -- grouped GEMMs on CTA pairs with the weights
// dequantised in the load path (the layer's E2M1 codes and E8M0 block scales never exist
// in bf16 outside shared memory).
//
//   gate/up:  D[256 weight rows, N tokens] = W13_e[rows, H] . Xs[tokens, H]^T, then
//             h[token, f] = silu(gate) * up, stored bf16 [R, F]
//   down:     D[256 hidden rows, N tokens] = W2_e[rows, F] . h[tokens, F]^T -> o_sorted [R, H]
//
// A cluster of two CTAs shares every MMA (tcgen05.mma.cta_group::2, M = 256): a pair tile
// is 512 weight rows (CTA r holds the 128-row groups 4m + r and 4m + 2 + r) x up to 256
// tokens of one expert group (CTA r holds token rows r*N/2 .. of the tile).  Per K step of
// 64 each CTA needs 256 weight rows of A (32 KB of bf16 built from 8 KB of codes) and at
// most 128 token rows of B (16 KB).
//
// The packed weights stream by TMA into their own ring: a code unit is 128 weight rows x
// 64 code bytes (two K steps, SW64 swizzle so that a warp's row-per-lane 16-byte reads
// hit every bank once) per 128-row group, and every fourth unit also brings the rows'
// next 16 scale bytes (eight K steps).  The ring is three units (six K steps) deep, so the
// global-memory latency of the weights is hidden behind the MMAs of the steps before.
// Two groups of four converter warps, taking alternate K steps, turn a K step of codes into
// the bf16 A operand in the 128-byte swizzle the MMA reads, and arrive on the leader's barrier
// after a proxy fence; while one group's step waits on its fence and cluster arrive, the other
// converts.  A word of eight codes becomes four bf16x2 words by bit placement (magnitude bits
// to bf16 bits 6..8 and the sign to bit 15 give the E2M1 value times 2^-126 exactly; one
// `mul.rn.bf16x2` by 2^(s-1) applies the E8M0 scale); blocks whose scale byte exceeds 128
// (2^(s-1) would not be a finite bf16) take byte-permute table lookups and a multiply by 2^(s-127).
// At the end of a tile the same warps run the epilogue (the tile's accumulators -> h with
// SwiGLU, or -> o_sorted): eight warps, two per TMEM lane quarter, so the kernel has ten warps
// and 168 registers per thread.
//
// Warp roles (both CTAs unless stated):
//   warp 0        lane 0: TMA producer of the token tile (completion counted on the leader's
//                 barrier); lane 1: TMA producer of the code units and scale groups (own CTA,
//                 own barriers)
//   warp 1        TMEM allocation (cta_group::2, 512 columns); in the leader, the
//                 single-thread MMA issuer
//   warps 2-9     two groups of four converter warps taking alternate K steps (thread r of a
//                 group builds row r of both 128-row groups of its steps); at a tile's end,
//                 its epilogue (TMEM lane quarter warp & 3, column chunks of the group's parity)
// Every wait is bounded: on timeout a role raises the CTA's abort flag, records
// kDevErrTimeout, drains the copies it issued, and every thread of both CTAs still reaches
// the teardown (MMAs complete, TMEM freed).
#include "gemm_common.cuh"

namespace ftmoe {

constexpr int kMxSt = 3;                               // A/B ring: one 64-deep K step per stage
constexpr int kMxATile = 2 * kAHalfBytes;              // 32 KB: two 128-row bf16 operands
constexpr int kMxBTile = 128 * kBK * 2;                // 16 KB: up to 128 token rows (this CTA's half)
constexpr int kMxUnitK = 2 * kBK;                      // K elements per code unit
constexpr int kMxUnitHalf = 128 * kMxUnitK / 2;        // 8 KB: 128 rows x 64 code bytes
constexpr int kMxUnitTile = 2 * kMxUnitHalf;           // 16 KB
constexpr int kMxCSt = 3;                              // code-unit ring depth
constexpr int kMxGroupK = 512;                         // K elements per scale group (16 bytes per row)
constexpr int kMxUnitsPerGroup = kMxGroupK / kMxUnitK; // 4
constexpr int kMxScaleHalf = 128 * 16;                 // 2 KB
constexpr int kMxScaleTile = 2 * kMxScaleHalf;         // 4 KB
constexpr int kMxConvWarps = 8;                        // two groups of four, alternating K steps
constexpr int kMxConvWarp0 = 2;
constexpr int kMxThreads = 32 * (kMxConvWarp0 + kMxConvWarps);   // 320: at most three warps per SM
                                                                  // sub-partition, 168 registers
constexpr int kMxXposeWarps = kMxConvWarps;

__host__ __device__ constexpr size_t mx_pair_smem_bytes() {
    return 1024 + size_t(kMxSt) * (kMxATile + kMxBTile) + size_t(kMxCSt) * kMxUnitTile + 2 * kMxScaleTile +
           kMxXposeWarps * kXposeBytes + 256 + 8 * 260;
}

__device__ __forceinline__ uint4 lds128(const uint8_t* p) {
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(su32(p)));
    return r;
}
__device__ __forceinline__ void sts128(uint8_t* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(su32(p)), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kMxThreads, 1)
moe_gemm_mx_pair_kernel(const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_s,
                        const __grid_constant__ CUtensorMap tm_sc, const __grid_constant__ CUtensorMap tm_ss,
                        const __grid_constant__ CUtensorMap tm_b0, const __grid_constant__ CUtensorMap tm_b1,
                        const __grid_constant__ CUtensorMap tm_b2, const __grid_constant__ CUtensorMap tm_b3,
                        const __grid_constant__ CUtensorMap tm_b4, GemmParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = sA + kMxSt * kMxATile;
    uint8_t* sC = sB + kMxSt * kMxBTile;
    uint8_t* sS = sC + kMxCSt * kMxUnitTile;
    uint8_t* sX = sS + 2 * kMxScaleTile;
    uint64_t* bfull = reinterpret_cast<uint64_t*>(sX + kMxXposeWarps * kXposeBytes);
    uint64_t* afull = bfull + kMxSt;
    uint64_t* empty = afull + kMxSt;
    uint64_t* cfull = empty + kMxSt;
    uint64_t* cempty = cfull + kMxCSt;
    uint64_t* tfull = cempty + kMxCSt;
    uint64_t* tempty = tfull + 1;
    uint64_t* mma_done = tempty + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* ntile_off = const_cast<int*>(reinterpret_cast<volatile int*>(tmem_slot + 2));
    int* s_off = ntile_off + 260;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank();
    const int cid = int(cluster_id_x()), ncl = int(cluster_count_x());
    const int G = p.G;
    for (int i = tid; i <= G; i += blockDim.x) {
        ntile_off[i] = p.sched[2 + i];
        s_off[i] = p.offsets[i];
    }
    if (tid == 0) {
        for (int s = 0; s < kMxSt; ++s) {
            mbar_init(&bfull[s], 1);                      // the leader's producer (both CTAs' bytes)
            mbar_init(&afull[s], kMxConvWarps);           // one converter group (4 warps) of each CTA
            mbar_init(&empty[s], 1);                      // the leader's MMA commit
        }
        for (int s = 0; s < kMxCSt; ++s) {
            mbar_init(&cfull[s], 1);                      // own code producer (+ TMA bytes)
            mbar_init(&cempty[s], kMxConvWarps);          // own converter warps
        }
        mbar_init(tfull, 1);
        mbar_init(tempty, 2 * kMxConvWarps);
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(tmem_slot)),
                     "r"(2 * kAccCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const uint32_t bfull_lead = mapa_rank(su32(bfull), 0);
    const uint32_t afull_lead = mapa_rank(su32(afull), 0);
    const uint32_t tempty_lead = mapa_rank(su32(tempty), 0);

    const int total = ntile_off[G] * p.m_tiles;
    const int nk = p.K / kBK;

    if (warp == 0) {
        // ------------------------------------------------ token-tile producer (both CTAs)
        if (lane == 0) {
            const CUtensorMap* bm[kNumBMaps] = {&tm_b0, &tm_b1, &tm_b2, &tm_b3, &tm_b4};
            int stage = 0;
            uint32_t phase = 0;
            int issued[kMxSt];
            uint32_t issued_par[kMxSt];
            for (int s = 0; s < kMxSt; ++s) issued[s] = 0;
            bool ok = true;
            for (int t = cid; t < total && ok; t += ncl) {
                const Tile tl = decode_tile<4>(t, ntile_off, G, s_off, p.m_tiles, p.m_rows);
                const int nh = ((tl.nvalid + 15) & ~15) >> 1;   // token rows per CTA
                int bi = 0;
                while (bi < kNumBMaps - 1 && (8 << bi) < nh) ++bi;
                const uint32_t bbytes = uint32_t(p.b_rows[bi]) * kBK * 2;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.wait_ns)) { ok = false; break; }
                    if (rank == 0) mbar_expect_tx(&bfull[stage], 2u * bbytes);
                    tma_2d_pair(bm[bi], bfull_lead + uint32_t(stage) * 8u, sB + stage * kMxBTile, kb * kBK,
                                tl.row0 + int(rank) * nh);
                    issued[stage] = 1;
                    issued_par[stage] = phase;
                    if (++stage == kMxSt) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok) { *abort_flag = 1; atomicExch(p.err, kDevErrTimeout); }
            // drain: the leader sees its full barriers complete (both CTAs' bytes landed); the
            // peer sees its empty barriers released (the leader consumed what it copied)
            for (int s = 0; s < kMxSt; ++s)
                if (issued[s]) {
                    if (rank == 0) mbar_wait(&bfull[s], issued_par[s], nullptr);
                    else mbar_wait(&empty[s], issued_par[s], nullptr);
                }
        } else if (lane == 1) {
            // -------------------------------------------- code-unit + scale-group producer (own CTA)
            int cst = 0, grp = 0;
            uint32_t cph = 0;
            int issued[kMxCSt];
            uint32_t issued_par[kMxCSt];
            for (int s = 0; s < kMxCSt; ++s) issued[s] = 0;
            const int nu = p.K / kMxUnitK;
            bool ok = true;
            for (int t = cid; t < total && ok; t += ncl) {
                const Tile tl = decode_tile<4>(t, ntile_off, G, s_off, p.m_tiles, p.m_rows);
                const bool shared_grp = p.has_shared && tl.g == p.E;
                const CUtensorMap* mc = shared_grp ? &tm_sc : &tm_c;
                const CUtensorMap* ms = shared_grp ? &tm_ss : &tm_s;
                const int e = shared_grp ? 0 : tl.g;
                for (int u = 0; u < nu; ++u) {
                    if (!mbar_wait(&cempty[cst], cph ^ 1, abort_flag, p.wait_ns)) { ok = false; break; }
                    const bool with_scales = (u % kMxUnitsPerGroup) == 0;
                    mbar_expect_tx(&cfull[cst], uint32_t(kMxUnitTile) + (with_scales ? uint32_t(kMxScaleTile) : 0u));
                    for (int hh = 0; hh < 2; ++hh) {
                        const int rg = tl.m * 4 + 2 * hh + int(rank);   // 128-row weight group
                        uint8_t* cdst = sC + cst * kMxUnitTile + hh * kMxUnitHalf;
                        uint8_t* sdst = sS + (grp & 1) * kMxScaleTile + hh * kMxScaleHalf;
                        const int kc = u * (kMxUnitK / 2), ksc = (u / kMxUnitsPerGroup) * 16;
                        if (p.mode == 0) {
                            tma_5d(mc, &cfull[cst], cdst, kc, 0, 0, rg * 4, e);
                            if (with_scales) tma_5d(ms, &cfull[cst], sdst, ksc, 0, 0, rg * 4, e);
                        } else {
                            tma_3d(mc, &cfull[cst], cdst, kc, rg * 128, e);
                            if (with_scales) tma_3d(ms, &cfull[cst], sdst, ksc, rg * 128, e);
                        }
                    }
                    issued[cst] = 1;
                    issued_par[cst] = cph;
                    if (u % kMxUnitsPerGroup == kMxUnitsPerGroup - 1) ++grp;
                    if (++cst == kMxCSt) { cst = 0; cph ^= 1; }
                }
            }
            if (!ok) { *abort_flag = 1; atomicExch(p.err, kDevErrTimeout); }
            for (int s = 0; s < kMxCSt; ++s)
                if (issued[s]) mbar_wait(&cfull[s], issued_par[s], nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (leader only)
        if (lane == 0) {
            if (rank == 0) {
                int stage = 0;
                uint32_t phase = 0, acc_phase = 0;
                bool ok = true;
                for (int t = cid; t < total && ok; t += ncl) {
                    const Tile tl = decode_tile<4>(t, ntile_off, G, s_off, p.m_tiles, p.m_rows);
                    const int N = (tl.nvalid + 15) & ~15;
                    const uint32_t idesc = idesc_bf16(256, N);
                    if (!mbar_wait_cluster(tempty, acc_phase ^ 1, abort_flag, p.wait_ns)) { ok = false; break; }
                    tc_fence_after();
                    for (int kb = 0; kb < nk; ++kb) {
                        if (!mbar_wait(&bfull[stage], phase, abort_flag, p.wait_ns)) { ok = false; break; }
                        if (!mbar_wait_cluster(&afull[stage], phase, abort_flag, p.wait_ns)) { ok = false; break; }
                        tc_fence_after();
                        const uint64_t bd = sdesc_sw128(su32(sB + stage * kMxBTile));
                        for (int h = 0; h < 2; ++h) {
                            const uint64_t ad = sdesc_sw128(su32(sA + stage * kMxATile + h * kAHalfBytes));
                            const uint32_t dtm = tmem_base + uint32_t(h * kAccCols);
#pragma unroll
                            for (int kk = 0; kk < kBK / 16; ++kk)
                                umma_bf16_pair(dtm, ad + uint64_t(kk * 2), bd + uint64_t(kk * 2), idesc, (kb | kk) != 0);
                        }
                        umma_commit_pair_both(&empty[stage]);
                        if (++stage == kMxSt) { stage = 0; phase ^= 1; }
                    }
                    if (!ok) break;
                    umma_commit_pair_both(tfull);
                    acc_phase ^= 1;
                }
                if (!ok) { *abort_flag = 1; atomicExch(p.err, kDevErrTimeout); }
                umma_commit_pair_both(mma_done);     // completion of every MMA issued above, in both CTAs
            }
            mbar_wait(mma_done, 0, nullptr);
        }
    } else {
        // ------------------------------------------------ converters: codes (smem) -> bf16 A (smem)
        // Two groups of four warps take alternate K steps (group gi the steps n = gi mod 2 of
        // the CTA's running step count n, i.e. half gi of every code unit), so the latency of
        // one step's conversion, proxy fence and cluster arrive overlaps the other group's
        // step.  Thread `row` of a group builds that row of both 128-row groups of the stage.
        const int gi = (warp - kMxConvWarp0) >> 2;
        const int row = tid - 32 * kMxConvWarp0 - 128 * gi;   // 0..127
        const int xsw = (row >> 1) & 3;                       // SW64 chunk permutation of this code row
        uint4 sreg[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
        bool ok = true;
        int n = gi;                                           // this CTA's running K-step index
        uint32_t acc_phase = 0;
        for (int t = cid; t < total && ok; t += ncl) {
            for (int kb = gi; kb < nk; kb += 2, n += 2) {
                const int u = n >> 1;                         // code unit; its half j = gi
                const int cst = u % kMxCSt;
                const uint32_t cph = uint32_t(u / kMxCSt) & 1u;
                const int stage = n % kMxSt;
                const uint32_t phase = uint32_t(n / kMxSt) & 1u;
                if (!mbar_wait(&cfull[cst], cph, abort_flag, p.wait_ns)) { ok = false; break; }
                if ((kb & 7) < 2)                             // first step of a scale group this group sees
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        sreg[h] = lds128(sS + ((n >> 3) & 1) * kMxScaleTile + h * kMxScaleHalf + row * 16);
                uint4 c0[2], c1[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint8_t* crow = sC + cst * kMxUnitTile + h * kMxUnitHalf + row * 64;
                    c0[h] = lds128(crow + (((2 * gi) ^ xsw) << 4));
                    c1[h] = lds128(crow + (((2 * gi + 1) ^ xsw) << 4));
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&cempty[cst]);
                if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.wait_ns)) { ok = false; break; }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint4 sv = sreg[h];
                    const uint32_t sw = (kb & 4) ? ((kb & 2) ? sv.w : sv.z) : ((kb & 2) ? sv.y : sv.x);
                    const uint32_t sp = sw >> (16 * (kb & 1));
                    const uint32_t b0 = sp & 0xFF, b1 = (sp >> 8) & 0xFF;
                    const bool place = b0 <= 128u && b1 <= 128u;   // 2^(s-1) finite in bf16
                    const uint32_t s0 = place ? e8m0_place_bf16x2(b0) : e8m0_bf16x2(b0);
                    const uint32_t s1 = place ? e8m0_place_bf16x2(b1) : e8m0_bf16x2(b1);
                    uint8_t* arow = sA + stage * kMxATile + h * kAHalfBytes + row * 128;
                    const uint32_t words[8] = {c0[h].x, c0[h].y, c0[h].z, c0[h].w, c1[h].x, c1[h].y, c1[h].z, c1[h].w};
                    if (place) {
#pragma unroll
                        for (int cch = 0; cch < 8; ++cch) {
                            uint32_t o[4];
                            e2m1x8_bf16_place(words[cch], cch < 4 ? s0 : s1, o);
                            sts128(arow + ((cch ^ (row & 7)) << 4), o[0], o[1], o[2], o[3]);
                        }
                    } else {
#pragma unroll
                        for (int cch = 0; cch < 8; ++cch) {   // 16-byte chunk cch = elements 8cch .. 8cch+7
                            uint32_t o[4];
                            e2m1x8_bf16(words[cch], cch < 4 ? s0 : s1, o);
                            sts128(arow + ((cch ^ (row & 7)) << 4), o[0], o[1], o[2], o[3]);
                        }
                    }
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(afull_lead + uint32_t(stage) * 8u);
            }
            if (ok) {
                // this tile's accumulators -> h / o_sorted: warp (lane quarter warp & 3) takes
                // the column chunks of parity gi
                const Tile tl = decode_tile<4>(t, ntile_off, G, s_off, p.m_tiles, p.m_rows);
                if (!mbar_wait(tfull, acc_phase, abort_flag, p.wait_ns)) { ok = false; break; }
                tc_fence_after();
                uint16_t* xb = reinterpret_cast<uint16_t*>(sX + (warp - kMxConvWarp0) * kXposeBytes);
                epilogue_tile<2>(p, tl, 2, tmem_base + (uint32_t((warp & 3) * 32) << 16), tl.m * 4 + int(rank), 2,
                                 warp & 3, gi, lane, xb);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(tempty_lead);
                acc_phase ^= 1;
            }
        }
        if (!ok) { *abort_flag = 1; if (lane == 0) atomicExch(p.err, kDevErrTimeout); }
    }
    // teardown: every MMA of the pair is complete (mma_done) and both CTAs are past their last
    // TMEM read and remote arrival before the pair's TMEM is freed and either CTA exits
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(2 * kAccCols));
}

// ------------------------------------------------------------------ host side
bool mx_pair_eligible(int mode, int H, int F) {
    const int K = mode == 0 ? H : F;
    const int m_rows = mode == 0 ? F / 64 : H / 128;
    return K % kMxGroupK == 0 && m_rows % 4 == 0;
}

// Code / scale tensor maps of one weight tensor (n_exp experts).  Gate/up: codes [E][2F][H/2]
// viewed as (H/2, 16, 2, F/16, E) so one box brings four blocks of 16 gate rows each followed
// by the 16 matching up rows; down: codes [E][H][F/2] as (F/2, H, E).  Scales likewise with
// K/32 bytes per row.
static bool mx_maps(int mode, int H, int F, int n_exp, const void* codes, const uint8_t* scales, CUtensorMap* mc,
                    CUtensorMap* ms) {
    if (mode == 0) {
        const uint64_t kq = uint64_t(H) / 2, ks = uint64_t(H) / 32;
        uint64_t dc[5] = {kq, 16, 2, uint64_t(F / 16), uint64_t(n_exp)};
        uint64_t sc[4] = {kq, uint64_t(F) * kq, 16 * kq, 2 * uint64_t(F) * kq};
        uint32_t bc[5] = {uint32_t(kMxUnitK / 2), 16, 2, 4, 1};
        uint64_t ds[5] = {ks, 16, 2, uint64_t(F / 16), uint64_t(n_exp)};
        uint64_t ss[4] = {ks, uint64_t(F) * ks, 16 * ks, 2 * uint64_t(F) * ks};
        uint32_t bs[5] = {16, 16, 2, 4, 1};
        return make_map(mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, 5, dc, sc, bc, CU_TENSOR_MAP_SWIZZLE_64B) &&
               make_map(ms, CU_TENSOR_MAP_DATA_TYPE_UINT8, scales, 5, ds, ss, bs, CU_TENSOR_MAP_SWIZZLE_NONE);
    }
    const uint64_t kq = uint64_t(F) / 2, ks = uint64_t(F) / 32;
    uint64_t dc[3] = {kq, uint64_t(H), uint64_t(n_exp)};
    uint64_t sc[2] = {kq, uint64_t(H) * kq};
    uint32_t bc[3] = {uint32_t(kMxUnitK / 2), 128, 1};
    uint64_t ds[3] = {ks, uint64_t(H), uint64_t(n_exp)};
    uint64_t ss[2] = {ks, uint64_t(H) * ks};
    uint32_t bs[3] = {16, 128, 1};
    return make_map(mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, 3, dc, sc, bc, CU_TENSOR_MAP_SWIZZLE_64B) &&
           make_map(ms, CU_TENSOR_MAP_DATA_TYPE_UINT8, scales, 3, ds, ss, bs, CU_TENSOR_MAP_SWIZZLE_NONE);
}

// returns 0 ok, 1 tensor-map failure, 2 launch failure
int launch_moe_gemm_mx_pair(const GemmLaunch& L, const GemmParams& p0, cudaStream_t st) {
    GemmParams p = p0;
    p.m_tiles = p.m_rows / 4;
    const int K = p.K;
    CUtensorMap mc{}, ms{}, msc{}, mss{}, tb[kNumBMaps]{};
    if (!mx_maps(L.mode, L.H, L.F, L.E, L.w, L.wscale, &mc, &ms)) return 1;
    if (L.S) {
        if (!mx_maps(L.mode, L.H, L.F, 1, L.sw, L.swscale, &msc, &mss)) return 1;
    } else {
        msc = mc;
        mss = ms;
    }
    // each CTA loads half of a token tile: boxes of 8 .. 128 rows
    const int rR8 = (L.R + 7) & ~7;
    for (int i = 0; i < kNumBMaps; ++i) {
        p.b_rows[i] = (8 << i) < rR8 ? (8 << i) : rR8;
        uint64_t dims[2] = {uint64_t(K), uint64_t(L.R)};
        uint64_t str[1] = {uint64_t(K) * 2};
        uint32_t box[2] = {kBK, uint32_t(p.b_rows[i])};
        if (!make_map(&tb[i], L.act, 2, dims, str, box)) return 1;
    }
    constexpr size_t smem = mx_pair_smem_bytes();
    static int max_clusters = 0;
    static PerDeviceOnce attr;
    if (attr([&] { return cudaFuncSetAttribute(moe_gemm_mx_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)); }) !=
        cudaSuccess)
        return 2;
    if (!max_clusters) {   // the same on every device of one model: queried once
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(2 * (num_sms() / 2));
        cfg.blockDim = dim3(kMxThreads);
        cfg.dynamicSmemBytes = smem;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, moe_gemm_mx_pair_kernel, &cfg) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = num_sms() / 2;
        }
        max_clusters = n;
    }
    int clusters = max_clusters;
    const int pair_tiles = L.max_tiles * p.m_tiles;
    if (pair_tiles < clusters) clusters = pair_tiles > 0 ? pair_tiles : 1;
    moe_gemm_mx_pair_kernel<<<2 * clusters, kMxThreads, smem, st>>>(mc, ms, msc, mss, tb[0], tb[1], tb[2], tb[3], tb[4], p);
    return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

}  // namespace ftmoe

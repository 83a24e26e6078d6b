// Step 3 (prefill) -- grouped expert GEMMs on the 5th-generation tensor cores.
//
//   gate/up:  D[128 weight rows, N tokens] = W13_e[rows, H] . Xs[tokens, H]^T, then
//             h[token, f] = silu(gate) * up  (fused epilogue), h stored bf16 [R, F]
//   down:     D[128 hidden rows, N tokens] = W2_e[rows, F] . h[tokens, F]^T,
//             o_sorted[token, hrow] stored bf16 [R, H]
//
// "Weights as A": the MMA M dimension walks weight rows and N walks the tokens of one
// expert group, so an expert with few tokens costs an MMA of N = round_up(n, 16) instead
// of a padded 128-row tile, and its activation box shrinks to the next power of two.
// For long contractions a CTA tile is 256 weight rows (two M=128 MMAs into two TMEM
// accumulators) x N tokens, so each activation stage feeds twice the math; for short ones
// it is 128 rows with double-buffered accumulators (see moe_gemm_kernel's HV).  The gate/up A tile interleaves gate and up rows in
// blocks of 16 (rows 32i..32i+15 = gate f0+16i.., rows 32i+16..32i+31 = up f0+16i..), so
// each TMEM lane quarter holds gate and up of the same 16 f values: lane l and l^16
// exchange halves with one shuffle, no shared-memory round trip.
//
// Warp roles (one CTA per SM, persistent over a device-side tile list):
//   warp 0      TMA producer (weights for BF16; activations always)
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer
//   warps 2-9   BF16: epilogue, two warps per TMEM lane quarter (tcgen05.ld 32x32b)
//   warps 2-5   MXFP4: epilogue;  warps 6-9: load E2M1 codes + E8M0 scales with 128-bit
//               loads, dequantise exactly to bf16 and write the SW128 A tile to smem
// Operands are K-major, 128-byte swizzled (3 x 64 KB or 4 x 48 KB stage ring); the fp32
// accumulators take all 512 TMEM columns.
// Every wait is bounded: on timeout the kernel records kDevErrTimeout, drains its own
// copies and MMAs, frees TMEM and returns.
#include "gemm_common.cuh"

namespace ftmoe {

// HV = 2: 256 weight rows per tile, both TMEM accumulators belong to one tile (single
//         buffered), 3 stages of 64 KB -- the least activation traffic per FLOP; for long K.
// HV = 1: 128 weight rows per tile, accumulators double buffered so the epilogue of tile i
//         overlaps the MMAs of tile i+1, 4 stages of 48 KB; for short K.
template <bool MX, int HV>
__global__ void __launch_bounds__(320, 1)
moe_gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_sw,
                const __grid_constant__ CUtensorMap tm_b0, const __grid_constant__ CUtensorMap tm_b1,
                const __grid_constant__ CUtensorMap tm_b2, const __grid_constant__ CUtensorMap tm_b3,
                const __grid_constant__ CUtensorMap tm_b4, GemmParams p) {
    constexpr int kEpiWarps = MX ? 4 : 8;
    constexpr int kSt = HV == 2 ? 3 : 4;                 // pipeline stages
    constexpr int kATile = HV * kAHalfBytes;             // A bytes per stage
    constexpr int kNBuf = HV == 2 ? 1 : 2;               // accumulator buffers
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + kSt * kATile;
    uint8_t* sX = sB + kSt * kBTileBytes;                // epilogue transpose buffers, 2 KB per warp
    uint64_t* full = reinterpret_cast<uint64_t*>(sX + 8 * kXposeBytes);
    uint64_t* empty = full + kSt;
    uint64_t* tfull = empty + kSt;
    uint64_t* tempty = tfull + kNBuf;
    uint64_t* mma_done = tempty + kNBuf;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* ntile_off = const_cast<int*>(reinterpret_cast<volatile int*>(tmem_slot + 2));
    int* s_off = ntile_off + 260;                        // group row offsets [G+1]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = p.G;
    for (int i = tid; i <= G; i += blockDim.x) {
        ntile_off[i] = p.sched[2 + i];
        s_off[i] = p.offsets[i];
    }
    if (tid == 0) {
        for (int s = 0; s < kSt; ++s) {
            mbar_init(&full[s], MX ? 1 + 4 : 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < kNBuf; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], kEpiWarps);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(tmem_slot)),
                     "r"(2 * kAccCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int total = ntile_off[G] * p.m_tiles;
    const int nk = p.K / kBK;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            const CUtensorMap* bm[kNumBMaps] = {&tm_b0, &tm_b1, &tm_b2, &tm_b3, &tm_b4};
            int stage = 0;
            uint32_t phase = 0;
            int issued[kSt];
            uint32_t issued_par[kSt];
            for (int s = 0; s < kSt; ++s) issued[s] = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                const Tile tl = decode_tile<HV>(t, ntile_off, G, s_off, p.m_tiles, p.m_rows);
                const bool shared_grp = p.has_shared && tl.g == p.E;
                const int bi = bmap_index(tl.nvalid);
                const uint32_t bbytes = uint32_t(p.b_rows[bi]) * kBK * 2;
                const uint32_t abytes = MX ? 0u : uint32_t(tl.halves) * kAHalfBytes;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.wait_ns)) { ok = false; break; }
                    uint8_t* a = sA + stage * kATile;
                    uint8_t* b = sB + stage * kBTileBytes;
                    const int k0 = kb * kBK;
                    mbar_expect_tx(&full[stage], abytes + bbytes);
                    if (!MX) {
                        const CUtensorMap* m = shared_grp ? &tm_sw : &tm_w;
                        const int e = shared_grp ? 0 : tl.g;
                        for (int h = 0; h < tl.halves; ++h) {
                            const int rg = tl.m * HV + h;       // 128-row weight group index
                            if (p.mode == 0) {
                                // (k, row-in-block, gate|up, 16-row block, expert): 4 blocks of 16
                                // gate + 16 up rows land interleaved, one copy per half
                                tma_5d(m, &full[stage], a + h * kAHalfBytes, k0, 0, 0, rg * 4, e);
                            } else {
                                tma_3d(m, &full[stage], a + h * kAHalfBytes, k0, rg * 128, e);
                            }
                        }
                    }
                    tma_2d(bm[bi], &full[stage], b, k0, tl.row0);
                    issued[stage] = 1;
                    issued_par[stage] = phase;
                    if (++stage == kSt) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok) { *abort_flag = 1; atomicExch(p.err, kDevErrTimeout); }
            // drain: every copy this thread issued must have landed before the CTA exits
            for (int s = 0; s < kSt; ++s)
                if (issued[s]) mbar_wait(&full[s], issued_par[s], nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0, buf = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                const Tile tl = decode_tile<HV>(t, ntile_off, G, s_off, p.m_tiles, p.m_rows);
                const int N = (tl.nvalid + 15) & ~15;
                const uint32_t idesc = idesc_bf16(128, N);
                if (!mbar_wait(&tempty[buf], acc_phase ^ 1, abort_flag, p.wait_ns)) { ok = false; break; }
                tc_fence_after();
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(&full[stage], phase, abort_flag, p.wait_ns)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t bd = sdesc_sw128(su32(sB + stage * kBTileBytes));
                    for (int h = 0; h < tl.halves; ++h) {
                        const uint64_t ad = sdesc_sw128(su32(sA + stage * kATile + h * kAHalfBytes));
                        const uint32_t dtm = tmem_base + uint32_t((buf * HV + h) * kAccCols);
#pragma unroll
                        for (int kk = 0; kk < kBK / 16; ++kk)
                            umma_bf16(dtm, ad + uint64_t(kk * 2), bd + uint64_t(kk * 2), idesc, (kb | kk) != 0);
                    }
                    umma_commit(&empty[stage]);
                    if (++stage == kSt) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                umma_commit(&tfull[buf]);
                if (++buf == kNBuf) { buf = 0; acc_phase ^= 1; }
            }
            if (!ok) { *abort_flag = 1; atomicExch(p.err, kDevErrTimeout); }
            umma_commit(mma_done);               // tracks completion of every MMA issued above
            mbar_wait(mma_done, 0, nullptr);
        }
    } else if (warp < 2 + kEpiWarps) {
        // ------------------------------------------------ epilogue (TMEM -> registers -> smem -> global)
        // Two 32-column chunks are loaded per tcgen05.wait; each chunk is transposed through a
        // per-warp shared buffer so the global stores are 16-byte vectors along the token row.
        const int q = warp & 3;                  // TMEM lanes 32q .. 32q+31
        const int part = (warp - 2) >> 2;        // which column chunks this warp takes
        constexpr int kParts = kEpiWarps / 4;
        uint16_t* xb = reinterpret_cast<uint16_t*>(sX + (warp - 2) * kXposeBytes);
        int buf = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total; t += gridDim.x) {
            const Tile tl = decode_tile<HV>(t, ntile_off, G, s_off, p.m_tiles, p.m_rows);
            if (!mbar_wait(&tfull[buf], acc_phase, abort_flag, p.wait_ns)) { ok = false; break; }
            tc_fence_after();
            epilogue_tile<kParts>(p, tl, tl.halves, tmem_base + (uint32_t(q * 32) << 16) + uint32_t(buf * HV * kAccCols),
                                  tl.m * HV, 1, q, part, lane, xb);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[buf]);
            if (++buf == kNBuf) { buf = 0; acc_phase ^= 1; }
        }
        if (!ok) { *abort_flag = 1; if (lane == 0) atomicExch(p.err, kDevErrTimeout); }
    } else if (MX) {
        // ------------------------------------------------ MXFP4 converter warps (one A row per half per thread)
        const int r0 = tid - 64 - 32 * kEpiWarps;   // 0..127: row r0 of each 128-row half
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        const int kq = p.K / 2, ks = p.K / 32;   // code / scale bytes per weight row
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
            const Tile tl = decode_tile<HV>(t, ntile_off, G, s_off, p.m_tiles, p.m_rows);
            const bool shared_grp = p.has_shared && tl.g == p.E;
            const size_t e = shared_grp ? 0 : size_t(tl.g);
            const uint8_t* qrow[HV];
            const uint8_t* srow[HV];
#pragma unroll
            for (int h = 0; h < HV; ++h) {
                const int rg = tl.m * HV + (h < tl.halves ? h : 0);   // a missing half re-reads half 0 (unused)
                int wrow;
                size_t rows_per_expert;
                if (p.mode == 0) {
                    const int i = r0 >> 5, j = r0 & 31;
                    const int f = rg * 64 + 16 * i + (j & 15);
                    wrow = j < 16 ? f : p.F + f;
                    rows_per_expert = size_t(2) * p.F;
                } else {
                    wrow = rg * 128 + r0;
                    rows_per_expert = size_t(p.H);
                }
                qrow[h] = (shared_grp ? p.swq : p.wq) + (e * rows_per_expert + wrow) * kq;
                srow[h] = (shared_grp ? p.sws : p.ws) + (e * rows_per_expert + wrow) * ks;
            }
            uint4 c[HV][2];
            uint32_t sc[HV];
#pragma unroll
            for (int h = 0; h < HV; ++h) {
                c[h][0] = ldg_nc_v4(qrow[h]);
                c[h][1] = ldg_nc_v4(qrow[h] + 16);
                sc[h] = *reinterpret_cast<const uint16_t*>(srow[h]);
            }
            for (int kb = 0; kb < nk; ++kb) {
                uint4 nx[HV][2];
                uint32_t nsc[HV];
#pragma unroll
                for (int h = 0; h < HV; ++h) {
                    nx[h][0] = c[h][0]; nx[h][1] = c[h][1]; nsc[h] = sc[h];
                    if (kb + 1 < nk) {
                        nx[h][0] = ldg_nc_v4(qrow[h] + (kb + 1) * 32);
                        nx[h][1] = ldg_nc_v4(qrow[h] + (kb + 1) * 32 + 16);
                        nsc[h] = *reinterpret_cast<const uint16_t*>(srow[h] + (kb + 1) * 2);
                    }
                }
                if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.wait_ns)) { ok = false; break; }
#pragma unroll
                for (int h = 0; h < HV; ++h) {
                    if (h >= tl.halves) break;
                    uint8_t* arow = sA + stage * kATile + h * kAHalfBytes + r0 * 128;
                    const uint32_t s0 = e8m0_bf16x2(sc[h] & 0xFF), s1 = e8m0_bf16x2(sc[h] >> 8);
                    const uint32_t words[8] = {c[h][0].x, c[h][0].y, c[h][0].z, c[h][0].w,
                                               c[h][1].x, c[h][1].y, c[h][1].z, c[h][1].w};
#pragma unroll
                    for (int cch = 0; cch < 8; ++cch) {  // 16-byte chunk cch = elements 8cch..8cch+7
                        uint32_t o[4];
                        e2m1x8_bf16(words[cch], cch < 4 ? s0 : s1, o);
                        *reinterpret_cast<uint4*>(arow + ((cch ^ (r0 & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
                    }
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(&full[stage]);
                if (++stage == kSt) { stage = 0; phase ^= 1; }
#pragma unroll
                for (int h = 0; h < HV; ++h) { c[h][0] = nx[h][0]; c[h][1] = nx[h][1]; sc[h] = nsc[h]; }
            }
        }
        if (!ok) { *abort_flag = 1; if (lane == 0) atomicExch(p.err, kDevErrTimeout); }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(2 * kAccCols));
    }
}

// ------------------------------------------------------------------ CTA pairs (BF16)
// Two CTAs of a cluster share every MMA (tcgen05.mma.cta_group::2, M = 256): CTA r supplies
// 128 weight rows of each MMA and half of the token tile (rows r*N/2 .. of it) from its own
// shared memory and keeps its 128 accumulator rows in its own TMEM.
//   HPC = 2 (gate/up, long K): a pair tile is 512 weight rows (two MMAs, four 128-row groups:
//           CTA r holds groups 4m + r and 4m + 2 + r) x up to 256 tokens; both accumulators
//           (2 x 256 columns) belong to one tile.  Per SM a stage carries 32 KB of weights and
//           at most 16 KB of tokens for the work the single-CTA 256 x 256 tile does with 64 KB,
//           so four stages fit.
//   HPC = 1 (down, short K): a pair tile is 256 weight rows (one MMA, CTA r holds group
//           2m + r) x up to 256 tokens; the accumulators are double buffered (2 x 256 columns)
//           so a tile's epilogue overlaps the next tile's MMAs, and six 32 KB stages fit.  Each
//           CTA reads half the token tile of the single-CTA kernel per FLOP (the token tile is
//           the larger operand of the down GEMM).
// A group index at or beyond m_rows (the last pair tile of an odd group count) is zero-filled
// by TMA and its results are not stored.
// Only the leader (rank 0) waits for operands and issues MMAs: both CTAs' TMA copies count on
// its `full` barrier, its commits arrive on the `empty` / `tfull` / `done` barriers of both
// CTAs, and both CTAs' epilogue warps arrive on its `tempty` barrier.  No TMA multicast.
constexpr int kPairBTile = 128 * kBK * 2;              // 16 KB: up to 128 token rows
template <int HPC> struct PairCfg {
    static constexpr int kATile = HPC * kAHalfBytes;
    static constexpr int kSt = HPC == 2 ? 4 : 6;
    static constexpr int kNBuf = HPC == 2 ? 1 : 2;
    static constexpr int kGroups = 2 * HPC;            // 128-row groups per pair tile
    static constexpr size_t smem() {
        return 1024 + size_t(kSt) * (kATile + kPairBTile) + 8 * kXposeBytes + 256 + 8 * 260;
    }
};

template <int HPC>
__device__ __forceinline__ int pair_group(int m, int h, uint32_t rank) {
    return HPC == 2 ? m * 4 + 2 * h + int(rank) : m * 2 + int(rank);
}

template <int HPC>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(320, 1)
moe_gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_sw,
                     const __grid_constant__ CUtensorMap tm_b0, const __grid_constant__ CUtensorMap tm_b1,
                     const __grid_constant__ CUtensorMap tm_b2, const __grid_constant__ CUtensorMap tm_b3,
                     const __grid_constant__ CUtensorMap tm_b4, GemmParams p) {
    using C = PairCfg<HPC>;
    constexpr int kEpiWarps = 8;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + C::kSt * C::kATile;
    uint8_t* sX = sB + C::kSt * kPairBTile;
    uint64_t* full = reinterpret_cast<uint64_t*>(sX + kEpiWarps * kXposeBytes);
    uint64_t* empty = full + C::kSt;
    uint64_t* tfull = empty + C::kSt;
    uint64_t* tempty = tfull + C::kNBuf;
    uint64_t* mma_done = tempty + C::kNBuf;
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
        for (int st = 0; st < C::kSt; ++st) {
            mbar_init(&full[st], 1);            // the leader's producer arrives (with all bytes expected)
            mbar_init(&empty[st], 1);           // the leader's MMA commit
        }
        for (int b = 0; b < C::kNBuf; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 2 * kEpiWarps);   // every epilogue warp of both CTAs
        }
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
    const uint32_t full_lead = mapa_rank(su32(full), 0);      // the leader's full[0]
    const uint32_t tempty_lead = mapa_rank(su32(tempty), 0);

    const int total = ntile_off[G] * p.m_tiles;
    const int nk = p.K / kBK;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            const CUtensorMap* bm[kNumBMaps] = {&tm_b0, &tm_b1, &tm_b2, &tm_b3, &tm_b4};
            int stage = 0;
            uint32_t phase = 0;
            int issued[C::kSt];
            uint32_t issued_par[C::kSt];
            for (int st = 0; st < C::kSt; ++st) issued[st] = 0;
            bool ok = true;
            for (int t = cid; t < total && ok; t += ncl) {
                const Tile tl = decode_tile<C::kGroups>(t, ntile_off, G, s_off, p.m_tiles, p.m_rows);
                const bool shared_grp = p.has_shared && tl.g == p.E;
                const int nh = ((tl.nvalid + 15) & ~15) >> 1;   // token rows per CTA
                int bi = 0;
                while (bi < kNumBMaps - 1 && (8 << bi) < nh) ++bi;
                const uint32_t bbytes = uint32_t(p.b_rows[bi]) * kBK * 2;
                const CUtensorMap* m = shared_grp ? &tm_sw : &tm_w;
                const int e = shared_grp ? 0 : tl.g;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.wait_ns)) { ok = false; break; }
                    uint8_t* a = sA + stage * C::kATile;
                    uint8_t* b = sB + stage * kPairBTile;
                    const int k0 = kb * kBK;
                    const uint32_t bar = full_lead + uint32_t(stage) * 8u;
                    if (rank == 0) mbar_expect_tx(&full[stage], 2u * (uint32_t(C::kATile) + bbytes));
                    for (int h = 0; h < HPC; ++h) {
                        const int rg = pair_group<HPC>(tl.m, h, rank);
                        if (p.mode == 0) tma_5d_pair(m, bar, a + h * kAHalfBytes, k0, 0, 0, rg * 4, e);
                        else tma_3d_pair(m, bar, a + h * kAHalfBytes, k0, rg * 128, e);
                    }
                    tma_2d_pair(bm[bi], bar, b, k0, tl.row0 + int(rank) * nh);
                    issued[stage] = 1;
                    issued_par[stage] = phase;
                    if (++stage == C::kSt) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok) { *abort_flag = 1; atomicExch(p.err, kDevErrTimeout); }
            // drain: the leader sees its full barriers complete (both CTAs' bytes landed); the
            // peer sees its empty barriers released (the leader consumed what it copied)
            for (int st = 0; st < C::kSt; ++st)
                if (issued[st]) {
                    if (rank == 0) mbar_wait(&full[st], issued_par[st], nullptr);
                    else mbar_wait(&empty[st], issued_par[st], nullptr);
                }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (leader only)
        if (lane == 0) {
            if (rank == 0) {
                int stage = 0, buf = 0;
                uint32_t phase = 0, acc_phase = 0;
                bool ok = true;
                for (int t = cid; t < total && ok; t += ncl) {
                    const Tile tl = decode_tile<C::kGroups>(t, ntile_off, G, s_off, p.m_tiles, p.m_rows);
                    const int N = (tl.nvalid + 15) & ~15;
                    const uint32_t idesc = idesc_bf16(256, N);
                    if (!mbar_wait_cluster(&tempty[buf], acc_phase ^ 1, abort_flag, p.wait_ns)) { ok = false; break; }
                    tc_fence_after();
                    for (int kb = 0; kb < nk; ++kb) {
                        if (!mbar_wait(&full[stage], phase, abort_flag, p.wait_ns)) { ok = false; break; }
                        tc_fence_after();
                        const uint64_t bd = sdesc_sw128(su32(sB + stage * kPairBTile));
                        for (int h = 0; h < HPC; ++h) {
                            const uint64_t ad = sdesc_sw128(su32(sA + stage * C::kATile + h * kAHalfBytes));
                            const uint32_t dtm = tmem_base + uint32_t((buf * HPC + h) * kAccCols);
#pragma unroll
                            for (int kk = 0; kk < kBK / 16; ++kk)
                                umma_bf16_pair(dtm, ad + uint64_t(kk * 2), bd + uint64_t(kk * 2), idesc, (kb | kk) != 0);
                        }
                        umma_commit_pair_both(&empty[stage]);
                        if (++stage == C::kSt) { stage = 0; phase ^= 1; }
                    }
                    if (!ok) break;
                    umma_commit_pair_both(&tfull[buf]);
                    if (++buf == C::kNBuf) { buf = 0; acc_phase ^= 1; }
                }
                if (!ok) { *abort_flag = 1; atomicExch(p.err, kDevErrTimeout); }
                umma_commit_pair_both(mma_done);     // completion of every MMA issued above, in both CTAs
            }
            mbar_wait(mma_done, 0, nullptr);
        }
    } else if (warp < 2 + kEpiWarps) {
        // ------------------------------------------------ epilogue (both CTAs, own 128 rows)
        const int q = warp & 3;
        const int part = (warp - 2) >> 2;
        constexpr int kParts = kEpiWarps / 4;
        uint16_t* xb = reinterpret_cast<uint16_t*>(sX + (warp - 2) * kXposeBytes);
        int buf = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int t = cid; t < total; t += ncl) {
            const Tile tl = decode_tile<C::kGroups>(t, ntile_off, G, s_off, p.m_tiles, p.m_rows);
            if (!mbar_wait(&tfull[buf], acc_phase, abort_flag, p.wait_ns)) { ok = false; break; }
            tc_fence_after();
            const int rg0 = pair_group<HPC>(tl.m, 0, rank);
            // groups past the weight rows (odd group counts) were zero-filled: nothing to store
            const int halves = HPC == 2 ? (rg0 + 2 < p.m_rows ? 2 : (rg0 < p.m_rows ? 1 : 0)) : (rg0 < p.m_rows ? 1 : 0);
            if (halves)
                epilogue_tile<kParts>(p, tl, halves, tmem_base + (uint32_t(q * 32) << 16) + uint32_t(buf * HPC * kAccCols),
                                      rg0, 2, q, part, lane, xb);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(tempty_lead + uint32_t(buf) * 8u);
            if (++buf == C::kNBuf) { buf = 0; acc_phase ^= 1; }
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
static size_t gemm_smem_bytes(int hv) {
    const int stages = hv == 2 ? 3 : 4;
    return 1024 + size_t(stages) * (hv * kAHalfBytes + kBTileBytes) + 8 * kXposeBytes + 256 + 8 * 260;
}

// Tile height: long contractions (K >= 1536) amortise the single-buffered 256-row tile's
// epilogue; short ones keep 128-row tiles with double-buffered accumulators.
static int pick_halves(int K) { return K >= 1536 ? 2 : 1; }

template <bool MX, int HV>
static int launch_variant(int grid, cudaStream_t st, const CUtensorMap& tw, const CUtensorMap& tsw, const CUtensorMap* tb,
                          const GemmParams& p) {
    const size_t smem = gemm_smem_bytes(HV);
    static PerDeviceOnce attr;
    if (attr([&] { return cudaFuncSetAttribute(moe_gemm_kernel<MX, HV>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)); }) !=
        cudaSuccess)
        return 2;
    moe_gemm_kernel<MX, HV><<<grid, 320, smem, st>>>(tw, tsw, tb[0], tb[1], tb[2], tb[3], tb[4], p);
    return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

template <int HPC>
static int launch_pair(const GemmLaunch& L, const GemmParams& p, const CUtensorMap& tw, const CUtensorMap& tsw,
                       cudaStream_t st) {
    using C = PairCfg<HPC>;
    const int K = p.K;
    // each CTA loads half of a token tile, so the token boxes are 8 .. 128 rows
    GemmParams pp = p;
    pp.m_tiles = (p.m_rows + C::kGroups - 1) / C::kGroups;
    CUtensorMap tbp[kNumBMaps]{};
    const int rR8 = (L.R + 7) & ~7;
    for (int i = 0; i < kNumBMaps; ++i) {
        pp.b_rows[i] = (8 << i) < rR8 ? (8 << i) : rR8;
        uint64_t dims[2] = {uint64_t(K), uint64_t(L.R)};
        uint64_t str[1] = {uint64_t(K) * 2};
        uint32_t box[2] = {kBK, uint32_t(pp.b_rows[i])};
        if (!make_map(&tbp[i], L.act, 2, dims, str, box)) return 1;
    }
    static int max_clusters = 0;
    constexpr size_t smem = C::smem();
    static PerDeviceOnce attr;
    if (attr([&] { return cudaFuncSetAttribute(moe_gemm_pair_kernel<HPC>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)); }) !=
        cudaSuccess)
        return 2;
    if (!max_clusters) {   // the same on every device of one model: queried once
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(2 * (num_sms() / 2));
        cfg.blockDim = dim3(320);
        cfg.dynamicSmemBytes = smem;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, moe_gemm_pair_kernel<HPC>, &cfg) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = num_sms() / 2;
        }
        max_clusters = n;
    }
    int clusters = max_clusters;
    const int pair_tiles = L.max_tiles * pp.m_tiles;
    if (pair_tiles < clusters) clusters = pair_tiles > 0 ? pair_tiles : 1;
    moe_gemm_pair_kernel<HPC><<<2 * clusters, 320, smem, st>>>(tw, tsw, tbp[0], tbp[1], tbp[2], tbp[3], tbp[4], pp);
    return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

// returns 0 ok, 1 tensor-map failure, 2 launch failure
int launch_moe_gemm(const GemmLaunch& L, cudaStream_t st) {
    const bool mx = L.wdtype == FT_W_MXFP4;
    const int K = L.mode == 0 ? L.H : L.F;
    CUtensorMap tw{}, tsw{}, tb[kNumBMaps]{};
    GemmParams p{};
    const int rR = (L.R + 15) & ~15;
    for (int i = 0; i < kNumBMaps; ++i) {
        p.b_rows[i] = (16 << i) < rR ? (16 << i) : rR;
        uint64_t dims[2] = {uint64_t(K), uint64_t(L.R)};
        uint64_t str[1] = {uint64_t(K) * 2};
        uint32_t box[2] = {kBK, uint32_t(p.b_rows[i])};
        if (!make_map(&tb[i], L.act, 2, dims, str, box)) return 1;
    }
    if (!mx) {
        if (L.mode == 0) {
            // w13 [E][2][F][H] viewed as (H, 16, 2, F/16, E): a (64, 16, 2, 4, 1) box is 4 blocks
            // of 16 gate rows each followed by the 16 matching up rows (one copy per 128 rows;
            // four 4-D copies per half measured 4-5 % slower)
            uint64_t dims[5] = {uint64_t(L.H), 16, 2, uint64_t(L.F / 16), uint64_t(L.E)};
            uint64_t str[4] = {uint64_t(L.H) * 2, uint64_t(L.F) * L.H * 2, uint64_t(16) * L.H * 2,
                               uint64_t(2) * L.F * L.H * 2};
            uint32_t box[5] = {kBK, 16, 2, 4, 1};
            if (!make_map(&tw, L.w, 5, dims, str, box)) return 1;
            if (L.S) {
                uint64_t d1[5] = {uint64_t(L.H), 16, 2, uint64_t(L.F / 16), 1};
                if (!make_map(&tsw, L.sw, 5, d1, str, box)) return 1;
            } else {
                tsw = tw;
            }
        } else {
            uint64_t dims[3] = {uint64_t(L.F), uint64_t(L.H), uint64_t(L.E)};
            uint64_t str[2] = {uint64_t(L.F) * 2, uint64_t(L.H) * L.F * 2};
            uint32_t box[3] = {kBK, 128, 1};
            if (!make_map(&tw, L.w, 3, dims, str, box)) return 1;
            if (L.S) {
                uint64_t d1[3] = {uint64_t(L.F), uint64_t(L.H), 1};
                if (!make_map(&tsw, L.sw, 3, d1, str, box)) return 1;
            } else {
                tsw = tw;
            }
        }
    } else {
        tw = tb[0];   // unused by the MXFP4 kernel (A comes from the converter warps)
        tsw = tb[0];
    }
    const int hv = pick_halves(K);
    p.mode = L.mode;
    p.wait_ns = gemm_wait_ns();
    p.K = K;
    p.m_rows = L.mode == 0 ? L.F / 64 : L.H / 128;
    p.m_tiles = (p.m_rows + hv - 1) / hv;
    p.G = L.E + (L.S ? 1 : 0);
    p.E = L.E;
    p.F = L.F;
    p.H = L.H;
    p.has_shared = L.S ? 1 : 0;
    p.offsets = L.offsets;
    p.sched = L.sched;
    p.out = L.out;
    p.out_ld = L.mode == 0 ? L.F : L.H;
    p.err = L.err;
    p.wq = static_cast<const uint8_t*>(L.w);
    p.ws = L.wscale;
    p.swq = static_cast<const uint8_t*>(L.sw);
    p.sws = L.swscale;
    if (mx && mx_pair_eligible(L.mode, L.H, L.F)) return launch_moe_gemm_mx_pair(L, p, st);
    // BF16 on CTA pairs: gate/up of long contractions in pair tiles of 512 weight rows (four
    // 128-row groups), down in pair tiles of 256 rows with double-buffered accumulators
    if (!mx && L.mode == 0 && hv == 2 && p.m_rows % 4 == 0) return launch_pair<2>(L, p, tw, tsw, st);
    if (!mx && L.mode == 1 && p.m_rows % 2 == 0) return launch_pair<1>(L, p, tw, tsw, st);
    int grid = num_sms();
    const int max_tiles = L.max_tiles * p.m_tiles;
    if (max_tiles < grid) grid = max_tiles > 0 ? max_tiles : 1;
    if (mx) return hv == 2 ? launch_variant<true, 2>(grid, st, tw, tsw, tb, p) : launch_variant<true, 1>(grid, st, tw, tsw, tb, p);
    return hv == 2 ? launch_variant<false, 2>(grid, st, tw, tsw, tb, p) : launch_variant<false, 1>(grid, st, tw, tsw, tb, p);
}

}  // namespace ftmoe

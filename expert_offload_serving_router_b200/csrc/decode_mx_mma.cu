// Steps 3/4 (decode, MXFP4 weights) on the block-scaled tensor cores.
//
// The MXFP4 GEMVs are bound by decoding E2M1 codes on the ALUs.  Here the tensor core takes the
// codes as they are: tcgen05.mma.kind::mxf8f6f4.block_scale multiplies E2M1 weights (A, with
// their E8M0 scale per 32 elements) by E4M3 activations (B, with E8M0 scales).  A single E4M3
// copy of the activations loses too much (the error study: 5.6e-2 of max|y| on the
// DeepSeek-V4-Flash-shaped layer, over the 3e-2 tolerance), so each activation row is carried as
// two planes -- hi = the OCP MX conversion of v, lo = the same conversion of v - hi, each with its
// own E8M0 scale per 32 (1.2e-3 of max|y| in the study).  Both planes form one B operand of
// 2 NB rows (hi rows, then lo rows), so each 32-deep K block is one MMA, and the epilogue adds
// accumulator column c and column NB + c.
//
//   quant2_kernel:  bf16 rows -> E4M3 planes hi, lo [rows, K] + E8M0 scales [rows, K/32] each.
//   decode_mx_mma_kernel<MODE>: items (active group, 128 weight rows), a contiguous run of them per
//       persistent CTA; per 256-deep K stage TMA brings 128 rows of codes unpacked to one byte per
//       element (16U4_ALIGN16B, SW128) and the two activation planes.  The MMA thread issues only
//       MMAs and commits.  The epilogue warps lay each item's weight scales (and, when they change,
//       the activation scales: once per launch for gate/up, once per group for down) out as
//       tcgen05.cp source atoms (32 rows x 16 bytes per K step: byte 16 (m % 32) + 4 (m / 32) + j
//       holds row m's scale of the step's j-th 32-block), and a copier warp moves them into
//       double-buffered TMEM columns (lane = row % 32 in every sub-partition, column = row / 32,
//       byte = block) an item ahead of the MMAs, ordered by mbarriers both ways.
//   decode_mx_fused_kernel: batches of up to 16 tokens with FFN <= 2048 -- gate/up and down items
//       in one persistent launch; the gate/up epilogue writes h as its two planes and raises a
//       per-group counter that down items wait for; the scale atoms get four warps of their own.
// Weights and activation planes are read once; every wait is bounded.
#include "gemm_common.cuh"
#include "decode_common.cuh"

namespace ftmoe {

// ------------------------------------------------------------------ activation planes
// One thread per (row, 32-element block): X1 = 2^(floor(log2 amax) - 8), hi = E4M3(v / X1)
// (round to nearest even, saturating at 448), r = v - X1 * hi (exact), X2 from max|r|, lo =
// E4M3(r / X2).  A block of zeros keeps the scale 2^0.  Rows >= rows_valid are written as zero.
__device__ __forceinline__ uint32_t e8m0_of(float amax, float& X) {
    if (!(amax > 0.f)) { X = 1.f; return 127u; }
    int e = ilogbf(amax) - 8;
    e = max(-127, min(127, e));
    X = ldexpf(1.f, e);
    return uint32_t(e + 127);
}
__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
    uint16_t lo, hi;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(lo) : "f"(a), "f"(b));
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(hi) : "f"(c), "f"(d));
    return uint32_t(lo) | (uint32_t(hi) << 16);
}
__device__ __forceinline__ void e4m3x4_dec(uint32_t q, float (&o)[4]) {
    uint32_t h0, h1;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h0) : "h"(uint16_t(q & 0xFFFF)));
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h1) : "h"(uint16_t(q >> 16)));
    const __half2 a = *reinterpret_cast<const __half2*>(&h0), b = *reinterpret_cast<const __half2*>(&h1);
    o[0] = __low2float(a); o[1] = __high2float(a); o[2] = __low2float(b); o[3] = __high2float(b);
}

__global__ void __launch_bounds__(256) quant2_kernel(const uint16_t* __restrict__ src, int rows_valid, int rows, int K,
                                                     uint8_t* hi, uint8_t* lo, uint8_t* shi, uint8_t* slo) {
    pdl_wait();
    pdl_trigger();
    const int nb = K / 32;
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= rows * nb) return;
    const int r = i / nb, b = i - r * nb;
    float v[32];
    if (r < rows_valid) {
        const uint4* s = reinterpret_cast<const uint4*>(src + size_t(r) * K + 32 * b);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 u = __ldcg(s + q);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) { v[8 * q + 2 * j] = bf16lo(w[j]); v[8 * q + 2 * j + 1] = bf16hi(w[j]); }
        }
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = 0.f;
    }
    float amax = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(v[j]));
    float X1, X2;
    const uint32_t s1 = e8m0_of(amax, X1);
    const float inv1 = 1.f / X1;                         // exact: a power of two
    uint32_t qh[8];
    float res[32];
    float amax2 = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        qh[q] = e4m3x4(v[4 * q] * inv1, v[4 * q + 1] * inv1, v[4 * q + 2] * inv1, v[4 * q + 3] * inv1);
        float d[4];
        e4m3x4_dec(qh[q], d);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            res[4 * q + j] = v[4 * q + j] - d[j] * X1;   // exact: v has 8 significant bits
            amax2 = fmaxf(amax2, fabsf(res[4 * q + j]));
        }
    }
    const uint32_t s2 = e8m0_of(amax2, X2);
    const float inv2 = 1.f / X2;
    uint32_t ql[8];
#pragma unroll
    for (int q = 0; q < 8; ++q)
        ql[q] = e4m3x4(res[4 * q] * inv2, res[4 * q + 1] * inv2, res[4 * q + 2] * inv2, res[4 * q + 3] * inv2);
    uint4* dh = reinterpret_cast<uint4*>(hi + size_t(r) * K + 32 * b);
    uint4* dl = reinterpret_cast<uint4*>(lo + size_t(r) * K + 32 * b);
    dh[0] = make_uint4(qh[0], qh[1], qh[2], qh[3]);
    dh[1] = make_uint4(qh[4], qh[5], qh[6], qh[7]);
    dl[0] = make_uint4(ql[0], ql[1], ql[2], ql[3]);
    dl[1] = make_uint4(ql[4], ql[5], ql[6], ql[7]);
    shi[size_t(r) * nb + b] = uint8_t(s1);
    slo[size_t(r) * nb + b] = uint8_t(s2);
}


__device__ __forceinline__ int group_token_of(int flat, int P, int k) { return flat < P ? flat / k : flat - P; }

// ------------------------------------------------------------------ block-scaled MMA
// A stage is a 256-deep K step made of two 128-deep sub-tiles: one barrier wait and one commit per
// eight MMAs (an mbarrier poll costs the issuing thread about as much as two small MMAs).
constexpr int kDxSt = 4;                          // stages
constexpr int kDxATile = 128 * 128;               // 16 KB: 128 rows x 128 codes, one byte each (one sub-tile)
constexpr int kDxBPlane = 32 * 128;               // 4 KB: up to 32 activation rows of one plane and sub-tile
constexpr int kDxAStage = 2 * kDxATile;           // 32 KB
constexpr int kDxBSub = 2 * kDxBPlane;            // 8 KB: a sub-tile's B operand, hi rows then lo rows
constexpr int kDxBStage = 2 * kDxBSub;            // 16 KB
constexpr int kDxThreads = 224;                   // producer, MMA issuer, four epilogue / atom warps, scale copier
constexpr int kDxMaxK = 4096;                     // largest contraction (scale atoms sized for it)
constexpr int kDxSteps = kDxMaxK / 128;           // K steps per item at most
constexpr int kDxAtomBuf = 2 * kDxSteps * 512;    // 32 KB of scale atoms: weight buffers and activation atoms
constexpr int kDxTmemCols = 512;
constexpr int kDxAccCols = 64;                    // accumulator columns per buffer: N = 2 NB (hi rows, then lo rows)

__host__ __device__ constexpr size_t dec_mx_smem() {
    return 1024 + size_t(kDxSt) * (kDxAStage + kDxBStage) + size_t(kDxAtomBuf) + 512;
}

struct DecMxParams {
    int T, k, E, H, F, G, NB, m_blocks, K;
    const int32_t* offsets;
    const int32_t* sorted_flat;
    const int32_t* sched;
    const uint8_t* wsc;               // weight scales [E, rows, K/32]
    const uint8_t* bsc_hi;            // activation scales [rows, K/32], one per plane
    const uint8_t* bsc_lo;
    uint16_t* h;
    uint16_t* o;
    uint32_t* err;
    unsigned long long wait_ns;
};

// kind::mxf8f6f4 block-scaled instruction descriptor: A E2M1, B E4M3, both K-major, E8M0
// scales, M = 128; sf ids select the scale byte of the K block
__device__ __forceinline__ uint32_t idesc_mx(int N, uint32_t sfa_id, uint32_t sfb_id) {
    return (sfb_id << 4) | (5u << 7) | (0u << 10) | (uint32_t(N >> 3) << 17) | (1u << 23) | (uint32_t(128 >> 4) << 24) |
           (sfa_id << 29);
}
__device__ __forceinline__ void umma_mx(uint32_t dtm, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t tsfa,
                                        uint32_t tsfb, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(dtm), "l"(ad), "l"(bd), "r"(idesc), "r"(acc), "r"(tsfa), "r"(tsfb));
}
// 32 rows x 16 bytes of shared memory (contiguous, no swizzle) -> TMEM lanes 0..31 of four
// columns, repeated in every lane quarter.  atom_desc gives the source descriptor of the atom at
// saddr; the atom 512 bytes on is that descriptor + 32.
__device__ __forceinline__ uint64_t atom_desc(uint32_t saddr) {
    uint64_t d = uint64_t((saddr >> 4) & 0x3FFFu);
    d |= uint64_t(128 >> 4) << 16;      // leading byte offset
    d |= uint64_t(128 >> 4) << 32;      // stride byte offset: next 8 rows
    d |= uint64_t(1) << 46;
    return d;
}
__device__ __forceinline__ void tmem_cp_desc(uint32_t taddr, uint64_t d) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(d) : "memory");
}
// the bounded wait, entered only when the phase is not already complete (the common case at
// steady state costs one try_wait)
__device__ __forceinline__ bool wait_fast(uint64_t* b, uint32_t parity, volatile int* abort, unsigned long long limit) {
    return mbar_try(b, parity) || mbar_wait(b, parity, abort, limit);
}
// a bounded mbarrier wait taken by lane 0 for the whole warp (warp-uniform outcome)
__device__ __forceinline__ bool warp_wait(uint64_t* b, uint32_t parity, volatile int* abort, unsigned long long limit) {
    int r = 0;
    if ((threadIdx.x & 31) == 0) r = wait_fast(b, parity, abort, limit) ? 1 : 0;
    r = __shfl_sync(0xffffffffu, r, 0);
    __syncwarp();
    return r != 0;
}

// The eight MMAs of one 256-deep stage: two 128-deep sub-tiles of four 32-deep K blocks each
// (scale byte j of every row's step word selects block j); sfa / sfb advance one step per
// sub-tile.  acc0: the stage's first MMA accumulates (false only for an item's first stage).
__device__ __forceinline__ void dx_stage_mmas(uint32_t dacc, uint64_t ad0, uint64_t bd0, int stage,
                                              const uint32_t (&idm)[4], uint32_t& sfa, uint32_t& sfb, bool acc0) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const uint64_t ad = ad0 + uint64_t((stage * kDxAStage + u * kDxATile) >> 4);
        const uint64_t bd = bd0 + uint64_t((stage * kDxBStage + u * kDxBSub) >> 4);
        umma_mx(dacc, ad, bd, idm[0], sfa, sfb, (acc0 || u) ? 1u : 0u);
        umma_mx(dacc, ad + 2, bd + 2, idm[1], sfa + (1u << 30), sfb + (1u << 30), 1u);
        umma_mx(dacc, ad + 4, bd + 4, idm[2], sfa + (2u << 30), sfb + (2u << 30), 1u);
        umma_mx(dacc, ad + 6, bd + 6, idm[3], sfa + (3u << 30), sfb + (3u << 30), 1u);
        sfa += 4u;
        sfb += 4u;
    }
}

// This thread's accumulator lane at `tacc`: column c of the hi rows plus column NB + c of the lo
// rows into v[c], c < NB (NB = 16 or 32); waited for.
__device__ __forceinline__ void dx_acc_load(uint32_t tacc, int NB, float (&v)[32]) {
    if (NB == 32) {
        float w[32];
        tmem_ld32_nowait(tacc, v);
        tmem_ld32_nowait(tacc + 32u, w);
        tmem_wait_ld(v, w);
#pragma unroll
        for (int c = 0; c < 32; ++c) v[c] += w[c];
    } else {
        tmem_ld32_nowait(tacc, v);
        tmem_wait_16(v);
        tmem_fence_regs(v + 16);
#pragma unroll
        for (int c = 0; c < 16; ++c) v[c] += v[16 + c];
    }
}

// One A-tile row's weight scales (`ws`: nv 16-byte vectors of four 128-deep K steps each) and,
// when do_act, one B row's activation scales (`bs`; the scale 1.0 where !valid) laid out as
// tcgen05.cp source atoms: the atom of step c at c x 512 bytes, byte 16 (row % 32) + 4 (row / 32)
// + j = the row's scale of 32-block j (row = et for weights, m for activations).  Every load is in
// flight before any is used (vectors past the row's last re-read it).
__device__ __forceinline__ void dx_lay_atoms(const uint4* ws, int nv, int et, uint8_t* wdst, bool do_act,
                                             const uint4* bs, bool valid, int m, uint8_t* adst) {
    uint4 wv[kDxSteps / 4], av[kDxSteps / 4];
#pragma unroll
    for (int c4 = 0; c4 < kDxSteps / 4; ++c4) wv[c4] = __ldg(ws + min(c4, nv - 1));
    if (do_act) {
#pragma unroll
        for (int c4 = 0; c4 < kDxSteps / 4; ++c4) av[c4] = __ldcg(bs + min(c4, nv - 1));
    }
#pragma unroll
    for (int c4 = 0; c4 < kDxSteps / 4; ++c4) {
        if (c4 >= nv) break;
        const uint32_t w4[4] = {wv[c4].x, wv[c4].y, wv[c4].z, wv[c4].w};
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
            *reinterpret_cast<uint32_t*>(wdst + (4 * c4 + cc) * 512 + 16 * (et & 31) + 4 * (et >> 5)) = w4[cc];
    }
    if (do_act) {
#pragma unroll
        for (int c4 = 0; c4 < kDxSteps / 4; ++c4) {
            if (c4 >= nv) break;
            const uint4 b = valid ? av[c4] : make_uint4(0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
            const uint32_t b4[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int cc = 0; cc < 4; ++cc)
                *reinterpret_cast<uint32_t*>(adst + (4 * c4 + cc) * 512 + 16 * (m & 31) + 4 * (m >> 5)) = b4[cc];
        }
    }
}

// Where an item's scale factors live.  TMEM columns: [0, 128) the two accumulator buffers, then
// nact activation-scale buffers and two weight-scale buffers of 4 columns per 128-deep K step
// (step c of a buffer at column base + 4 c).  Shared memory (the 32 KB atom area): gate/up --
// weight atom buffers 0 and 1 at 0 and nk x 512 bytes, the activation atoms (built once) first
// in buffer 1's place; down -- the activation atoms of the current group at 0, then nwb weight
// atom buffers.
struct DxScaleLayout {
    int nk, nact, nwb;
    __device__ int act_col(int run) const { return 128 + 4 * nk * (run % nact); }
    __device__ int w_col(int j) const { return 128 + 4 * nk * (nact + (j & 1)); }
};
template <int MODE>
__device__ __forceinline__ DxScaleLayout dx_layout(int nk) {
    DxScaleLayout L;
    L.nk = nk;
    L.nact = MODE == 0 ? 1 : (128 + 16 * nk <= kDxTmemCols ? 2 : 1);
    const int atom = nk * 512;
    L.nwb = MODE == 0 ? 2 : min(2, (kDxAtomBuf - atom) / atom);
    return L;
}

// The activation operand an item reads: gate/up -- x, the same for every item; down -- its group's
// rows of h.  A change of key means new activation scales.
template <int MODE>
__device__ __forceinline__ int dx_act_key(const DecMxParams& p, int it) {
    return MODE == 0 ? 0 : p.sched[2 + (p.G + 1) + it / p.m_blocks];
}

template <int MODE>
__global__ void __launch_bounds__(kDxThreads, 1)
decode_mx_mma_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_bh,
                     const __grid_constant__ CUtensorMap tm_bl, DecMxParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = sA + kDxSt * kDxAStage;                      // [stage][sub-tile] hi rows 0..NB-1, lo rows NB..2NB-1
    uint8_t* sAtoms = sB + kDxSt * kDxBStage;                 // scale atoms (DxScaleLayout)
    uint64_t* full = reinterpret_cast<uint64_t*>(sAtoms + kDxAtomBuf);
    uint64_t* empty = full + kDxSt;
    uint64_t* tfull = empty + kDxSt;
    uint64_t* tempty = tfull + 2;
    uint64_t* atoms_full = tempty + 2;    // [weight atom buffer] an item's atoms laid out
    uint64_t* atoms_free = atoms_full + 2;// [weight atom buffer] an item's atoms copied to TMEM
    uint64_t* sf_ready = atoms_free + 2;  // [TMEM weight-scale buffer] an item's scales in TMEM
    uint64_t* mma_done = sf_ready + 2;
    uint64_t* cp_done = mma_done + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(cp_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    pdl_wait();          // routing, the activation planes and h come from the preceding kernels
    pdl_trigger();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_items = p.sched[1] * p.m_blocks;
    // a contiguous run of items per CTA: consecutive items mostly share their group, so down items
    // reuse the activation scales already in TMEM
    const int i0 = int((long long)blockIdx.x * n_items / gridDim.x);
    const int i1 = int((long long)(blockIdx.x + 1) * n_items / gridDim.x);
    const int n_my = i1 - i0;
    if (n_my <= 0) return;
    const int nk = p.K / 128;                // 128-deep K steps (scale atoms); stages cover two
    const DxScaleLayout SL = dx_layout<MODE>(nk);
    if (tid == 0) {
        for (int s = 0; s < kDxSt; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4);
            mbar_init(&atoms_full[b], 4);
            mbar_init(&atoms_free[b], 1);
            mbar_init(&sf_ready[b], 1);
        }
        mbar_init(mma_done, 1);
        mbar_init(cp_done, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(tmem_slot)),
                     "r"(kDxTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int P = p.T * p.k;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer: codes + both activation planes
        if (lane == 0) {
            // the transaction count of the unpacking code copy is its packed size (4 bits per
            // code), half of the 16 KB it fills in shared memory
            const uint32_t bytes = 2u * (uint32_t(kDxATile) / 2u + 2u * uint32_t(p.NB) * 128u);
            int step = 0, s = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int it = i0; it < i1 && ok; ++it) {
                const int slot = it / p.m_blocks, rg = it - slot * p.m_blocks;
                const int g = p.sched[2 + (p.G + 1) + slot];
                const int brow = MODE == 0 ? 0 : p.offsets[g];
                for (int kb = 0; kb < nk / 2; ++kb, ++step) {
                    if (!wait_fast(&empty[s], phase ^ 1u, abort_flag, p.wait_ns)) { ok = false; break; }
                    mbar_expect_tx(&full[s], bytes);
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int k0 = (2 * kb + u) * 128;
                        uint8_t* a = sA + s * kDxAStage + u * kDxATile;
                        if (MODE == 0) tma_5d(&tm_w, &full[s], a, k0, 0, 0, rg * 4, g);
                        else tma_3d(&tm_w, &full[s], a, k0, rg * 128, g);
                        // one B operand of 2 NB rows: the lo plane's rows follow the hi plane's (NB x
                        // 128 bytes later: a whole number of 1 KB swizzle atoms)
                        uint8_t* b = sB + s * kDxBStage + u * kDxBSub;
                        tma_2d(&tm_bh, &full[s], b, k0, brow);
                        tma_2d(&tm_bl, &full[s], b + p.NB * 128, k0, brow);
                    }
                    if (++s == kDxSt) { s = 0; phase ^= 1u; }
                }
            }
            if (!ok) { *abort_flag = 1; atomicExch(p.err, kDevErrTimeout); }
            for (int st = step - kDxSt > 0 ? step - kDxSt : 0; st < step; ++st)
                mbar_wait(&full[st % kDxSt], uint32_t(st / kDxSt) & 1u, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer: one MMA per 32-deep K block
        // At decode sizes this thread is the critical path (an MMA with N <= 64 occupies the tensor
        // pipe for only ~56 cycles), so it issues nothing but MMAs and commits: the scale factors
        // reach TMEM through the copier warp, every descriptor is computed once per launch and the
        // descriptors advance by adding (start address >> 4) offsets.
        if (lane == 0) {
            uint32_t idm[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) idm[j] = idesc_mx(2 * p.NB, uint32_t(j), uint32_t(j));
            const uint64_t ad0 = sdesc_sw128(su32(sA)), bd0 = sdesc_sw128(su32(sB));
            int stage = 0, run = -1, prev_key = -1;
            uint32_t phase = 0;
            bool ok = true;
            for (int j = 0; j < n_my && ok; ++j) {
                const int key = dx_act_key<MODE>(p, i0 + j);
                if (j == 0 || key != prev_key) ++run;
                prev_key = key;
                const int buf = j & 1;
                const uint32_t par = uint32_t(j >> 1) & 1u;
                if (!wait_fast(&sf_ready[buf], par, abort_flag, p.wait_ns)) { ok = false; break; }
                if (!wait_fast(&tempty[buf], par ^ 1u, abort_flag, p.wait_ns)) { ok = false; break; }
                tc_fence_after();
                const uint32_t dacc = tmem + uint32_t(kDxAccCols * buf);
                uint32_t sfa = tmem + uint32_t(SL.w_col(j)), sfb = tmem + uint32_t(SL.act_col(run));
                for (int kb = 0; kb < nk / 2; ++kb) {
                    // the stage's operands were all written by TMA (async proxy): its barrier's
                    // completion orders them before these MMAs, no thread-sync fence needed
                    if (!wait_fast(&full[stage], phase, abort_flag, p.wait_ns)) { ok = false; break; }
                    dx_stage_mmas(dacc, ad0, bd0, stage, idm, sfa, sfb, kb != 0);
                    umma_commit(&empty[stage]);
                    if (++stage == kDxSt) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                umma_commit(&tfull[buf]);
            }
            if (!ok) { *abort_flag = 1; atomicExch(p.err, kDevErrTimeout); }
            umma_commit(mma_done);
            mbar_wait(mma_done, 0, nullptr);
        }
    } else if (warp == 6) {
        // ------------------------------------------------ scale copier: atoms -> TMEM, ahead of the MMAs
        // Item j's weight scales go to TMEM buffer j & 1 once item j - 2 (the buffer's last reader)
        // has completed; new activation scales go to their buffer once no issued item still reads it.
        if (lane == 0) {
            const uint64_t cp0 = atom_desc(su32(sAtoms));
            const int atom_steps = nk;                 // one 512-byte atom per step: descriptor + 32 each
            int run = -1, prev_key = -1;
            bool ok = true;
            for (int j = 0; j < n_my; ++j) {
                const int key = dx_act_key<MODE>(p, i0 + j);
                const bool act_new = j == 0 || key != prev_key;
                if (act_new) ++run;
                prev_key = key;
                const int wb = j % SL.nwb;
                if (!wait_fast(&atoms_full[wb], uint32_t(j / SL.nwb) & 1u, abort_flag, p.wait_ns)) { ok = false; break; }
                if (j >= 2 && !wait_fast(&tfull[j & 1], uint32_t((j - 2) >> 1) & 1u, abort_flag, p.wait_ns)) { ok = false; break; }
                if (act_new && SL.nact == 1 && j >= 1 &&
                    !wait_fast(&tfull[(j - 1) & 1], uint32_t((j - 1) >> 1) & 1u, abort_flag, p.wait_ns)) { ok = false; break; }
                tc_fence_after();
                if (act_new) {
                    const uint64_t a0 = cp0 + uint64_t(MODE == 0 ? 32 * atom_steps : 0);
                    for (int c = 0; c < nk; ++c) tmem_cp_desc(tmem + uint32_t(SL.act_col(run) + 4 * c), a0 + uint64_t(32 * c));
                }
                const uint64_t w0 = cp0 + uint64_t(32 * atom_steps * (MODE == 0 ? wb : 1 + wb));
                for (int c = 0; c < nk; ++c) tmem_cp_desc(tmem + uint32_t(SL.w_col(j) + 4 * c), w0 + uint64_t(32 * c));
                umma_commit(&sf_ready[j & 1]);
                umma_commit(&atoms_free[wb]);
            }
            if (!ok) { *abort_flag = 1; atomicExch(p.err, kDevErrTimeout); }
            umma_commit(cp_done);
            mbar_wait(cp_done, 0, nullptr);
        }
    } else {
        // ------------------------------------------------ scale atoms, then the epilogue
        // Item j + 1's atoms are laid out as soon as its atom buffer is free, before item j's
        // epilogue.  Atom of K step c: byte 16 (m % 32) + 4 (m / 32) + jb = scale of 32-block jb of
        // row m (weights: the A-tile row; activations: B row m < 2 NB -- the hi plane's rows, then
        // the lo plane's).
        const int q = warp & 3, et = tid - 64;   // et: 0..127
        const int nsb = p.K / 32;                // scale bytes per row
        const size_t rows_e = MODE == 0 ? size_t(2) * p.F : size_t(p.H);
        const int atom = nk * 512;
        auto build_atoms = [&](int j, bool act_new) {
            const int it2 = i0 + j;
            const int slot2 = it2 / p.m_blocks, rg2 = it2 - slot2 * p.m_blocks;
            const int g2 = p.sched[2 + (p.G + 1) + slot2];
            const int r02 = p.offsets[g2], n2 = p.offsets[g2 + 1] - r02;
            const int wb = j % SL.nwb;
            uint8_t* wdst = sAtoms + (MODE == 0 ? wb : 1 + wb) * atom;
            uint8_t* adst = sAtoms + (MODE == 0 ? atom : 0);
            int wrow;     // weight row of A-tile row et (gate/up: blocks of 16 gate rows then the 16 up rows)
            if (MODE == 0) {
                const int i = et >> 5, jj = et & 31, f = rg2 * 64 + 16 * i + (jj & 15);
                wrow = jj < 16 ? f : p.F + f;
            } else {
                wrow = rg2 * 128 + et;
            }
            const int pl = et >> 5, nrow = et & 31, m = pl * p.NB + nrow;   // B row of the merged operand
            const bool do_act = act_new && et < 64 && nrow < p.NB;
            const bool valid = MODE == 0 ? nrow < p.T : nrow < n2;
            const int brow = MODE == 0 ? nrow : r02 + nrow;
            const uint8_t* bsrc = pl ? p.bsc_lo : p.bsc_hi;
            dx_lay_atoms(reinterpret_cast<const uint4*>(p.wsc + (size_t(g2) * rows_e + wrow) * nsb), nk / 4, et, wdst,
                         do_act, reinterpret_cast<const uint4*>(bsrc + size_t(valid ? brow : 0) * nsb), valid, m, adst);
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(&atoms_full[wb]);
        };
        // the wait for item x's atoms to have been copied (its buffer's phase x / nwb)
        auto copied = [&](int x) {
            return warp_wait(&atoms_free[x % SL.nwb], uint32_t(x / SL.nwb) & 1u, abort_flag, p.wait_ns);
        };
        bool ok = true;
        build_atoms(0, true);
        for (int j = 0; j < n_my; ++j) {
            const int it = i0 + j;
            const int slot = it / p.m_blocks, rg = it - slot * p.m_blocks;
            const int g = p.sched[2 + (p.G + 1) + slot];
            const int r0 = p.offsets[g], n = p.offsets[g + 1] - r0;
            if (j + 1 < n_my) {
                const bool act_new = MODE == 1 && dx_act_key<MODE>(p, it + 1) != dx_act_key<MODE>(p, it);
                // the weight buffer's previous item, the activation atoms' last copy (item j), and
                // for gate/up item 1 the activation atoms that shared buffer 1 (copied with item 0)
                if (j + 1 >= SL.nwb && !copied(j + 1 - SL.nwb)) { ok = false; break; }
                if ((act_new || (MODE == 0 && j == 0)) && !copied(j)) { ok = false; break; }
                build_atoms(j + 1, act_new);
            }
            // lane l < n stands for row r0 + l of the group; gate/up: its token
            const int my_tok = (MODE == 0 && lane < n) ? group_token_of(p.sorted_flat[r0 + lane], P, p.k) : -1;
            const int buf = j & 1;
            if (!warp_wait(&tfull[buf], uint32_t(j >> 1) & 1u, abort_flag, p.wait_ns)) { ok = false; break; }
            tc_fence_after();
            float v[32];
            dx_acc_load(tmem + (uint32_t(q * 32) << 16) + uint32_t(kDxAccCols * buf), p.NB, v);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[buf]);
            if (MODE == 0) {
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    if (c >= p.NB) break;
                    const unsigned hit = __ballot_sync(0xffffffffu, my_tok == c);
                    if (!hit) continue;
                    const int r = r0 + __ffs(hit) - 1;
                    const float other = __shfl_xor_sync(0xffffffffu, v[c], 16);
                    const float hv = silu_mul(lane < 16 ? v[c] : other, lane < 16 ? other : v[c]);
                    const uint32_t b = f2bf(hv);
                    const uint32_t pair = b | (__shfl_down_sync(0xffffffffu, b, 1) << 16);
                    if (lane < 16 && !(lane & 1))
                        *reinterpret_cast<uint32_t*>(p.h + size_t(r) * p.F + 64 * rg + 16 * q + lane) = pair;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (i < n) p.o[size_t(r0 + i) * p.H + 128 * rg + 32 * q + lane] = f2bf(v[i]);
            }
        }
        if (!ok) { *abort_flag = 1; if (lane == 0) atomicExch(p.err, kDevErrTimeout); }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kDxTmemCols));
    }
}


// ------------------------------------------------------------------ gate/up and down in one launch
// For FFN widths up to 2048 both GEMVs run as one persistent launch: CTA b takes items b,
// b + gridDim.x, ... of the list [gate/up items | down items].  The gate/up epilogue writes h
// straight as the two E4M3 planes with their E8M0 scales (the steps of quant2_kernel on the
// bf16-rounded h; the two warps that hold a 32-column block exchange their partial maxima through
// shared memory) and then raises its group's counter.  A down item's producer waits for all the
// group's gate/up epilogues before its TMA reads h, and the warps that lay out its activation
// scales wait too before they load them.  Each down item is read twice (producer, copier once its
// atoms exist): the last of the 2 x dn_blocks reads of a group leaves both counters at zero.
constexpr int kFxMaxKDn = 2048;            // largest down contraction (F) of the fused plan
// Batches of up to 16 tokens: the one launch saves the second launch's ramp and fills the
// gate/up tail (dsv4_flash T = 4 / 8: 93 -> 87 / 153 -> 146 us); at 32 tokens the strided down
// items (new activation scales for every one) and two-row gate/up epilogues cost what it saves.
constexpr int kFxMaxT = 16;
constexpr int kFxWBuf = kDxAtomBuf / 2;    // 16 KB weight-atom buffers at 0 and 16 KB
constexpr int kFxDnAct = kFxWBuf / 2;      // down items' activation atoms at 8 KB (<= 16 steps)
constexpr int kFxThreads = 352;            // producer, MMA issuer, four epilogue warps, copier, four atom builders

__host__ __device__ constexpr size_t dec_mx_fused_smem() { return dec_mx_smem() + 1024; }

struct DecMxFusedParams {
    int T, k, E, H, F, G, NB, gu_blocks, dn_blocks;
    const int32_t* offsets;
    const int32_t* sorted_flat;
    const int32_t* sched;
    const uint8_t* wsc13;        // gate/up weight scales [E, 2F, H/32]
    const uint8_t* wsc2;         // down weight scales [E, H, F/32]
    const uint8_t* xsh;          // x plane scales [32, H/32]
    const uint8_t* xsl;
    uint8_t* hh;                 // h planes [R, F] and their scales [R, F/32]
    uint8_t* hl;
    uint8_t* hsh;
    uint8_t* hsl;
    uint16_t* o;
    uint32_t* ready;             // [2G]: gate/up epilogue warps done per group, then down reads
    uint32_t* err;
    unsigned long long wait_ns;
};

struct FxItem {
    int g, rg, r0, n;
    bool down;
};
__device__ __forceinline__ FxItem fx_item(const DecMxFusedParams& p, int it, int n_gu) {
    FxItem d;
    d.down = it >= n_gu;
    const int li = d.down ? it - n_gu : it;
    const int nb = d.down ? p.dn_blocks : p.gu_blocks;
    const int slot = li / nb;
    d.rg = li - slot * nb;
    d.g = p.sched[2 + (p.G + 1) + slot];
    d.r0 = p.offsets[d.g];
    d.n = p.offsets[d.g + 1] - d.r0;
    return d;
}
__device__ __forceinline__ int fx_act_key(const FxItem& d) { return d.down ? d.g : -1; }
// one of a down item's two reads of its group's counter is done
__device__ __forceinline__ void fx_read_done(const DecMxFusedParams& p, int g) {
    if (atomicAdd(p.ready + p.G + g, 1u) == uint32_t(2 * p.dn_blocks - 1)) {
        p.ready[g] = 0u;
        p.ready[p.G + g] = 0u;
    }
}
// one thread's bounded wait for all the group's gate/up epilogue warps
__device__ __forceinline__ bool fx_group_wait(const DecMxFusedParams& p, int g, volatile int* abort_flag) {
    const uint32_t target = 4u * uint32_t(p.gu_blocks);     // four epilogue warps per gate/up item
    const unsigned long long t0 = gtimer();
    while (ld_acquire_u32(p.ready + g) < target) {
        if (*abort_flag || gtimer() - t0 > p.wait_ns) return false;
        __nanosleep(64);
    }
    return true;
}
// the same wait by a whole warp (every lane acquires; the outcome is warp-uniform)
__device__ __forceinline__ bool fx_group_wait_warp(const DecMxFusedParams& p, int g, volatile int* abort_flag) {
    const uint32_t target = 4u * uint32_t(p.gu_blocks);
    const unsigned long long t0 = gtimer();
    for (;;) {
        if (__all_sync(0xffffffffu, ld_acquire_u32(p.ready + g) >= target)) return true;
        if (__any_sync(0xffffffffu, *abort_flag != 0 || gtimer() - t0 > p.wait_ns)) return false;
        __nanosleep(64);
    }
}
__device__ __forceinline__ float warp_max(float m) {
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    return m;
}

__global__ void __launch_bounds__(kFxThreads, 1)
decode_mx_fused_kernel(const __grid_constant__ CUtensorMap tm_w13, const __grid_constant__ CUtensorMap tm_w2,
                       const __grid_constant__ CUtensorMap tm_xh, const __grid_constant__ CUtensorMap tm_xl,
                       const __grid_constant__ CUtensorMap tm_hh, const __grid_constant__ CUtensorMap tm_hl,
                       DecMxFusedParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = sA + kDxSt * kDxAStage;
    uint8_t* sAtoms = sB + kDxSt * kDxBStage;  // weight atoms [0, 16K) and [16K, 32K); x atoms at 16K; down activation atoms at 8K
    uint64_t* full = reinterpret_cast<uint64_t*>(sAtoms + kDxAtomBuf);
    uint64_t* empty = full + kDxSt;
    uint64_t* tfull = empty + kDxSt;
    uint64_t* tempty = tfull + 2;
    uint64_t* atoms_full = tempty + 2;
    uint64_t* atoms_free = atoms_full + 2;
    uint64_t* sf_ready = atoms_free + 2;
    uint64_t* mma_done = sf_ready + 2;
    uint64_t* cp_done = mma_done + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(cp_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    uint64_t* pair_bar = reinterpret_cast<uint64_t*>(tmem_slot + 2);     // [pair of epilogue warps]
    float* xch = reinterpret_cast<float*>(sAtoms + kDxAtomBuf + 512);   // [pair][round][half][32 rows] partial maxima

    pdl_wait();          // routing and the x planes come from the preceding kernels
    pdl_trigger();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_gu = p.sched[1] * p.gu_blocks;
    const int n_items = n_gu + p.sched[1] * p.dn_blocks;
    if (int(blockIdx.x) >= n_items) return;
    const int n_my = (n_items - int(blockIdx.x) + int(gridDim.x) - 1) / int(gridDim.x);
    const int nk_gu = p.H / 128, nk_dn = p.F / 128, nk_max = max(nk_gu, nk_dn);
    // TMEM: accumulators [0, 128); x scales at 128 or the two down activation-scale buffers at
    // 128 + 4 nk_dn a; weight-scale buffers at wbase + 4 nk_max b
    const int wbase = 128 + 4 * max(nk_gu, 2 * nk_dn);
    if (tid == 0) {
        for (int s = 0; s < kDxSt; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4);
            mbar_init(&atoms_full[b], 4);
            mbar_init(&atoms_free[b], 1);
            mbar_init(&sf_ready[b], 1);
        }
        mbar_init(mma_done, 1);
        mbar_init(cp_done, 1);
        mbar_init(&pair_bar[0], 2);
        mbar_init(&pair_bar[1], 2);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(tmem_slot)),
                     "r"(kDxTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int P = p.T * p.k;
    auto item = [&](int j) { return fx_item(p, int(blockIdx.x) + j * int(gridDim.x), n_gu); };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer: codes + both activation planes
        if (lane == 0) {
            const uint32_t bytes = 2u * (uint32_t(kDxATile) / 2u + 2u * uint32_t(p.NB) * 128u);
            int s = 0;
            long step = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int j = 0; j < n_my && ok; ++j) {
                const FxItem d = item(j);
                if (d.down) {
                    // every h row of the group written before the first B load
                    if (!fx_group_wait(p, d.g, abort_flag)) { ok = false; break; }
                    asm volatile("fence.proxy.async.global;" ::: "memory");   // h (generic writes) -> TMA reads
                    fx_read_done(p, d.g);
                }
                const int nk = d.down ? nk_dn : nk_gu;
                const int brow = d.down ? d.r0 : 0;
                for (int kb = 0; kb < nk / 2; ++kb, ++step) {
                    if (!wait_fast(&empty[s], phase ^ 1u, abort_flag, p.wait_ns)) { ok = false; break; }
                    mbar_expect_tx(&full[s], bytes);
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int k0 = (2 * kb + u) * 128;
                        uint8_t* a = sA + s * kDxAStage + u * kDxATile;
                        if (d.down) tma_3d(&tm_w2, &full[s], a, k0, d.rg * 128, d.g);
                        else tma_5d(&tm_w13, &full[s], a, k0, 0, 0, d.rg * 4, d.g);
                        uint8_t* b = sB + s * kDxBStage + u * kDxBSub;
                        tma_2d(d.down ? &tm_hh : &tm_xh, &full[s], b, k0, brow);
                        tma_2d(d.down ? &tm_hl : &tm_xl, &full[s], b + p.NB * 128, k0, brow);
                    }
                    if (++s == kDxSt) { s = 0; phase ^= 1u; }
                }
            }
            if (!ok) { *abort_flag = 1; atomicExch(p.err, kDevErrTimeout); }
            for (long st = step - kDxSt > 0 ? step - kDxSt : 0; st < step; ++st)
                mbar_wait(&full[st % kDxSt], uint32_t(st / kDxSt) & 1u, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer: MMAs and commits only
        if (lane == 0) {
            uint32_t idm[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) idm[j] = idesc_mx(2 * p.NB, uint32_t(j), uint32_t(j));
            const uint64_t ad0 = sdesc_sw128(su32(sA)), bd0 = sdesc_sw128(su32(sB));
            int stage = 0, drun = -1, prev_key = -2;
            uint32_t phase = 0;
            bool ok = true;
            for (int j = 0; j < n_my && ok; ++j) {
                const FxItem d = item(j);
                const int key = fx_act_key(d);
                if (d.down && key != prev_key) ++drun;
                prev_key = key;
                const int buf = j & 1;
                const uint32_t par = uint32_t(j >> 1) & 1u;
                if (!wait_fast(&sf_ready[buf], par, abort_flag, p.wait_ns)) { ok = false; break; }
                if (!wait_fast(&tempty[buf], par ^ 1u, abort_flag, p.wait_ns)) { ok = false; break; }
                tc_fence_after();
                const uint32_t dacc = tmem + uint32_t(kDxAccCols * buf);
                uint32_t sfa = tmem + uint32_t(wbase + 4 * nk_max * buf);
                uint32_t sfb = tmem + uint32_t(d.down ? 128 + 4 * nk_dn * (drun & 1) : 128);
                const int nk = d.down ? nk_dn : nk_gu;
                for (int kb = 0; kb < nk / 2; ++kb) {
                    if (!wait_fast(&full[stage], phase, abort_flag, p.wait_ns)) { ok = false; break; }
                    dx_stage_mmas(dacc, ad0, bd0, stage, idm, sfa, sfb, kb != 0);
                    umma_commit(&empty[stage]);
                    if (++stage == kDxSt) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                umma_commit(&tfull[buf]);
            }
            if (!ok) { *abort_flag = 1; atomicExch(p.err, kDevErrTimeout); }
            umma_commit(mma_done);
            mbar_wait(mma_done, 0, nullptr);
        }
    } else if (warp == 6) {
        // ------------------------------------------------ scale copier
        // Weight scales to buffer j & 1 once item j - 2 completed; activation scales when they
        // change -- the down buffers overlap the x scales, so the first down item waits for the
        // item before it.
        if (lane == 0) {
            const uint64_t cp0 = atom_desc(su32(sAtoms));
            int drun = -1, prev_key = -2;
            bool ok = true;
            for (int j = 0; j < n_my; ++j) {
                const FxItem d = item(j);
                const int key = fx_act_key(d);
                const bool act_new = key != prev_key;
                const bool first_down = d.down && j > 0 && prev_key == -1;
                if (d.down && act_new) ++drun;
                prev_key = key;
                const int wb = j & 1;
                if (!wait_fast(&atoms_full[wb], uint32_t(j >> 1) & 1u, abort_flag, p.wait_ns)) { ok = false; break; }
                if (d.down) fx_read_done(p, d.g);    // the item's activation scales (if any) are loaded
                if (j >= 2 && !wait_fast(&tfull[wb], uint32_t((j - 2) >> 1) & 1u, abort_flag, p.wait_ns)) { ok = false; break; }
                if (first_down && !wait_fast(&tfull[(j - 1) & 1], uint32_t((j - 1) >> 1) & 1u, abort_flag, p.wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int nk = d.down ? nk_dn : nk_gu;
                if (act_new) {
                    const uint32_t acol = d.down ? uint32_t(128 + 4 * nk_dn * (drun & 1)) : 128u;
                    const uint64_t a0 = cp0 + uint64_t((d.down ? kFxDnAct : kFxWBuf) >> 4);
                    for (int c = 0; c < nk; ++c) tmem_cp_desc(tmem + acol + uint32_t(4 * c), a0 + uint64_t(32 * c));
                }
                const uint64_t w0 = cp0 + uint64_t((wb * kFxWBuf) >> 4);
                const uint32_t wcol = uint32_t(wbase + 4 * nk_max * wb);
                for (int c = 0; c < nk; ++c) tmem_cp_desc(tmem + wcol + uint32_t(4 * c), w0 + uint64_t(32 * c));
                umma_commit(&sf_ready[wb]);
                umma_commit(&atoms_free[wb]);
            }
            if (!ok) { *abort_flag = 1; atomicExch(p.err, kDevErrTimeout); }
            umma_commit(cp_done);
            mbar_wait(cp_done, 0, nullptr);
        }
    } else if (warp >= 7) {
        // ------------------------------------------------ scale atoms (thread et: A-tile row et)
        // Item j's atoms go to buffer j & 1 once item j - 2's were copied (item 1: once item 0's,
        // whose x atoms sat in buffer 1; new down activation atoms: once item j - 1's).  These
        // warps run ahead of the epilogues, so a down item's wait for its group's h never holds
        // up the gate/up epilogues that produce it.
        const int et = tid - 224;                // 0..127
        const bool act_warp = et < 64;           // these load activation scales
        auto copied = [&](int x) { return warp_wait(&atoms_free[x & 1], uint32_t(x >> 1) & 1u, abort_flag, p.wait_ns); };
        bool ok = true;
        int prev_key = -2;
        for (int j = 0; j < n_my; ++j) {
            const FxItem d = item(j);
            const int key = fx_act_key(d);
            const bool act_new = key != prev_key;
            prev_key = key;
            if (j >= 2 && !copied(j - 2)) { ok = false; break; }
            if (j == 1 && !item(0).down && !copied(0)) { ok = false; break; }
            if (j >= 1 && act_new && d.down && !copied(j - 1)) { ok = false; break; }
            if (act_new && d.down && act_warp && !fx_group_wait_warp(p, d.g, abort_flag)) { ok = false; break; }
            const int nk = d.down ? nk_dn : nk_gu;
            const int nsb = 4 * nk;              // scale bytes per row
            uint8_t* wdst = sAtoms + (j & 1) * kFxWBuf;
            uint8_t* adst = sAtoms + (d.down ? kFxDnAct : kFxWBuf);
            int wrow;
            if (!d.down) {
                const int i = et >> 5, jj = et & 31, fr = d.rg * 64 + 16 * i + (jj & 15);
                wrow = jj < 16 ? fr : p.F + fr;
            } else {
                wrow = d.rg * 128 + et;
            }
            const uint8_t* wsc = d.down ? p.wsc2 + (size_t(d.g) * p.H + wrow) * nsb
                                        : p.wsc13 + (size_t(d.g) * 2 * p.F + wrow) * nsb;
            const int pl = et >> 5, nrow = et & 31, m = pl * p.NB + nrow;   // B row of the merged operand
            const bool do_act = act_new && act_warp && nrow < p.NB;
            const bool valid = d.down ? nrow < d.n : nrow < p.T;
            const int brow = d.down ? d.r0 + nrow : nrow;
            const uint8_t* bsrc = d.down ? (pl ? p.hsl : p.hsh) : (pl ? p.xsl : p.xsh);
            dx_lay_atoms(reinterpret_cast<const uint4*>(wsc), nk / 4, et, wdst, do_act,
                         reinterpret_cast<const uint4*>(bsrc + size_t(valid ? brow : 0) * nsb), valid, m, adst);
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(&atoms_full[j & 1]);
        }
        if (!ok) { *abort_flag = 1; if (lane == 0) atomicExch(p.err, kDevErrTimeout); }
    } else {
        // ------------------------------------------------ epilogue warps 2..5 (TMEM lane quarter q)
        const int q = warp & 3;
        // the two warps of a 32-column h block meet on their pair's barrier (two arrivals a phase)
        const int pr = q >> 1, hf = q & 1;
        int ps = 0;
        auto pair_sync = [&]() {
            __syncwarp();
            if (lane == 0) mbar_arrive(&pair_bar[pr]);
            const bool r = warp_wait(&pair_bar[pr], uint32_t(ps & 1), abort_flag, p.wait_ns);
            ++ps;
            return r;
        };
        bool ok = true;
        for (int j = 0; j < n_my && ok; ++j) {
            const FxItem d = item(j);
            const int my_tok = (!d.down && lane < d.n) ? group_token_of(p.sorted_flat[d.r0 + lane], P, p.k) : -1;
            const int buf = j & 1;
            if (!warp_wait(&tfull[buf], uint32_t(j >> 1) & 1u, abort_flag, p.wait_ns)) { ok = false; break; }
            tc_fence_after();
            const uint32_t tacc = tmem + (uint32_t(q * 32) << 16) + uint32_t(kDxAccCols * buf);
            if (d.down) {
                float v[32];
                dx_acc_load(tacc, p.NB, v);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[buf]);
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (i < d.n) p.o[size_t(d.r0 + i) * p.H + 128 * d.rg + 32 * q + lane] = f2bf(v[i]);
            } else {
                // One group row (token) at a time: its accumulator column read straight from TMEM.
                // Lanes < 16: h at column f = 64 rg + 16 q + lane (gate row lane, up row lane + 16);
                // warps q = 2 pr, 2 pr + 1 hold 32-column block pr.  Each writes its partial max|h|,
                // meets its partner, forms the block's first scale and plane, writes its partial
                // max|h - hi|, meets again, and stores both planes (slot rl of each array is this
                // row's; the next item writes them only after both warps passed the last meeting).
                float* x1 = xch + pr * 128;        // [half][row] partial max|h|
                float* x2 = x1 + 64;               // [half][row] partial max|h - hi|
                const int f = 64 * d.rg + 16 * q + lane;
                for (int rl = 0; rl < d.n; ++rl) {
                    const int c = __shfl_sync(0xffffffffu, my_tok, rl);
                    float ah, al;
                    tmem_ld1x2(tacc + uint32_t(c), tacc + uint32_t(p.NB + c), ah, al);
                    const float acc = ah + al;
                    const float other = __shfl_xor_sync(0xffffffffu, acc, 16);
                    const float hv = lane < 16 ? bf16lo(uint32_t(f2bf(silu_mul(acc, other)))) : 0.f;
                    const float m1 = warp_max(fabsf(hv));
                    if (lane == 0) x1[hf * 32 + rl] = m1;
                    if (!pair_sync()) { ok = false; break; }
                    float X1, X2, d4[4];
                    const uint32_t s1 = e8m0_of(fmaxf(x1[rl], x1[32 + rl]), X1);
                    const uint32_t hi = e4m3x4(hv * (1.f / X1), 0.f, 0.f, 0.f) & 0xFFu;
                    e4m3x4_dec(hi, d4);
                    const float res = hv - d4[0] * X1;
                    const float m2 = warp_max(lane < 16 ? fabsf(res) : 0.f);
                    if (lane == 0) x2[hf * 32 + rl] = m2;
                    if (!pair_sync()) { ok = false; break; }
                    const uint32_t s2 = e8m0_of(fmaxf(x2[rl], x2[32 + rl]), X2);
                    const uint32_t lo = e4m3x4(res * (1.f / X2), 0.f, 0.f, 0.f) & 0xFFu;
                    const int r = d.r0 + rl;
                    if (lane < 16) {
                        p.hh[size_t(r) * p.F + f] = uint8_t(hi);
                        p.hl[size_t(r) * p.F + f] = uint8_t(lo);
                    }
                    if (hf == 0 && lane == 0) {
                        p.hsh[size_t(r) * (p.F / 32) + 2 * d.rg + pr] = uint8_t(s1);
                        p.hsl[size_t(r) * (p.F / 32) + 2 * d.rg + pr] = uint8_t(s2);
                    }
                }
                if (!ok) break;
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[buf]);
                __threadfence();
                __syncwarp();
                if (lane == 0) atomicAdd(p.ready + d.g, 1u);
            }
        }
        if (!ok) { *abort_flag = 1; if (lane == 0) atomicExch(p.err, kDevErrTimeout); }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kDxTmemCols));
    }
}


// ------------------------------------------------------------------ host side
bool decode_mx_eligible(const DecodeArgs& a) {
    return a.wdtype == FT_W_MXFP4 && !a.eptr && !a.S && a.T >= 1 && a.T <= 32 && a.H % 512 == 0 && a.F % 512 == 0 &&
           a.H <= kDxMaxK && a.F <= kDxMaxK;
}

bool decode_mx_fused(const DecodeArgs& a) { return a.F <= kFxMaxKDn && a.T <= kFxMaxT; }

template <typename... KArgs, typename... Args>
static cudaError_t launch_dep(void (*kern)(KArgs...), int grid, int block, size_t smem, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

static bool plane_map(CUtensorMap* m, const void* base, int K, int rows, int NB) {
    uint64_t d[2] = {uint64_t(K), uint64_t(rows)}, s[1] = {uint64_t(K)};
    uint32_t b[2] = {128, uint32_t(NB)};
    return make_map(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, 2, d, s, b);
}

cudaError_t launch_decode_mx(const DecodeArgs& a, cudaStream_t st) {
    const int T = a.T, H = a.H, F = a.F, E = a.E, k = a.k;
    const int R = T * k, G = E;
    const int na_max = R < G ? R : G;
    const int NB = T <= 16 ? 16 : 32;
    // scratch: x planes [32, H] x 2 + scales, h planes [R, F] x 2 + scales (256-byte aligned parts)
    uint8_t* q = a.mx_ws;
    auto take = [&](size_t bytes) { uint8_t* r = q; q += (bytes + 255) & ~size_t(255); return r; };
    uint8_t* xh = take(32 * size_t(H));
    uint8_t* xl = take(32 * size_t(H));
    uint8_t* xsh = take(32 * size_t(H) / 32);
    uint8_t* xsl = take(32 * size_t(H) / 32);
    uint8_t* hh = take(size_t(R) * F);
    uint8_t* hl = take(size_t(R) * F);
    uint8_t* hsh = take(size_t(R) * F / 32);
    uint8_t* hsl = take(size_t(R) * F / 32);

    DecMxParams p{};
    p.T = T; p.k = k; p.E = E; p.H = H; p.F = F; p.G = G; p.NB = NB;
    p.offsets = a.offsets;
    p.sorted_flat = a.sorted_flat;
    p.sched = a.sched;
    p.h = a.h;
    p.o = a.y ? a.o_ws : a.o_sorted;
    p.err = a.err;
    p.wait_ns = gemm_wait_ns();

    CUtensorMap gw{}, dw{}, gbh{}, gbl{}, dbh{}, dbl{};
    {   // codes unpacked to a byte per element by TMA; gate/up as (H, 16, 2, F/16, E) blocks of 16 gate + 16 up rows
        uint64_t dims[5] = {uint64_t(H), 16, 2, uint64_t(F / 16), uint64_t(E)};
        uint64_t str[4] = {uint64_t(H) / 2, uint64_t(F) * H / 2, uint64_t(16) * H / 2, uint64_t(2) * F * H / 2};
        uint32_t box[5] = {128, 16, 2, 4, 1};
        if (!make_map(&gw, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, a.w13, 5, dims, str, box)) return cudaErrorInvalidValue;
        uint64_t d3[3] = {uint64_t(F), uint64_t(H), uint64_t(E)};
        uint64_t s3[2] = {uint64_t(F) / 2, uint64_t(H) * F / 2};
        uint32_t b3[3] = {128, 128, 1};
        if (!make_map(&dw, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, a.w2, 3, d3, s3, b3)) return cudaErrorInvalidValue;
    }
    if (!plane_map(&gbh, xh, H, 32, NB) || !plane_map(&gbl, xl, H, 32, NB) || !plane_map(&dbh, hh, F, R, NB) ||
        !plane_map(&dbl, hl, F, R, NB))
        return cudaErrorInvalidValue;
    if (decode_mx_fused(a)) {
        // x planes, then gate/up and down in one persistent launch (h planes written by its epilogue)
        constexpr size_t fsmem = dec_mx_fused_smem();
        static PerDeviceOnce fattr;
        {
            const cudaError_t e = fattr([&] {
                return cudaFuncSetAttribute(decode_mx_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(fsmem));
            });
            if (e != cudaSuccess) return e;
        }
        DecMxFusedParams f{};
        f.T = T; f.k = k; f.E = E; f.H = H; f.F = F; f.G = G; f.NB = NB;
        f.gu_blocks = F / 64;
        f.dn_blocks = H / 128;
        f.offsets = a.offsets;
        f.sorted_flat = a.sorted_flat;
        f.sched = a.sched;
        f.wsc13 = a.w13s;
        f.wsc2 = a.w2s;
        f.xsh = xsh; f.xsl = xsl;
        f.hh = hh; f.hl = hl; f.hsh = hsh; f.hsl = hsl;
        f.o = p.o;
        f.ready = a.err + kWsReady;
        f.err = a.err;
        f.wait_ns = p.wait_ns;
        const int items = na_max * (f.gu_blocks + f.dn_blocks);
        cudaError_t e = launch_dep(quant2_kernel, (32 * (H / 32) + 255) / 256, 256, 0, st, a.x, T, 32, H, xh, xl, xsh, xsl);
        if (e != cudaSuccess) return e;
        e = launch_dep(decode_mx_fused_kernel, items < num_sms() ? items : num_sms(), kFxThreads, fsmem, st, gw, dw, gbh,
                       gbl, dbh, dbl, f);
        if (e != cudaSuccess) return e;
        if (a.y) e = launch_combine_dependent(T, H, k, 0, R, a.o_ws, a.inv_pos, a.topk_w, a.y, st);
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
    }
    constexpr size_t smem = dec_mx_smem();
    static PerDeviceOnce attr;
    {
        const cudaError_t e = attr([&] {
            cudaError_t r = cudaFuncSetAttribute(decode_mx_mma_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
            if (r == cudaSuccess)
                r = cudaFuncSetAttribute(decode_mx_mma_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
            return r;
        });
        if (e != cudaSuccess) return e;
    }
    const int cap = num_sms();            // persistent: one CTA per SM (ring and scale atoms fill shared memory)
    cudaError_t e = launch_dep(quant2_kernel, (32 * (H / 32) + 255) / 256, 256, 0, st, a.x, T, 32, H, xh, xl, xsh, xsl);
    if (e != cudaSuccess) return e;
    p.K = H;
    p.m_blocks = F / 64;
    p.wsc = a.w13s;
    p.bsc_hi = xsh;
    p.bsc_lo = xsl;
    e = launch_dep(decode_mx_mma_kernel<0>, na_max * p.m_blocks < cap ? na_max * p.m_blocks : cap, kDxThreads, smem, st,
                   gw, gbh, gbl, p);
    if (e != cudaSuccess) return e;
    e = launch_dep(quant2_kernel, (R * (F / 32) + 255) / 256, 256, 0, st, static_cast<const uint16_t*>(a.h), R, R, F, hh,
                   hl, hsh, hsl);
    if (e != cudaSuccess) return e;
    p.K = F;
    p.m_blocks = H / 128;
    p.wsc = a.w2s;
    p.bsc_hi = hsh;
    p.bsc_lo = hsl;
    e = launch_dep(decode_mx_mma_kernel<1>, na_max * p.m_blocks < cap ? na_max * p.m_blocks : cap, kDxThreads, smem, st,
                   dw, dbh, dbl, p);
    if (e != cudaSuccess) return e;
    if (a.y) e = launch_combine_dependent(T, H, k, 0, R, a.o_ws, a.inv_pos, a.topk_w, a.y, st);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace ftmoe

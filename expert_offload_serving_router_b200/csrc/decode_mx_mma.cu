// Steps 3/4 (decode, MXFP4 weights) on the block-scaled tensor cores.
//
// The MXFP4 GEMVs are bound by decoding E2M1 codes on the ALUs.  Here the tensor core takes the
// codes as they are: tcgen05.mma.kind::mxf8f6f4.block_scale multiplies E2M1 weights (A, with
// their E8M0 scale per 32 elements) by E4M3 activations (B, with E8M0 scales).  A single E4M3
// copy of the activations loses too much (the error study: 5.6e-2 of max|y| on the
// DeepSeek-V4-Flash-shaped layer, over the 3e-2 tolerance), so each activation row is carried as
// two planes -- hi = the OCP MX conversion of v, lo = the same conversion of v - hi, each with its
// own E8M0 scale per 32 (1.2e-3 of max|y| in the study) -- and every K step issues one MMA per
// plane into the same fp32 accumulator.
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
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const uint64_t ad = ad0 + uint64_t((stage * kDxAStage + u * kDxATile) >> 4);
                        const uint64_t bd = bd0 + uint64_t((stage * kDxBStage + u * kDxBSub) >> 4);
                        // the four 32-deep K blocks of the sub-tile (scale byte j of each row's step word)
                        umma_mx(dacc, ad, bd, idm[0], sfa, sfb, (kb | u) != 0);
                        umma_mx(dacc, ad + 2, bd + 2, idm[1], sfa + (1u << 30), sfb + (1u << 30), 1u);
                        umma_mx(dacc, ad + 4, bd + 4, idm[2], sfa + (2u << 30), sfb + (2u << 30), 1u);
                        umma_mx(dacc, ad + 6, bd + 6, idm[3], sfa + (3u << 30), sfb + (3u << 30), 1u);
                        sfa += 4u;
                        sfb += 4u;
                    }
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
            // a row's scales arrive as 16-byte vectors (four K steps each), all loads in flight:
            // issued unconditionally (vectors past the row's last re-read it) so none waits on a branch
            const uint4* ws = reinterpret_cast<const uint4*>(p.wsc + (size_t(g2) * rows_e + wrow) * nsb);
            const int nv = nk / 4;
            uint4 wv[kDxSteps / 4];
#pragma unroll
            for (int c4 = 0; c4 < kDxSteps / 4; ++c4) wv[c4] = __ldg(ws + min(c4, nv - 1));
#pragma unroll
            for (int c4 = 0; c4 < kDxSteps / 4; ++c4) {
                if (c4 >= nv) break;
                const uint32_t w4[4] = {wv[c4].x, wv[c4].y, wv[c4].z, wv[c4].w};
#pragma unroll
                for (int cc = 0; cc < 4; ++cc)
                    *reinterpret_cast<uint32_t*>(wdst + (4 * c4 + cc) * 512 + 16 * (et & 31) + 4 * (et >> 5)) = w4[cc];
            }
            if (act_new && et < 64 && (et & 31) < p.NB) {
                const int pl = et >> 5, nrow = et & 31, m = pl * p.NB + nrow;   // B row of the merged operand
                const uint8_t* bsrc = pl ? p.bsc_lo : p.bsc_hi;
                const int brow = MODE == 0 ? nrow : r02 + nrow;
                const bool valid = MODE == 0 ? nrow < p.T : nrow < n2;
                const uint4* bs = reinterpret_cast<const uint4*>(bsrc + size_t(valid ? brow : 0) * nsb);
#pragma unroll
                for (int c4 = 0; c4 < kDxSteps / 4; ++c4) wv[c4] = __ldcg(bs + min(c4, nv - 1));
#pragma unroll
                for (int c4 = 0; c4 < kDxSteps / 4; ++c4) {
                    if (c4 >= nv) break;
                    const uint4 b = valid ? wv[c4] : make_uint4(0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
                    const uint32_t b4[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc)
                        *reinterpret_cast<uint32_t*>(adst + (4 * c4 + cc) * 512 + 16 * (m & 31) + 4 * (m >> 5)) = b4[cc];
                }
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(&atoms_full[wb]);
        };
        // the wait for item x's atoms to have been copied (its buffer's phase x / nwb)
        auto copied = [&](int x) {
            return wait_fast(&atoms_free[x % SL.nwb], uint32_t(x / SL.nwb) & 1u, abort_flag, p.wait_ns);
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
            if (!mbar_wait(&tfull[buf], uint32_t(j >> 1) & 1u, abort_flag, p.wait_ns)) { ok = false; break; }
            tc_fence_after();
            float v[32];
            // column c of the hi rows plus column NB + c of the lo rows
            const uint32_t tacc = tmem + (uint32_t(q * 32) << 16) + uint32_t(kDxAccCols * buf);
            if (p.NB == 32) {
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


// ------------------------------------------------------------------ host side
bool decode_mx_eligible(const DecodeArgs& a) {
    return a.wdtype == FT_W_MXFP4 && !a.eptr && !a.S && a.T >= 1 && a.T <= 32 && a.H % 512 == 0 && a.F % 512 == 0 &&
           a.H <= kDxMaxK && a.F <= kDxMaxK;
}

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
    constexpr size_t smem = dec_mx_smem();
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(decode_mx_mma_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(decode_mx_mma_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return e;
        attr = true;
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

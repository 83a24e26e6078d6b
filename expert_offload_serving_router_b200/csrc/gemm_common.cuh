// Pieces shared by the grouped expert GEMM kernels (BF16 and MXFP4 weights): tile sizes,
// launch parameters, the exact MXFP4 -> bf16 decoder, the device-side tile schedule and the
// TMEM -> global epilogue (SwiGLU for gate/up).
#pragma once
#include "sm100.cuh"

namespace ftmoe {

constexpr int kBK = 64;                        // K per stage (one 128-byte swizzle atom of bf16)
constexpr int kAHalfBytes = 128 * kBK * 2;     // 16 KB: one 128-row MMA operand
constexpr int kBTileBytes = kGemmBN * kBK * 2; // 32 KB: up to 256 token rows
constexpr int kAccCols = 256;                  // one accumulator = 128 lanes x 256 fp32 columns
constexpr int kNumBMaps = 5;                   // activation boxes of 16, 32, 64, 128, 256 rows
constexpr int kXposeBytes = 2048;              // per epilogue warp: 32 tokens x 32 bf16

struct GemmParams {
    int mode;               // 0 gate/up, 1 down
    int K;                  // H or F
    int m_tiles;            // weight-row tiles: ceil(m_rows / HV)
    int m_rows;             // 128-row weight groups: F/64 (gate/up, 64 gate + 64 up rows) or H/128 (down)
    int G, E, F, H;
    int has_shared;
    const int32_t* offsets; // [G+1]
    const int32_t* sched;   // [0] n-tiles, [2..2+G] ntile_off
    uint16_t* out;          // h [R,F] or o_sorted [R,H]
    int out_ld;
    uint32_t* err;
    int b_rows[kNumBMaps];  // rows of activation box i (16 << i, clamped to round_up(R, 16))
    // MXFP4 weights (A operand built by converter warps)
    const uint8_t* wq;      // routed codes  [E, rows, K/2]
    const uint8_t* ws;      // routed scales [E, rows, K/32]
    const uint8_t* swq;     // shared codes  [1, rows, K/2]
    const uint8_t* sws;     // shared scales
    unsigned long long wait_ns;   // bound on each pipeline wait (ns without progress)
};

// ------------------------------------------------------------------ exact MXFP4 -> bf16
// Eight E2M1 codes (byte i: element 2i in the low nibble, 2i+1 in the high nibble) to four
// bf16x2 words, scaled by the block's E8M0 scale.  Magnitudes {0,.5,1,1.5,2,3,4,6} are
// looked up with byte permutes (bf16 high / low bytes), the sign bit is moved in, and the
// power-of-two scale multiply is exact in bf16.
__device__ __forceinline__ void e2m1x8_bf16(uint32_t w, uint32_t scale2, uint32_t (&o)[4]) {
    const uint32_t HB_LO = 0x3F3F3F00u, HB_HI = 0x40404040u;
    const uint32_t LB_LO = 0xC0800000u, LB_HI = 0xC0804000u;
    const uint32_t mag = w & 0x77777777u;
    const uint32_t hb0 = __byte_perm(HB_LO, HB_HI, mag);
    const uint32_t lb0 = __byte_perm(LB_LO, LB_HI, mag);
    const uint32_t hb1 = __byte_perm(HB_LO, HB_HI, mag >> 16);
    const uint32_t lb1 = __byte_perm(LB_LO, LB_HI, mag >> 16);
    const uint32_t s_lo = (w << 4) & 0x80808080u;
    const uint32_t s_hi = w & 0x80808080u;
    uint32_t v[4];
    v[0] = __byte_perm(lb0, hb0, 0x5140);
    v[1] = __byte_perm(lb0, hb0, 0x7362);
    v[2] = __byte_perm(lb1, hb1, 0x5140);
    v[3] = __byte_perm(lb1, hb1, 0x7362);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t sg = __byte_perm(s_lo, s_hi, 0x4000u + 0x1111u * i) & 0x80008000u;
        uint32_t x = v[i] | sg;
        asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(o[i]) : "r"(x), "r"(scale2));
    }
}
// The same eight codes by bit placement: the three magnitude bits of a code moved to bf16 bits
// 6..8 and its sign to bit 15 form exactly E2M1(code) * 2^-126 (code magnitude 1 -> the bf16
// subnormal 2^-127; e = 1..3 -> normals), so one exact multiply by 2^(s - 1) gives
// E2M1 * 2^(s - 127).  Valid for scale bytes s <= 128 (2^(s - 1) must be a finite bf16);
// scale2m1 = bf16x2 of 2^(s - 1).  Per output word: one byte permute pairs codes 2i (low half)
// and 2i+1 (high half) with zero bytes around them, a shift places the magnitude, one
// multiply-add moves the sign from bit 9 to bit 15 (adds sign * (2^15 - 2^9)).
__device__ __forceinline__ void e2m1x8_bf16_place(uint32_t w, uint32_t scale2m1, uint32_t (&o)[4]) {
    const uint32_t lo = w & 0x0F0F0F0Fu;           // codes 0, 2, 4, 6 (one per byte)
    const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;    // codes 1, 3, 5, 7
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        // bytes: lo.byte i, 0, hi.byte i, 0 (a selector with its top bit set replicates the sign
        // of the selected byte, < 0x80 here, so it yields 0; __byte_perm would drop that bit)
        uint32_t pr;
        asm("prmt.b32 %0, %1, %2, %3;" : "=r"(pr) : "r"(lo), "r"(hi), "r"(0x8080u | uint32_t(i) | (uint32_t(4 + i) << 8)));
        const uint32_t v = (pr << 6) + (pr & 0x00080008u) * 0xFC0u;
        asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(o[i]) : "r"(v), "r"(scale2m1));
    }
}
// bf16x2 of 2^(s - 1) for the bit-placement decode (s <= 128)
__device__ __forceinline__ uint32_t e8m0_place_bf16x2(uint32_t s) {
    const uint32_t b = (s + 126u) << 7;
    return b | (b << 16);
}
__device__ __forceinline__ uint32_t e8m0_bf16x2(uint32_t s) {
    uint32_t b = s == 0 ? 0x0040u : (s == 255 ? 0x7FC0u : (s << 7));
    return b | (b << 16);
}

// ------------------------------------------------------------------ tile schedule
struct Tile { int g, m, row0, nvalid, halves; };

// HV = 128-row weight halves per tile.  Tile t -> (group g, weight-row tile m, token tile)
// with m fastest, so the CTAs that share a token tile run together (L2 reuse).
template <int HV>
__device__ __forceinline__ Tile decode_tile(int t, const int* ntile_off, int G, const int* offsets, int m_tiles,
                                            int m_rows) {
    Tile r;
    int u = t / m_tiles;
    r.m = t - u * m_tiles;
    int lo = 0, hi = G;   // largest g with ntile_off[g] <= u
    while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if (ntile_off[mid] <= u) lo = mid; else hi = mid;
    }
    r.g = lo;
    int ni = u - ntile_off[lo];
    r.row0 = offsets[lo] + ni * kGemmBN;
    r.nvalid = min(kGemmBN, offsets[lo + 1] - r.row0);
    r.halves = min(HV, m_rows - HV * r.m);   // the last weight-row tile may hold fewer halves
    return r;
}

__device__ __forceinline__ int bmap_index(int n) {   // smallest box of 16 << i rows holding n rows
    int i = 0;
    while (i < kNumBMaps - 1 && (16 << i) < n) ++i;
    return i;
}

// Epilogue of one tile for one warp: TMEM lanes 32q..32q+31 (tbase already includes them
// and the accumulator buffer), accumulator half hh at column hh * kAccCols, weight-row group
// rg_base + rg_step * hh; this warp takes 32-column chunks part, part + kParts, ...  Two chunks
// are loaded per tcgen05.wait, each transposed through the warp's 2 KB buffer xb so the global
// stores are 16-byte vectors along the token row (gate/up: SwiGLU of the interleaved halves).
template <int kParts>
__device__ __forceinline__ void epilogue_tile(const GemmParams& p, const Tile& tl, int halves, uint32_t tbase,
                                              int rg_base, int rg_step, int q, int part, int lane, uint16_t* xb) {
    const int nch = (tl.nvalid + 31) >> 5;
    const int per_half = (nch - part + kParts - 1) / kParts;   // chunks c = part, part + kParts, ...
    const int items = halves * per_half;
    for (int it = 0; it < items; it += 2) {
        float v[2][32];
        int hh[2], cc[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int iu = it + u < items ? it + u : it;
            hh[u] = iu / per_half;
            cc[u] = part + kParts * (iu - hh[u] * per_half);
            tmem_ld32_nowait(tbase + uint32_t(hh[u] * kAccCols + cc[u] * 32), v[u]);
        }
        tmem_wait_ld(v[0], v[1]);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            if (it + u >= items) break;
            const int c = cc[u], rg = rg_base + rg_step * hh[u];
            if (p.mode == 0) {
                const int fl = lane & 15;
                const bool lo = lane < 16;
                // token row t of the transpose buffer starts at xrow(t): rows 16..31 sit 32 bytes
                // further on, so the two half-warps' 2-byte stores fall in different banks
                auto xrow = [](int t) { return t * 16 + (t >= 16 ? 16 : 0); };
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float send = lo ? v[u][16 + i] : v[u][i];
                    const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
                    const float gt = lo ? v[u][i] : recv;
                    const float up = lo ? recv : v[u][16 + i];
                    xb[xrow(lo ? i : 16 + i) + fl] = f2bf(silu_mul(gt, up));
                }
                __syncwarp();
                const int fbase = rg * 64 + 16 * q;
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const int ch = lane + 32 * r, tok = ch >> 1, pp = ch & 1;
                    const int n = c * 32 + tok;
                    if (n < tl.nvalid)
                        *reinterpret_cast<uint4*>(p.out + size_t(tl.row0 + n) * p.out_ld + fbase + 8 * pp) =
                            *reinterpret_cast<const uint4*>(xb + xrow(tok) + 8 * pp);
                }
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) xb[j * 32 + lane] = f2bf(v[u][j]);
                __syncwarp();
                const int hbase = rg * 128 + 32 * q;
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int ch = lane + 32 * r, tok = ch >> 2, pp = ch & 3;
                    const int n = c * 32 + tok;
                    if (n < tl.nvalid)
                        *reinterpret_cast<uint4*>(p.out + size_t(tl.row0 + n) * p.out_ld + hbase + 8 * pp) =
                            *reinterpret_cast<const uint4*>(xb + tok * 32 + 8 * pp);
                }
            }
            __syncwarp();
        }
    }
}

// MXFP4 grouped GEMM on CTA pairs with TMA-streamed codes (gemm_mx_sm100.cu): used when K is a
// multiple of 512 and the 128-row weight groups come in fours; returns 0 ok, 1 tensor-map
// failure, 2 launch failure
bool mx_pair_eligible(int mode, int H, int F);
int launch_moe_gemm_mx_pair(const GemmLaunch& L, const GemmParams& p, cudaStream_t st);

}  // namespace ftmoe

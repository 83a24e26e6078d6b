// Step 3/4 (decode) -- few tokens per expert: the layer is a stream over the routed
// experts' weights, so the kernels below are built around 128-bit non-allocating weight
// loads with many bytes in flight per SM, and touch every routed weight byte once.
//
//   decode_gateup_kernel:  grid (active-group slot, F/16).  One warp = one f at a time:
//       gate row f and up row F+f of w13_e streamed once, dotted with the group's token
//       rows (staged in shared memory), h = silu(gate) * up -> bf16 h[row, f].
//   decode_down_kernel:    grid H/16.  Each CTA owns 16 hidden rows; for every active
//       group it streams those rows of w2_e and dots them with the group's h rows into a
//       shared [R][16] product tile, then combines y[t, hrow] = sum_j g[t,j] * prod[pos(t,j)]
//       (+ shared expert) in j order in fp32 -- no atomics, deterministic.  With y == NULL
//       it writes o_sorted[r, hrow] = bf16(prod) instead (the unfused experts entry point).
// BF16 weights use fma.rn.f32.bf16 (exact products, fp32 accumulation).  MXFP4 weights
// are decoded with cvt.rn.f16x2.e2m1x2 (exact) and accumulated per 32-element block with
// fma.rn.f32.f16 against f16 activations, then scaled once by the block's E8M0 scale.
// The f16 activation copy is exact for 2^-17 <= |v| <= 65504 (bf16 has 8 significant bits).
#include "kernels.h"

namespace ftmoe {



struct EW { const uint8_t *w13, *w13s, *w2, *w2s; };

__device__ __forceinline__ EW expert_w(const DecodeArgs& a, int g) {
    EW r;
    if (g >= a.E) { r.w13 = a.sw13; r.w13s = a.sw13s; r.w2 = a.sw2; r.w2s = a.sw2s; return r; }
    if (a.eptr) {
        r.w13 = static_cast<const uint8_t*>(a.eptr[4 * g + 0]);
        r.w13s = static_cast<const uint8_t*>(a.eptr[4 * g + 1]);
        r.w2 = static_cast<const uint8_t*>(a.eptr[4 * g + 2]);
        r.w2s = static_cast<const uint8_t*>(a.eptr[4 * g + 3]);
        return r;
    }
    const size_t HF = size_t(a.H) * a.F;
    if (a.wdtype == FT_W_BF16) {
        r.w13 = a.w13 + size_t(g) * 2 * HF * 2;
        r.w2 = a.w2 + size_t(g) * HF * 2;
        r.w13s = r.w2s = nullptr;
    } else {
        r.w13 = a.w13 + size_t(g) * 2 * HF / 2;
        r.w13s = a.w13s + size_t(g) * 2 * HF / 32;
        r.w2 = a.w2 + size_t(g) * HF / 2;
        r.w2s = a.w2s + size_t(g) * HF / 32;
    }
    return r;
}

// acc += (w.lo * x.lo) + (w.hi * x.hi), exact products, fp32 accumulate
__device__ __forceinline__ void fma2_bf16(float& acc, uint32_t w, uint32_t x) {
    asm("{\n\t.reg .b16 wl, wh, xl, xh;\n\tmov.b32 {wl, wh}, %1;\n\tmov.b32 {xl, xh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, wl, xl, %0;\n\tfma.rn.f32.bf16 %0, wh, xh, %0;\n\t}"
        : "+f"(acc) : "r"(w), "r"(x));
}
__device__ __forceinline__ void fma2_f16(float& acc, uint32_t w, uint32_t x) {
    asm("{\n\t.reg .b16 wl, wh, xl, xh;\n\tmov.b32 {wl, wh}, %1;\n\tmov.b32 {xl, xh}, %2;\n\t"
        "fma.rn.f32.f16 %0, wl, xl, %0;\n\tfma.rn.f32.f16 %0, wh, xh, %0;\n\t}"
        : "+f"(acc) : "r"(w), "r"(x));
}
// two E2M1 codes (one byte) -> f16x2 (low nibble in the low half), exact
__device__ __forceinline__ uint32_t e2m1x2_f16x2(uint32_t byte) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\t.reg .b16 s;\n\tcvt.u16.u32 s, %1;\n\tcvt.u8.u16 t, s;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
        : "=r"(r) : "r"(byte));
    return r;
}
__device__ __forceinline__ float e8m0f(uint32_t s) { return s == 0 ? __uint_as_float(0x00400000u) : __uint_as_float(s << 23); }
__device__ __forceinline__ uint32_t f32x2_to_f16x2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// dot of one 32-element MXFP4 block (16 code bytes) with 32 f16 activations (4 x uint4)
__device__ __forceinline__ float mx_block_dot(const uint4& c, const uint4* xv) {
    float a0 = 0.f, a1 = 0.f;
    const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {            // 4 code bytes per word -> 8 elements
        const uint4 xx = xv[q];
        const uint32_t xw[4] = {xx.x, xx.y, xx.z, xx.w};
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            uint32_t wf = e2m1x2_f16x2((cw[q] >> (8 * b)) & 0xFFu);
            if (b & 1) fma2_f16(a1, wf, xw[b]); else fma2_f16(a0, wf, xw[b]);
        }
    }
    return a0 + a1;
}

// ------------------------------------------------------------------ gate/up + SwiGLU
constexpr int kFPB = 16;      // f values per CTA (2 per warp)

template <int TB, bool MX>
__global__ void __launch_bounds__(256) decode_gateup_kernel(DecodeArgs a) {
    extern __shared__ uint4 xs4[];                   // [TB][H] bf16 (BF16) or f16 (MXFP4)
    const int G = a.E + (a.S ? 1 : 0);
    const int n_active = a.sched[1];
    const int slot = blockIdx.x;
    if (slot >= n_active) return;
    const int g = a.sched[2 + (G + 1) + slot];
    const int r0 = a.offsets[g];
    const int n = a.offsets[g + 1] - r0;
    const int P = a.T * a.k;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const EW w = expert_w(a, g);
    const int H = a.H, F = a.F;
    const int nv = H / 8;                            // 16-byte activation vectors per row
    for (int tb = 0; tb < n; tb += TB) {
        const int nb = min(TB, n - tb);
        __syncthreads();
        for (int i = warp; i < nb; i += 8) {
            int p = a.sorted_flat[r0 + tb + i];
            int t = p < P ? p / a.k : p - P;
            const uint4* src = reinterpret_cast<const uint4*>(a.x + size_t(t) * H);
            uint4* dst = xs4 + size_t(i) * nv;
            for (int v = lane; v < nv; v += 32) {
                uint4 u = __ldg(src + v);
                if (MX) {
                    u = make_uint4(f32x2_to_f16x2(bf16lo(u.x), bf16hi(u.x)), f32x2_to_f16x2(bf16lo(u.y), bf16hi(u.y)),
                                   f32x2_to_f16x2(bf16lo(u.z), bf16hi(u.z)), f32x2_to_f16x2(bf16lo(u.w), bf16hi(u.w)));
                }
                dst[v] = u;
            }
        }
        __syncthreads();
        for (int fi = 0; fi < kFPB / 8; ++fi) {
            const int f = blockIdx.y * kFPB + warp * (kFPB / 8) + fi;
            if (f >= F) break;
            float ag[TB], au[TB];
#pragma unroll
            for (int i = 0; i < TB; ++i) { ag[i] = 0.f; au[i] = 0.f; }
            if (!MX) {
                const uint4* gr = reinterpret_cast<const uint4*>(w.w13 + size_t(f) * H * 2);
                const uint4* ur = reinterpret_cast<const uint4*>(w.w13 + size_t(F + f) * H * 2);
                for (int c0 = lane; c0 < nv; c0 += 32 * 4) {
                    uint4 wg[4], wu[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        int c = c0 + 32 * u;
                        if (c < nv) { wg[u] = ldg_nc_v4(gr + c); wu[u] = ldg_nc_v4(ur + c); }
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        int c = c0 + 32 * u;
                        if (c >= nv) break;
#pragma unroll
                        for (int i = 0; i < TB; ++i) {
                            if (i >= nb) break;
                            uint4 xv = xs4[size_t(i) * nv + c];
                            fma2_bf16(ag[i], wg[u].x, xv.x); fma2_bf16(ag[i], wg[u].y, xv.y);
                            fma2_bf16(ag[i], wg[u].z, xv.z); fma2_bf16(ag[i], wg[u].w, xv.w);
                            fma2_bf16(au[i], wu[u].x, xv.x); fma2_bf16(au[i], wu[u].y, xv.y);
                            fma2_bf16(au[i], wu[u].z, xv.z); fma2_bf16(au[i], wu[u].w, xv.w);
                        }
                    }
                }
            } else {
                const int nblk = H / 32;
                const uint4* gq = reinterpret_cast<const uint4*>(w.w13 + size_t(f) * (H / 2));
                const uint4* uq = reinterpret_cast<const uint4*>(w.w13 + size_t(F + f) * (H / 2));
                const uint8_t* gs = w.w13s + size_t(f) * nblk;
                const uint8_t* us = w.w13s + size_t(F + f) * nblk;
                for (int b0 = lane; b0 < nblk; b0 += 32 * 4) {
                    uint4 cg[4], cu[4];
                    uint32_t sg[4], su[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        int b = b0 + 32 * u;
                        if (b < nblk) { cg[u] = ldg_nc_v4(gq + b); cu[u] = ldg_nc_v4(uq + b); sg[u] = gs[b]; su[u] = us[b]; }
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        int b = b0 + 32 * u;
                        if (b >= nblk) break;
                        const float scg = e8m0f(sg[u]), scu = e8m0f(su[u]);
#pragma unroll
                        for (int i = 0; i < TB; ++i) {
                            if (i >= nb) break;
                            const uint4* xv = xs4 + size_t(i) * nv + b * 4;
                            ag[i] = fmaf(mx_block_dot(cg[u], xv), scg, ag[i]);
                            au[i] = fmaf(mx_block_dot(cu[u], xv), scu, au[i]);
                        }
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < TB; ++i) {
                if (i >= nb) break;
                float gs_ = warp_sum(ag[i]);
                float us_ = warp_sum(au[i]);
                if (lane == 0) a.h[size_t(r0 + tb + i) * F + f] = f2bf(silu_mul(gs_, us_));
            }
        }
    }
}

// ------------------------------------------------------------------ down + combine
constexpr int kRPB = 16;      // hidden rows per CTA
constexpr int kMaxDecodeRows = 32 * (kMaxTopK + 1);

template <bool MX>
__global__ void __launch_bounds__(256) decode_down_kernel(DecodeArgs a) {
    __shared__ float prod[kMaxDecodeRows][kRPB + 1];
    const int G = a.E + (a.S ? 1 : 0);
    const int n_active = a.sched[1];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = a.H, F = a.F;
    const int hbase = blockIdx.x * kRPB;
    const int items = n_active * kRPB;
    for (int it = warp; it < items; it += 8) {
        const int slot = it / kRPB, j = it - slot * kRPB;
        const int g = a.sched[2 + (G + 1) + slot];
        const int hrow = hbase + j;
        if (hrow >= H) continue;
        const int r0 = a.offsets[g], n = a.offsets[g + 1] - r0;
        const EW w = expert_w(a, g);
        if (!MX) {
            const int nv = F / 8;
            const uint4* wr = reinterpret_cast<const uint4*>(w.w2 + size_t(hrow) * F * 2);
            // weight row into registers (F <= 4096 -> <= 16 vectors per lane)
            uint4 wv[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                int c = lane + 32 * u;
                if (c < nv) wv[u] = ldg_nc_v4(wr + c);
            }
            for (int r = 0; r < n; ++r) {
                const uint4* hr = reinterpret_cast<const uint4*>(a.h + size_t(r0 + r) * F);
                float s0 = 0.f, s1 = 0.f;
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    int c = lane + 32 * u;
                    if (c < nv) {
                        uint4 hv = __ldg(hr + c);
                        fma2_bf16(s0, wv[u].x, hv.x); fma2_bf16(s1, wv[u].y, hv.y);
                        fma2_bf16(s0, wv[u].z, hv.z); fma2_bf16(s1, wv[u].w, hv.w);
                    }
                }
                float s = warp_sum(s0 + s1);
                if (lane == 0) prod[r0 + r][j] = s;
            }
        } else {
            const int nblk = F / 32;
            const uint4* wq = reinterpret_cast<const uint4*>(w.w2 + size_t(hrow) * (F / 2));
            const uint8_t* wsr = w.w2s + size_t(hrow) * nblk;
            uint4 cv[4];
            uint32_t sv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {          // F <= 4096 -> <= 4 blocks per lane
                int b = lane + 32 * u;
                if (b < nblk) { cv[u] = ldg_nc_v4(wq + b); sv[u] = wsr[b]; }
            }
            for (int r = 0; r < n; ++r) {
                const uint4* hr = reinterpret_cast<const uint4*>(a.h + size_t(r0 + r) * F);
                float s = 0.f;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    int b = lane + 32 * u;
                    if (b < nblk) {
                        uint4 xv[4];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            uint4 hv = __ldg(hr + b * 4 + q);
                            xv[q] = make_uint4(f32x2_to_f16x2(bf16lo(hv.x), bf16hi(hv.x)),
                                               f32x2_to_f16x2(bf16lo(hv.y), bf16hi(hv.y)),
                                               f32x2_to_f16x2(bf16lo(hv.z), bf16hi(hv.z)),
                                               f32x2_to_f16x2(bf16lo(hv.w), bf16hi(hv.w)));
                        }
                        s = fmaf(mx_block_dot(cv[u], xv), e8m0f(sv[u]), s);
                    }
                }
                s = warp_sum(s);
                if (lane == 0) prod[r0 + r][j] = s;
            }
        }
    }
    __syncthreads();
    const int P = a.T * a.k;
    if (a.y) {
        for (int q = tid; q < a.T * kRPB; q += 256) {
            const int t = q / kRPB, j = q - t * kRPB;
            const int hrow = hbase + j;
            if (hrow >= H) continue;
            float acc = 0.f;
            for (int jj = 0; jj < a.k; ++jj) {
                int pos = a.inv_pos[t * a.k + jj];
                acc = fmaf(a.topk_w[t * a.k + jj], prod[pos][j], acc);
            }
            if (a.S) acc += prod[a.inv_pos[P + t]][j];
            a.y[size_t(t) * H + hrow] = f2bf(acc);
        }
    } else {
        const int R = a.offsets[G];
        for (int q = tid; q < R * kRPB; q += 256) {
            const int r = q / kRPB, j = q - r * kRPB;
            const int hrow = hbase + j;
            if (hrow < H) a.o_sorted[size_t(r) * H + hrow] = f2bf(prod[r][j]);
        }
    }
}

// ------------------------------------------------------------------ host launch
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st) {
    if (a.T <= 0) return cudaSuccess;
    const int P = a.T * a.k, R = P + (a.S ? a.T : 0);
    const int G = a.E + (a.S ? 1 : 0);
    const int na_max = R < G ? R : G;
    const bool mx = a.wdtype == FT_W_MXFP4;
    int TB = 1;
    while (TB < a.T && TB < 8) TB <<= 1;
    // keep the staged token rows within 64 KB of shared memory
    while (TB > 1 && size_t(TB) * a.H * 2 > 65536) TB >>= 1;
    const size_t smem = size_t(TB) * a.H * 2;
    dim3 g1(na_max, (a.F + kFPB - 1) / kFPB);
#define FT_GU(TBV)                                                                                         \
    do {                                                                                                   \
        auto kern = mx ? decode_gateup_kernel<TBV, true> : decode_gateup_kernel<TBV, false>;              \
        if (smem > 48 * 1024) {                                                                            \
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)); \
            if (e != cudaSuccess) return e;                                                                \
        }                                                                                                  \
        kern<<<g1, 256, smem, st>>>(a);                                                                    \
    } while (0)
    switch (TB) {
        case 1: FT_GU(1); break;
        case 2: FT_GU(2); break;
        case 4: FT_GU(4); break;
        default: FT_GU(8); break;
    }
#undef FT_GU
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    dim3 g2((a.H + kRPB - 1) / kRPB);
    if (mx) decode_down_kernel<true><<<g2, 256, 0, st>>>(a);
    else decode_down_kernel<false><<<g2, 256, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace ftmoe

// Device helpers shared by the decode kernels (three-kernel path and fused layer kernel):
// expert weight addressing, exact-product dot steps for BF16 and MXFP4, warp transpose-reduce,
// bulk async copies and programmatic-dependent-launch controls.
#pragma once
#include "kernels.h"
#include "sm100.cuh"

namespace ftmoe {

// gpu-scope acquire load of a cross-CTA counter (the tensor-core decodes' per-group readiness)
__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* a) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
    return v;
}

struct EW { const uint8_t *w13, *w13s, *w2, *w2s; };

// Programmatic dependent launch: a kernel launched with the programmatic-serialization
// attribute may start while its predecessor finishes; griddepcontrol.wait blocks until the
// predecessor grid has completed and its memory is visible (a no-op for plain launches).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

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

// One 32-element MXFP4 block (16 code bytes) as 16 f16x2 words: word 4q+b holds elements
// 8q+2b (low half) and 8q+2b+1, exactly.
__device__ __forceinline__ void mx_block_cvt(const uint4& c, uint32_t (&wf)[16]) {
    const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int b = 0; b < 4; ++b) wf[4 * q + b] = e2m1x2_f16x2((cw[q] >> (8 * b)) & 0xFFu);
}
// dot of a converted block with 32 f16 activations (4 x uint4): exact products, two fp32 chains
__device__ __forceinline__ float mx_cvt_dot(const uint32_t (&wf)[16], const uint4* xv) {
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 xx = xv[q];
        fma2_f16(a0, wf[4 * q + 0], xx.x);
        fma2_f16(a1, wf[4 * q + 1], xx.y);
        fma2_f16(a0, wf[4 * q + 2], xx.z);
        fma2_f16(a1, wf[4 * q + 3], xx.w);
    }
    return a0 + a1;
}
// the same dot with conversion and products interleaved (fewer live registers)
__device__ __forceinline__ float mx_block_dot(const uint4& c, const uint4* xv) {
    float a0 = 0.f, a1 = 0.f;
    const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 xx = xv[q];
        const uint32_t xw[4] = {xx.x, xx.y, xx.z, xx.w};
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const uint32_t wf = e2m1x2_f16x2((cw[q] >> (8 * b)) & 0xFFu);
            if (b & 1) fma2_f16(a1, wf, xw[b]); else fma2_f16(a0, wf, xw[b]);
        }
    }
    return a0 + a1;
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(su32(dst)), "l"(src), "r"(bytes), "r"(su32(bar)) : "memory");
}

constexpr int kFPB = 8;       // f values per CTA (one per warp)

// Staged rows are kept with their 16-byte vectors permuted inside aligned groups of eight:
// vector v sits at xswz(v).  The MXFP4 GEMV reads vectors 4b .. 4b+3 for block b = lane (+32u),
// i.e. a 64-byte stride across the warp; the permutation spreads each such read over all
// eight 16-byte bank groups (conflict-free), and it keeps unit-stride reads conflict-free.
__device__ __forceinline__ int xswz(int v) { return v ^ ((v >> 3) & 3); }

// Stage token row t of x into shared row dst_row (bf16, or f16 for MXFP4); one warp.
template <bool MX>
__device__ __forceinline__ void stage_x_row(const DecodeArgs& a, uint4* xs4, int t, int dst_row, int lane) {
    const int nv = a.H / 8;
    const uint4* src = reinterpret_cast<const uint4*>(a.x + size_t(t) * a.H);
    uint4* dst = xs4 + size_t(dst_row) * nv;
    for (int v = lane; v < nv; v += 32) {
        uint4 u = __ldg(src + v);
        if (MX) {
            u = make_uint4(f32x2_to_f16x2(bf16lo(u.x), bf16hi(u.x)), f32x2_to_f16x2(bf16lo(u.y), bf16hi(u.y)),
                           f32x2_to_f16x2(bf16lo(u.z), bf16hi(u.z)), f32x2_to_f16x2(bf16lo(u.w), bf16hi(u.w)));
        }
        dst[xswz(v)] = u;
    }
}

// Gate/up items item0, item0 + stride, ... of (active group, 8-value f block): one f per
// warp, gate and up rows streamed once with 128-bit loads and dotted with the group's token
// rows; h = silu(gate) * up.  FULLX: all token rows are already staged in xs4; otherwise the
// group's rows are staged per batch of TB.  Routing (sched, offsets, sorted_flat) comes
// through `a`, global or shared.
template <int TB, bool MX, bool FULLX, int U = 8>
__device__ __forceinline__ void gateup_items(const DecodeArgs& a, uint4* xs4, int* stok, int item0, int stride) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = a.H, F = a.F;
    const int nv = H / 8;
    const int G = a.E + (a.S ? 1 : 0);
    const int P = a.T * a.k;
    const int nfb = (F + kFPB - 1) / kFPB;
    const int n_active = a.sched[1];
    // f-block fastest so a CTA's items mostly share their group (and its staged rows)
    for (int item = item0; item < n_active * nfb; item += stride) {
    const int slot = item / nfb, fblk = item - slot * nfb;
    const int g = a.sched[2 + (G + 1) + slot];
    const int r0 = a.offsets[g];
    const int n = a.offsets[g + 1] - r0;
    const EW w = expert_w(a, g);
    for (int tb = 0; tb < n; tb += TB) {
        const int nb = min(TB, n - tb);
        __syncthreads();
        if (FULLX) {
            if (tid < nb) {
                const int p = a.sorted_flat[r0 + tb + tid];
                stok[tid] = p < P ? p / a.k : p - P;
            }
        } else {
            for (int i = warp; i < nb; i += 8) {
                const int p = a.sorted_flat[r0 + tb + i];
                stage_x_row<MX>(a, xs4, p < P ? p / a.k : p - P, i, lane);
            }
            if (tid < nb) stok[tid] = tid;
        }
        __syncthreads();
        for (int fi = 0; fi < kFPB / 8; ++fi) {
            const int f = fblk * kFPB + warp * (kFPB / 8) + fi;
            if (f >= F) break;
            float ag[TB], au[TB];
#pragma unroll
            for (int i = 0; i < TB; ++i) { ag[i] = 0.f; au[i] = 0.f; }
            if (!MX) {
                const uint4* gr = reinterpret_cast<const uint4*>(w.w13 + size_t(f) * H * 2);
                const uint4* ur = reinterpret_cast<const uint4*>(w.w13 + size_t(F + f) * H * 2);
                for (int c0 = lane; c0 < nv; c0 += 32 * U) {
                    uint4 wg[U], wu[U];
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        int c = c0 + 32 * u;
                        if (c < nv) { wg[u] = ldg_nc_v4(gr + c); wu[u] = ldg_nc_v4(ur + c); }
                    }
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        int c = c0 + 32 * u;
                        if (c >= nv) break;
#pragma unroll
                        for (int i = 0; i < TB; ++i) {
                            if (i >= nb) break;
                            uint4 xv = xs4[size_t(stok[i]) * nv + xswz(c)];
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
                        if (TB == 1) {
#pragma unroll
                            for (int i = 0; i < TB; ++i) {
                                if (i >= nb) break;
                                const uint4* xrow = xs4 + size_t(stok[i]) * nv;
                                const uint4 xv[4] = {xrow[xswz(4 * b)], xrow[xswz(4 * b + 1)], xrow[xswz(4 * b + 2)],
                                                     xrow[xswz(4 * b + 3)]};
                                ag[i] = fmaf(mx_block_dot(cg[u], xv), scg, ag[i]);
                                au[i] = fmaf(mx_block_dot(cu[u], xv), scu, au[i]);
                            }
                            continue;
                        }
                        // E2M1 -> f16 once per block, shared by every token of the batch
                        uint32_t fg[16], fu[16];
                        mx_block_cvt(cg[u], fg);
                        mx_block_cvt(cu[u], fu);
#pragma unroll
                        for (int i = 0; i < TB; ++i) {
                            if (i >= nb) break;
                            const uint4* xrow = xs4 + size_t(stok[i]) * nv;
                            const uint4 xv[4] = {xrow[xswz(4 * b)], xrow[xswz(4 * b + 1)], xrow[xswz(4 * b + 2)],
                                                 xrow[xswz(4 * b + 3)]};
                            ag[i] = fmaf(mx_cvt_dot(fg, xv), scg, ag[i]);
                            au[i] = fmaf(mx_cvt_dot(fu, xv), scu, au[i]);
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
}


// Four hidden rows j0..j0+3 of a block of one expert's down weights -- rows of F/2 code bytes
// (MXFP4) or 2F bytes (BF16) from `codes`, F/32 scale bytes per row from `scales`, in shared or
// global memory -- dotted with the group's n h rows starting at permuted row r0; products land
// in prod[row][j] (pitch RPB + 1).  One warp; lanes split F, a transpose-reduce leaves each
// row's sum on one lane.  CG: h was written by other CTAs of the same grid, so it is read
// around the L1.
template <bool MX, bool CG>
__device__ __forceinline__ void down_item4(const DecodeArgs& a, const uint8_t* codes, const uint8_t* scales, int RPB,
                                           int j0, int r0, int n, float* prod, int lane) {
    const int F = a.F;
    const size_t wrow = MX ? size_t(F) / 2 : size_t(F) * 2;
    const size_t srow = MX ? size_t(F) / 32 : 0;
    const int nvec = MX ? F / 32 : F / 8;
    const uint8_t* wb = codes;
    for (int r = 0; r < n; ++r) {
        const uint4* hr = reinterpret_cast<const uint4*>(a.h + size_t(r0 + r) * F);
        float v[4] = {0.f, 0.f, 0.f, 0.f};
        for (int q = lane; q < nvec; q += 32) {
            if (!MX) {
                const uint4 hv = CG ? __ldcg(hr + q) : __ldg(hr + q);
#pragma unroll
                for (int rr = 0; rr < 4; ++rr) {
                    const uint4 wv = *reinterpret_cast<const uint4*>(wb + size_t(j0 + rr) * wrow + size_t(q) * 16);
                    fma2_bf16(v[rr], wv.x, hv.x); fma2_bf16(v[rr], wv.y, hv.y);
                    fma2_bf16(v[rr], wv.z, hv.z); fma2_bf16(v[rr], wv.w, hv.w);
                }
            } else {
                uint4 xv[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const uint4 hv = CG ? __ldcg(hr + 4 * q + u) : __ldg(hr + 4 * q + u);
                    xv[u] = make_uint4(f32x2_to_f16x2(bf16lo(hv.x), bf16hi(hv.x)), f32x2_to_f16x2(bf16lo(hv.y), bf16hi(hv.y)),
                                       f32x2_to_f16x2(bf16lo(hv.z), bf16hi(hv.z)), f32x2_to_f16x2(bf16lo(hv.w), bf16hi(hv.w)));
                }
#pragma unroll
                for (int rr = 0; rr < 4; ++rr) {
                    const uint4 wv = *reinterpret_cast<const uint4*>(wb + size_t(j0 + rr) * wrow + size_t(q) * 16);
                    const uint32_t sc = scales[size_t(j0 + rr) * srow + q];
                    v[rr] = fmaf(mx_block_dot(wv, xv), e8m0f(sc), v[rr]);
                }
            }
        }
        tr_step(v, 4, 16, lane);
        tr_step(v, 2, 8, lane);
        v[0] += __shfl_xor_sync(0xffffffffu, v[0], 4);
        v[0] += __shfl_xor_sync(0xffffffffu, v[0], 2);
        v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
        if ((lane & 7) == 0) {   // lane l holds row 2*bit4(l) + bit3(l)
            const int sel = ((lane >> 4) & 1) * 2 + ((lane >> 3) & 1);
            prod[size_t(r0 + r) * (RPB + 1) + j0 + sel] = v[0];
        }
    }
}

}  // namespace ftmoe

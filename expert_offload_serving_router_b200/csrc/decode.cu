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
#include "decode_common.cuh"

namespace ftmoe {



// ------------------------------------------------------------------ gate/up + SwiGLU
// U: 16-byte weight vectors per lane kept in flight per row (BF16); MINB: resident CTAs per SM
// the register budget is cut for (more warps in flight hide the load latency of small batches).
template <int TB, bool MX, bool FULLX, int U, int MINB>
__global__ void __launch_bounds__(256, MINB) decode_gateup_kernel(DecodeArgs a) {
    // FULLX: every token row [T][H] staged once (bf16, or f16 for MXFP4) before the
    // programmatic dependency wait -- the layer input is complete before the router ran --
    // so the routing-dependent part starts straight with the weight stream.
    extern __shared__ uint4 xs4[];
    __shared__ int stok[TB];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (FULLX)
        for (int t = warp; t < a.T; t += 8) stage_x_row<MX>(a, xs4, t, t, lane);
    pdl_wait();
    pdl_trigger();
    gateup_items<TB, MX, FULLX, U>(a, xs4, stok, blockIdx.x, gridDim.x);
}

// ------------------------------------------------------------------ down + combine
constexpr int kRPB = 8;       // hidden rows per CTA
constexpr int kMaxDecodeRows = 32 * (kMaxTopK + 1);

template <bool MX, int CPL>
__global__ void __launch_bounds__(256, 2) decode_down_kernel(DecodeArgs a) {
    // CPL = weight vectors per lane per row (BF16: 16-byte chunks of 8; MXFP4: 32-element blocks)
    constexpr int RB = (MX ? 8 : 24) / CPL >= 8 ? 8 : (MX ? 8 : 24) / CPL >= 4 ? 4 : (MX ? 8 : 24) / CPL >= 2 ? 2 : 1;
    constexpr int NB = kRPB / RB;               // row batches per active group
    __shared__ float prod[kMaxDecodeRows][kRPB + 1];
    pdl_trigger();   // the next layer's router may launch; it waits for this grid before writing
    pdl_wait();
    const int G = a.E + (a.S ? 1 : 0);
    const int n_active = a.sched[1];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = a.H, F = a.F;
    const int hbase = blockIdx.x * kRPB;
    const int nvec = MX ? F / 32 : F / 8;      // vectors per row
    for (int it = warp; it < n_active * NB; it += 8) {
        const int slot = it / NB, j0 = (it - slot * NB) * RB;
        const int g = a.sched[2 + (G + 1) + slot];
        const int r0 = a.offsets[g], n = a.offsets[g + 1] - r0;
        const EW w = expert_w(a, g);
        // stream RB weight rows (all loads issued before any use)
        uint4 wv[RB][CPL];
        uint32_t ws_[RB][CPL];
#pragma unroll
        for (int rr = 0; rr < RB; ++rr) {
            const int hrow = min(hbase + j0 + rr, H - 1);
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                const int c = lane + 32 * i;
                if (c < nvec) {
                    if (!MX) {
                        wv[rr][i] = ldg_nc_v4(w.w2 + (size_t(hrow) * F + size_t(c) * 8) * 2);
                    } else {
                        wv[rr][i] = ldg_nc_v4(w.w2 + size_t(hrow) * (F / 2) + size_t(c) * 16);
                        ws_[rr][i] = w.w2s[size_t(hrow) * (F / 32) + c];
                    }
                }
            }
        }
        for (int r = 0; r < n; ++r) {
            const uint4* hr = reinterpret_cast<const uint4*>(a.h + size_t(r0 + r) * F);
            float s[RB];
#pragma unroll
            for (int rr = 0; rr < RB; ++rr) s[rr] = 0.f;
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                const int c = lane + 32 * i;
                if (c >= nvec) break;
                if (!MX) {
                    const uint4 hv = __ldg(hr + c);
#pragma unroll
                    for (int rr = 0; rr < RB; ++rr) {
                        fma2_bf16(s[rr], wv[rr][i].x, hv.x); fma2_bf16(s[rr], wv[rr][i].y, hv.y);
                        fma2_bf16(s[rr], wv[rr][i].z, hv.z); fma2_bf16(s[rr], wv[rr][i].w, hv.w);
                    }
                } else {
                    uint4 xv[4];
#pragma unroll
                    for (int qq = 0; qq < 4; ++qq) {
                        const uint4 hv = __ldg(hr + c * 4 + qq);
                        xv[qq] = make_uint4(f32x2_to_f16x2(bf16lo(hv.x), bf16hi(hv.x)), f32x2_to_f16x2(bf16lo(hv.y), bf16hi(hv.y)),
                                            f32x2_to_f16x2(bf16lo(hv.z), bf16hi(hv.z)), f32x2_to_f16x2(bf16lo(hv.w), bf16hi(hv.w)));
                    }
#pragma unroll
                    for (int rr = 0; rr < RB; ++rr) s[rr] = fmaf(mx_block_dot(wv[rr][i], xv), e8m0f(ws_[rr][i]), s[rr]);
                }
            }
            // transpose-reduce the RB partial sums across the warp
            float v[RB];
#pragma unroll
            for (int rr = 0; rr < RB; ++rr) v[rr] = s[rr];
            int nv_ = RB;
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) {
                if (nv_ > 1) { tr_step(v, nv_, off, lane); nv_ >>= 1; }
                else v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
            }
            // lane l holds the sum of value index sel(l): bit (4 - level) of l picks the upper half
            int sel = 0;
            {
                int m = RB, off = 16;
                while (m > 1) { sel = sel * 2 + ((lane & off) ? 1 : 0); m >>= 1; off >>= 1; }
            }
            const int lead = (lane & ~((32 / RB) - 1)) == lane;   // one lane per value index
            if (lead) {
                const int j = j0 + sel;
                if (hbase + j < H) prod[r0 + r][j] = v[0];
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

// Single-pass variant for small batches: all routed experts' RPB rows of W2 fit in shared
// memory together, so each CTA issues every weight copy (one bulk async copy per expert, plus
// one for its MXFP4 scales) before the programmatic dependency wait -- the routing was final
// before the gate/up kernel started, only h comes from it -- and the weights stream while
// the gate/up kernel finishes.  Warp items are (expert, 4 rows), dot products from shared
// memory, then the same products tile and combine as above.
struct DownBulkCfg { int RPB, chunk, nbuf, R; };

template <bool MX>
__global__ void __launch_bounds__(256, 2) decode_down_bulk_kernel(DecodeArgs a, DownBulkCfg c) {
    extern __shared__ __align__(128) uint8_t dsm[];
    const int RPB = c.RPB;
    float* prod = reinterpret_cast<float*>(dsm);                                   // [R][RPB + 1]
    uint8_t* wbuf = dsm + ((size_t(c.R) * (RPB + 1) * 4 + 127) & ~size_t(127));    // [nbuf][chunk]
    uint64_t* full = reinterpret_cast<uint64_t*>(wbuf + size_t(c.nbuf) * c.chunk);
    __shared__ int s_g[kMaxExperts + 1];
    __shared__ int s_bad;
    pdl_trigger();   // the next layer's router may launch; it waits for this grid before writing
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = a.H, F = a.F;
    const int G = a.E + (a.S ? 1 : 0);
    const int hbase = blockIdx.x * RPB;
    const size_t wrow = MX ? size_t(F) / 2 : size_t(F) * 2;      // weight bytes per row
    const size_t srow = MX ? size_t(F) / 32 : 0;                 // scale bytes per row
    const int n_active = __ldcg(a.sched + 1);
    for (int i = tid; i < n_active; i += blockDim.x) s_g[i] = __ldcg(a.sched + 2 + (G + 1) + i);
    if (tid == 0) {
        s_bad = n_active > c.nbuf;   // more experts than buffers: the host sizing was wrong
        for (int i = 0; i < c.nbuf; ++i) mbar_init(&full[i], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (s_bad) {
        if (tid == 0) atomicExch(a.err, kDevErrShape);
        pdl_wait();
        return;
    }
    if (tid == 0) {
        for (int i = 0; i < n_active; ++i) {
            const EW w = expert_w(a, s_g[i]);
            uint8_t* dst = wbuf + size_t(i) * c.chunk;
            const uint32_t wb = uint32_t(RPB * wrow), sb = uint32_t(RPB * srow);
            mbar_expect_tx(&full[i], wb + sb);
            bulk_g2s(dst, w.w2 + size_t(hbase) * wrow, wb, &full[i]);
            if (MX) bulk_g2s(dst + wb, w.w2s + size_t(hbase) * srow, sb, &full[i]);
        }
    }
    pdl_wait();   // h from the gate/up kernel
    const int gpr = RPB / 4;
    for (int it = warp; it < n_active * gpr; it += 8) {
        const int slot = it / gpr, j0 = 4 * (it - slot * gpr);
        if (!mbar_wait(&full[slot], 0, nullptr)) { s_bad = 1; continue; }
        const int g = s_g[slot];
        const int r0 = a.offsets[g], n = a.offsets[g + 1] - r0;
        const uint8_t* wb = wbuf + size_t(slot) * c.chunk;
        down_item4<MX, false>(a, wb, wb + size_t(RPB) * wrow, RPB, j0, r0, n, prod, lane);
    }
    __syncthreads();
    if (s_bad) {
        if (tid == 0) {
            atomicExch(a.err, kDevErrTimeout);
            for (int i = 0; i < n_active; ++i) mbar_wait(&full[i], 0, nullptr);   // let copies land
        }
        return;
    }
    const int P = a.T * a.k;
    if (a.y) {
        for (int q = tid; q < a.T * RPB; q += blockDim.x) {
            const int t = q / RPB, j = q - t * RPB;
            float acc = 0.f;
            for (int jj = 0; jj < a.k; ++jj) {
                const int pos = a.inv_pos[t * a.k + jj];
                acc = fmaf(a.topk_w[t * a.k + jj], prod[size_t(pos) * (RPB + 1) + j], acc);
            }
            if (a.S) acc += prod[size_t(a.inv_pos[P + t]) * (RPB + 1) + j];
            a.y[size_t(t) * H + hbase + j] = f2bf(acc);
        }
    } else {
        const int R = a.offsets[G];
        for (int q = tid; q < R * RPB; q += blockDim.x) {
            const int r = q / RPB, j = q - r * RPB;
            a.o_sorted[size_t(r) * H + hbase + j] = f2bf(prod[size_t(r) * (RPB + 1) + j]);
        }
    }
}

// ------------------------------------------------------------------ host launch
template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

// BF16 decode batches of at least this many tokens run on the tensor cores (decode_mma.cu);
// smaller ones stream through the SIMT GEMVs below.  With a shared expert one group always holds
// every token, and the tensor cores win from two tokens on (gemma4_26b_a4b T = 2 / 4: 55.3 ->
// 50.5 / 84.2 -> 69.9 us); without one from four (qwen3_a3b T = 3: 39.9 vs 42.3, T = 4 even,
// T = 6: 56.9 -> 49.4 us)
constexpr int kDecodeMmaMinT = 4;
constexpr int kDecodeMmaMinTShared = 2;
// MXFP4 decode batches of 4+ tokens run on the block-scaled tensor cores (ft_set_block_scaled_decode
// selects never / always / that default); smaller ones on the GEMVs below, faster there

DecodePath decode_path(const DecodeArgs& a) {
    if (a.T >= (a.S ? kDecodeMmaMinTShared : kDecodeMmaMinT) && decode_mma_eligible(a)) return kDecodeMma;
    if (block_scaled_decode(a.T) && decode_mx_eligible(a)) return decode_mx_fused(a) ? kDecodeMxFused : kDecodeMxTwo;
    return kDecodeGemv;
}

int decode_path_kernels(DecodePath p, bool combine) {
    switch (p) {
        case kDecodeMma: return 1 + combine;                 // decode_mma_kernel, combine
        case kDecodeMxFused: return 2 + combine;             // quant2 (x), decode_mx_fused_kernel, combine
        case kDecodeMxTwo: return 4 + combine;               // quant2 (x), gate/up, quant2 (h), down, combine
        default: return 2;                                   // gate/up GEMV, down GEMV (+ combine, fused)
    }
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st) {
    if (a.T <= 0) return cudaSuccess;
    const DecodePath path = decode_path(a);
    if (path == kDecodeMma) return launch_decode_mma(a, st);
    if (path == kDecodeMxFused || path == kDecodeMxTwo) return launch_decode_mx(a, st);
    const int P = a.T * a.k, R = P + (a.S ? a.T : 0);
    const int G = a.E + (a.S ? 1 : 0);
    {
        cudaError_t ce = launch_slot_table_check(a.sched, G, a.E, a.eptr, a.wdtype == FT_W_MXFP4, a.err, st);
        if (ce != cudaSuccess) return ce;
    }
    const int na_max = R < G ? R : G;
    const bool mx = a.wdtype == FT_W_MXFP4;
    int TB = 1;
    while (TB < a.T && TB < 8) TB <<= 1;
    // small batches stage all token rows once per CTA (before the dependency wait); larger
    // ones stage each group's rows per batch of TB
    const bool fullx = size_t(a.T) * a.H * 2 <= 64 * 1024;
    while (!fullx && TB > 1 && size_t(TB) * a.H * 2 > 65536) TB >>= 1;
    const size_t smem = size_t(fullx ? a.T : TB) * a.H * 2;
    int items = na_max * ((a.F + kFPB - 1) / kFPB);   // upper bound; the kernel strides over the real count
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms <= 0) sms = 148;
    }
    // one-token batches: four (MXFP4: three) resident CTAs per SM, fewer vectors in flight per lane
    const bool wide = TB == 1 && fullx;
    const int per_sm = wide ? (mx ? 3 : 4) : 2;
    dim3 g1(items < per_sm * sms ? items : per_sm * sms);     // one wave
    cudaError_t e = cudaSuccess;
    if (wide) {
        e = mx ? launch_pdl(decode_gateup_kernel<1, true, true, 4, 3>, g1, dim3(256), smem, st, a)
               : launch_pdl(decode_gateup_kernel<1, false, true, 4, 4>, g1, dim3(256), smem, st, a);
        if (e != cudaSuccess) return e;
    } else {
#define FT_GU(TBV, MXV, FX)                                                                                   \
    do {                                                                                                      \
        auto kern = decode_gateup_kernel<TBV, MXV, FX, 8, 2>;                                                 \
        if (smem > 48 * 1024) {                                                                               \
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));            \
            if (e != cudaSuccess) return e;                                                                   \
        }                                                                                                     \
        e = launch_pdl(kern, g1, dim3(256), smem, st, a);                                                    \
    } while (0)
#define FT_GU2(TBV)                                                                                           \
    do {                                                                                                      \
        if (mx) { if (fullx) FT_GU(TBV, true, true); else FT_GU(TBV, true, false); }                         \
        else { if (fullx) FT_GU(TBV, false, true); else FT_GU(TBV, false, false); }                           \
    } while (0)
    switch (TB) {
        case 1: FT_GU2(1); break;
        case 2: FT_GU2(2); break;
        case 4: FT_GU2(4); break;
        default: FT_GU2(8); break;
    }
#undef FT_GU2
#undef FT_GU
    }
    if (e != cudaSuccess) return e;
    // down: the single-pass bulk-copy kernel when every routed expert's row block fits in
    // shared memory at two CTAs per SM, else the register-streaming kernel
    {
        constexpr size_t kBulkSmem = 110 * 1024;
        const size_t wrow = mx ? size_t(a.F) / 2 + size_t(a.F) / 32 : size_t(a.F) * 2;
        auto need = [&](int rpb) {
            return ((size_t(R) * (rpb + 1) * 4 + 127) & ~size_t(127)) + size_t(na_max) * (size_t(rpb) * wrow + 8);
        };
        int rpb = 0;
        if (a.H % 16 == 0 && a.H / 8 > 2 * sms && need(16) <= kBulkSmem) rpb = 16;
        else if (need(8) <= kBulkSmem) rpb = 8;
        if (rpb && R <= kMaxDecodeRows) {
            DownBulkCfg c{rpb, int(size_t(rpb) * wrow), na_max, R};
            const size_t dsm = need(rpb);
            static PerDeviceOnce attr[2];
            auto kern = mx ? decode_down_bulk_kernel<true> : decode_down_bulk_kernel<false>;
            e = attr[mx]([&] { return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kBulkSmem)); });
            if (e != cudaSuccess) return e;
            e = launch_pdl(kern, dim3(a.H / rpb), dim3(256), dsm, st, a, c);
            if (e != cudaSuccess) return e;
            return cudaGetLastError();
        }
    }
    dim3 g2((a.H + kRPB - 1) / kRPB);
    const int vec = mx ? a.F / 32 : a.F / 8;          // vectors per weight row
    const int cpl = (vec + 31) / 32;
#define FT_DN(MXV, C) e = launch_pdl(decode_down_kernel<MXV, C>, g2, dim3(256), 0, st, a)
    if (mx) {
        if (cpl <= 1) FT_DN(true, 1); else if (cpl <= 2) FT_DN(true, 2); else if (cpl <= 4) FT_DN(true, 4);
        else return cudaErrorInvalidValue;
    } else {
        if (cpl <= 1) FT_DN(false, 1); else if (cpl <= 2) FT_DN(false, 2); else if (cpl <= 3) FT_DN(false, 3);
        else if (cpl <= 4) FT_DN(false, 4); else if (cpl <= 6) FT_DN(false, 6); else if (cpl <= 8) FT_DN(false, 8);
        else if (cpl <= 12) FT_DN(false, 12); else FT_DN(false, 16);
    }
#undef FT_DN
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace ftmoe

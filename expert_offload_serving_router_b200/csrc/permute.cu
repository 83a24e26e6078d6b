// Step 2 -- permutation: stable counting sort of the flat pairs p = t*k + j by expert id,
// the shared expert (S = 1) appended as group E holding tokens in order (flat id P + t).
//
// General path (three launches, any R):
//   perm_count:   one CTA per 1024-pair chunk; per-chunk histogram and each pair's stable
//                 rank inside its chunk (warp __match_any_sync + per-warp counts).
//   perm_scan:    one CTA; per-group running sums over chunks (chunk bases), exclusive
//                 scan over groups (offsets), GEMM tile schedule and active-group list.
//   perm_scatter: one CTA per chunk; pos = chunk base + local rank; writes sorted_flat,
//                 inv_pos and (optionally) gathers x rows into x_sorted with 16-byte moves.
// Small path (R <= 1024): one warp sorts (warp_permute_small), the CTA gathers.
#include "kernels.h"
#include "permute_small.cuh"

namespace ftmoe {

struct PermArgs {
    int T, k, E, S, H;
    const int32_t* idx;
    const uint16_t* x;
    uint16_t* x_sorted;
    int32_t* chunk_cnt;    // [C][G]
    int32_t* chunk_base;   // [C][G]
    int32_t* local_rank;   // [R]
    PermOut out;
};

__device__ __forceinline__ int pair_group(const PermArgs& a, int i, int P) {
    if (i >= P) return a.E;
    int g = a.idx[i];
    return (g >= 0 && g < a.E) ? g : -1;
}

__global__ void __launch_bounds__(256) perm_count_kernel(PermArgs a) {
    __shared__ int run[kMaxExperts + 2];
    __shared__ int wcnt[8][kMaxExperts + 2];
    const int P = a.T * a.k, R = P + (a.S ? a.T : 0), G = a.E + (a.S ? 1 : 0);
    const int c = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int g = tid; g < G; g += 256) run[g] = 0;
    for (int sub = 0; sub < kPermChunk / 256; ++sub) {
        for (int i = tid; i < 8 * (kMaxExperts + 2); i += 256) (&wcnt[0][0])[i] = 0;
        __syncthreads();
        const int i = c * kPermChunk + sub * 256 + tid;
        int g = i < R ? pair_group(a, i, P) : -2;
        if (g == -1) atomicExch(a.out.err, kDevErrBadExpert);
        unsigned peers = __match_any_sync(0xffffffffu, g);
        int rk = __popc(peers & ((1u << lane) - 1u));
        if (g >= 0 && rk == 0) wcnt[warp][g] = __popc(peers);
        __syncthreads();
        if (g >= 0) {
            int before = run[g];
            for (int w = 0; w < warp; ++w) before += wcnt[w][g];
            a.local_rank[i] = before + rk;
        }
        __syncthreads();
        for (int gg = tid; gg < G; gg += 256) {
            int s = 0;
#pragma unroll
            for (int w = 0; w < 8; ++w) s += wcnt[w][gg];
            run[gg] += s;
        }
    }
    __syncthreads();
    for (int g = tid; g < G; g += 256) a.chunk_cnt[size_t(c) * G + g] = run[g];
}

__global__ void __launch_bounds__(1024) perm_scan_kernel(PermArgs a, int C) {
    __shared__ int tot[kMaxExperts + 2];
    __shared__ int flag[kMaxExperts + 2];
    __shared__ int tmp[33];
    const int G = a.E + (a.S ? 1 : 0);
    const int g = threadIdx.x;
    if (g < G) {
        int r = 0;
#pragma unroll 8
        for (int c = 0; c < C; ++c) {
            int v = a.chunk_cnt[size_t(c) * G + g];
            a.chunk_base[size_t(c) * G + g] = r;
            r += v;
        }
        tot[g] = r;
        flag[g] = r > 0 ? 1 : 0;
    }
    __syncthreads();
    int n_active = block_exclusive_scan(flag, G, tmp);
    if (g < G) {
        if (tot[g] > 0) a.out.sched[2 + (G + 1) + flag[g]] = g;
    }
    __syncthreads();
    if (g < G) flag[g] = (tot[g] + kGemmBN - 1) / kGemmBN;
    __syncthreads();
    int ntiles = block_exclusive_scan(flag, G, tmp);
    if (g < G) a.out.sched[2 + g] = flag[g];
    if (g == 0) {
        a.out.sched[0] = ntiles;
        a.out.sched[1] = n_active;
        a.out.sched[2 + G] = ntiles;
    }
    int total = block_exclusive_scan(tot, G, tmp);
    if (g < G) {
        a.out.offsets[g] = tot[g];
        for (int c = 0; c < C; ++c) a.chunk_base[size_t(c) * G + g] += tot[g];
    }
    if (g == 0) a.out.offsets[G] = total;
}

// One CTA per 128 pairs (8 warps x 16): scatter the permutation, then gather the x rows.
constexpr int kScatterItems = 128;

// A warp copies rows q, q + 1 (q = 2 warp, 2 warp + 16, ...) of the CTA's pairs from x into
// x_sorted, every 16-byte vector of both rows loaded before the first store (NV per lane and
// row: rows of up to 32 NV vectors).  Rows whose pair is dropped (pos < 0) are skipped; the
// loads of a missing second row re-read the first (in range) and are not stored.
template <int NV>
__device__ __forceinline__ void gather_two_rows(const PermArgs& a, const int* spos, const int* stok, int n, int nv,
                                                int warp, int lane) {
    for (int q = 2 * warp; q < n; q += 16) {
        const int pos0 = spos[q], pos1 = q + 1 < n ? spos[q + 1] : -1;
        const uint4* src0 = reinterpret_cast<const uint4*>(a.x + size_t(stok[q]) * a.H);
        const uint4* src1 = reinterpret_cast<const uint4*>(a.x + size_t(q + 1 < n ? stok[q + 1] : stok[q]) * a.H);
        uint4* dst0 = reinterpret_cast<uint4*>(a.x_sorted + size_t(pos0 < 0 ? 0 : pos0) * a.H);
        uint4* dst1 = reinterpret_cast<uint4*>(a.x_sorted + size_t(pos1 < 0 ? 0 : pos1) * a.H);
        uint4 u0[NV], u1[NV];
#pragma unroll
        for (int j = 0; j < NV; ++j) {
            const int v = lane + 32 * j;
            if (v < nv) {
                if (pos0 >= 0) u0[j] = __ldg(src0 + v);
                if (pos1 >= 0) u1[j] = __ldg(src1 + v);
            }
        }
#pragma unroll
        for (int j = 0; j < NV; ++j) {
            const int v = lane + 32 * j;
            if (v < nv) {
                if (pos0 >= 0) dst0[v] = u0[j];
                if (pos1 >= 0) dst1[v] = u1[j];
            }
        }
    }
}

// GV: the gather form, chosen on the host from H: 8 / 12 = two rows per warp with GV vectors per
// lane and row (rows of up to 256 / 384 vectors), 0 = one row per warp, 4 vectors in flight.
template <int GV>
__global__ void __launch_bounds__(256) perm_scatter_kernel(PermArgs a) {
    __shared__ int spos[kScatterItems];
    __shared__ int stok[kScatterItems];
    const int P = a.T * a.k, R = P + (a.S ? a.T : 0), G = a.E + (a.S ? 1 : 0);
    const int tid = threadIdx.x;
    const int i0 = blockIdx.x * kScatterItems;
    const int n = min(kScatterItems, R - i0);
    if (tid < n) {
        const int i = i0 + tid;
        const int c = i / kPermChunk;
        const int g = pair_group(a, i, P);
        int pos = -1;
        if (g >= 0) {
            pos = a.chunk_base[size_t(c) * G + g] + a.local_rank[i];
            a.out.sorted_flat[pos] = i;
            a.out.inv_pos[i] = pos;
        }
        spos[tid] = pos;
        stok[tid] = i < P ? i / a.k : i - P;
    }
    if (!a.x_sorted) return;
    __syncthreads();
    // gather, 16-byte vectors.  Rows of up to 4 KB (6 KB): one warp moves two rows at once with
    // all their vectors in flight (8 / 12 per lane and row); longer rows: one warp per row, 4
    // vectors in flight per lane (measured best for each at H = 2048, 2816 and 4096).
    const int lane = tid & 31, warp = tid >> 5;
    const int nv = a.H / 8;
    if constexpr (GV > 0) {
        gather_two_rows<GV>(a, spos, stok, n, nv, warp, lane);
        return;
    }
    for (int q = warp; q < n; q += 8) {
        const int pos = spos[q];
        if (pos < 0) continue;
        const uint4* src = reinterpret_cast<const uint4*>(a.x + size_t(stok[q]) * a.H);
        uint4* dst = reinterpret_cast<uint4*>(a.x_sorted + size_t(pos) * a.H);
        for (int v0 = lane; v0 < nv; v0 += 128) {
            uint4 u[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (v0 + 32 * j < nv) u[j] = __ldg(src + v0 + 32 * j);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (v0 + 32 * j < nv) dst[v0 + 32 * j] = u[j];
        }
    }
}

__global__ void __launch_bounds__(256) perm_small_kernel(const int32_t* idx, int T, int k, int E, int S, PermOut out,
                                                         const uint16_t* x, uint16_t* x_sorted, int H) {
    __shared__ int32_t sidx[1024];
    __shared__ int cnt[kMaxExperts + 2];
    const int P = T * k, R = P + (S ? T : 0);
    for (int i = threadIdx.x; i < P; i += blockDim.x) sidx[i] = idx[i];
    __syncthreads();
    if (threadIdx.x < 32) warp_permute_small(sidx, T, k, E, S, cnt, out);
    if (!x_sorted) return;
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nv = H / 8;
    for (int i = warp; i < R; i += blockDim.x / 32) {
        const int g = i < P ? sidx[i] : E;
        if (g < 0 || g >= E + (i >= P ? 1 : 0)) continue;
        const int pos = out.inv_pos[i];
        const int t = i < P ? i / k : i - P;
        const uint4* src = reinterpret_cast<const uint4*>(x + size_t(t) * H);
        uint4* dst = reinterpret_cast<uint4*>(x_sorted + size_t(pos) * H);
        for (int v = lane; v < nv; v += 32) dst[v] = __ldg(src + v);
    }
}

cudaError_t launch_permute(int T, int k, int E, int S, int H, const int32_t* idx, const uint16_t* x,
                           uint16_t* x_sorted, int32_t* chunk_cnt, int32_t* chunk_base, int32_t* local_rank,
                           const PermOut& out, cudaStream_t st) {
    if (T <= 0) return cudaSuccess;
    const int P = T * k, R = P + (S ? T : 0);
    if (R <= 1024) {
        perm_small_kernel<<<1, 256, 0, st>>>(idx, T, k, E, S, out, x, x_sorted, H);
    } else {
        const int C = (R + kPermChunk - 1) / kPermChunk;
        PermArgs a{T, k, E, S, H, idx, x, x_sorted, chunk_cnt, chunk_base, local_rank, out};
        perm_count_kernel<<<C, 256, 0, st>>>(a);
        perm_scan_kernel<<<1, 1024, 0, st>>>(a, C);
        const int grid = (R + kScatterItems - 1) / kScatterItems, nv = H / 8;
        if (!x_sorted || nv <= 256) perm_scatter_kernel<8><<<grid, 256, 0, st>>>(a);
        else if (nv <= 384) perm_scatter_kernel<12><<<grid, 256, 0, st>>>(a);
        else perm_scatter_kernel<0><<<grid, 256, 0, st>>>(a);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_perm_check(idx, T, k, E, S, out, st);
}

}  // namespace ftmoe

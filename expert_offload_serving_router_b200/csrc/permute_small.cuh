// Counting-sort building blocks shared by the fused decode route+permute kernel, the
// standalone small permute and the chunked permute's scan.
#pragma once
#include "common.cuh"

namespace ftmoe {

// In-place exclusive scan of n <= 4*blockDim ints in shared memory; returns the total.
// blockDim.x must be a multiple of 32 and <= 1024.  `tmp` needs 33 ints.
__device__ inline int block_exclusive_scan(int* data, int n, int* tmp) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    int v[4];
    int local = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int idx = tid * 4 + i;
        v[i] = idx < n ? data[idx] : 0;
        local += v[i];
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
    }
    if (lane == 31) tmp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nw ? tmp[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int u = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += u;
        }
        if (lane < nw) tmp[lane] = wi - w;   // exclusive warp offsets
        if (lane == 31) tmp[32] = wi;       // grand total
    }
    __syncthreads();
    int run = tmp[warp] + incl - local;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int idx = tid * 4 + i;
        if (idx < n) data[idx] = run;
        run += v[i];
    }
    int total = tmp[32];
    __syncthreads();
    return total;
}

struct PermOut {
    int32_t* offsets;      // [G+1]
    int32_t* sorted_flat;  // [R]
    int32_t* inv_pos;      // [R]
    int32_t* sched;        // [2 + 2*(G+1)]: total tiles (BN rows), n_active, ntile_off[G+1], active[G]
    uint32_t* err;         // device error flag
    uint32_t* ready;       // [2G] the tensor-core decode's per-group counters, zeroed here (may be null)
};

// Single-warp counting sort for decode-sized batches (R <= a few hundred pairs): no block
// barriers.  Called by one full warp; `idx_smem` holds the [T,k] routed ids, `cnt` is
// shared scratch of G+1 ints.  Same outputs as the chunked path: offsets, stable positions
// (ascending flat index within a group), active-group list and GEMM tile schedule.
__device__ inline void warp_permute_small(const int32_t* idx_smem, int T, int k, int E, int S, int* cnt, PermOut out) {
    const int lane = threadIdx.x & 31;
    const int P = T * k;
    const int R = P + (S ? T : 0);
    const int G = E + (S ? 1 : 0);
    for (int g = lane; g <= G; g += 32) cnt[g] = 0;
    if (out.ready)
        for (int g = lane; g < 2 * G; g += 32) out.ready[g] = 0u;
    __syncwarp();
    for (int i = lane; i < R; i += 32) {
        const int g = i < P ? idx_smem[i] : E;
        if (g < 0 || g >= E + (i >= P ? 1 : 0)) atomicExch(out.err, kDevErrBadExpert);
        else atomicAdd(&cnt[g], 1);
    }
    __syncwarp();
    // one pass over the groups: lane owns the contiguous block [g0, g1); exclusive scans of
    // counts (offsets), active flags (active-list rank) and 256-row tiles (tile schedule)
    const int per = (G + 31) / 32;
    const int g0 = min(G, lane * per), g1 = min(G, g0 + per);
    int sc = 0, sa = 0, st = 0;
    for (int g = g0; g < g1; ++g) {
        const int c = cnt[g];
        sc += c;
        sa += c > 0;
        st += (c + kGemmBN - 1) / kGemmBN;
    }
    int ic = sc, ia = sa, it = st;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int uc = __shfl_up_sync(0xffffffffu, ic, o);
        const int ua = __shfl_up_sync(0xffffffffu, ia, o);
        const int ut = __shfl_up_sync(0xffffffffu, it, o);
        if (lane >= o) { ic += uc; ia += ua; it += ut; }
    }
    int oc = ic - sc, oa = ia - sa, ot = it - st;       // exclusive prefixes at g0
    for (int g = g0; g < g1; ++g) {
        const int c = cnt[g];
        out.offsets[g] = oc;
        out.sched[2 + g] = ot;
        if (c > 0) out.sched[2 + (G + 1) + oa] = g;
        cnt[g] = oc;                                     // becomes the scatter cursor
        oc += c;
        oa += c > 0;
        ot += (c + kGemmBN - 1) / kGemmBN;
    }
    if (lane == 31) {
        out.offsets[G] = ic;
        out.sched[0] = it;
        out.sched[1] = ia;
        out.sched[2 + G] = it;
    }
    __syncwarp();
    // stable scatter, 32 pairs at a time in flat order: rank inside the chunk from
    // __match_any_sync, base from the group cursor, the lowest peer advances the cursor
    for (int base = 0; base < R; base += 32) {
        const int i = base + lane;
        int g = -1;
        if (i < R) {
            g = i < P ? idx_smem[i] : E;
            if (g < 0 || g >= E + (i >= P ? 1 : 0)) g = -1;
        }
        const unsigned peers = __match_any_sync(0xffffffffu, g);
        const int rk = __popc(peers & ((1u << lane) - 1u));
        int pos = 0;
        if (g >= 0) pos = cnt[g] + rk;
        __syncwarp();
        if (g >= 0 && rk == 0) cnt[g] += __popc(peers);
        __syncwarp();
        if (g >= 0) {
            out.sorted_flat[pos] = i;
            out.inv_pos[i] = pos;
        }
    }
}

}  // namespace ftmoe

// Single-CTA counting sort used for decode-sized batches (R = T*k + S*T <= a few hundred
// pairs).  Shared by the fused route+permute kernel and the standalone small permute.
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
};

// Scratch in shared memory: grp[R], cnt[G+1], flag[G+1], tmp[33].
// `idx_smem` holds the [T,k] routed ids.  Whole block participates.
__device__ inline void block_permute_small(const int32_t* idx_smem, int T, int k, int E, int S,
                                           int* grp, int* cnt, int* flag, int* tmp, PermOut out) {
    const int P = T * k;
    const int R = P + (S ? T : 0);
    const int G = E + (S ? 1 : 0);
    for (int g = threadIdx.x; g <= G; g += blockDim.x) cnt[g] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < R; i += blockDim.x) {
        int g = (i < P) ? idx_smem[i] : E;
        if (g < 0 || g >= E + (i >= P ? 1 : 0)) {  // out-of-range id: flag it, count nowhere
            atomicExch(out.err, kDevErrBadExpert);
            g = -1;
        } else {
            atomicAdd(&cnt[g], 1);
        }
        grp[i] = g;
    }
    __syncthreads();
    // active flags and tiles per group (scan inputs) before the counts are overwritten
    for (int g = threadIdx.x; g < G; g += blockDim.x) flag[g] = cnt[g] > 0 ? 1 : 0;
    __syncthreads();
    int n_active = block_exclusive_scan(flag, G, tmp);  // flag[g] = rank among active groups
    // active list; ntile counts go into the sched array directly
    for (int g = threadIdx.x; g < G; g += blockDim.x) {
        int c = cnt[g];
        if (c > 0) out.sched[2 + (G + 1) + flag[g]] = g;
        flag[g] = (c + kGemmBN - 1) / kGemmBN;
    }
    __syncthreads();
    int ntiles = block_exclusive_scan(flag, G, tmp);
    for (int g = threadIdx.x; g < G; g += blockDim.x) out.sched[2 + g] = flag[g];
    if (threadIdx.x == 0) {
        out.sched[0] = ntiles;
        out.sched[1] = n_active;
        out.sched[2 + G] = ntiles;
    }
    int total = block_exclusive_scan(cnt, G, tmp);   // cnt[g] = offsets[g]
    for (int g = threadIdx.x; g < G; g += blockDim.x) out.offsets[g] = cnt[g];
    if (threadIdx.x == 0) out.offsets[G] = total;
    // stable scatter: rank of pair i = number of earlier pairs in the same group
    for (int i = threadIdx.x; i < R; i += blockDim.x) {
        int g = grp[i];
        if (g < 0) continue;
        int r = 0;
        for (int j = 0; j < i; ++j) r += (grp[j] == g);
        int pos = cnt[g] + r;
        out.sorted_flat[pos] = i;
        out.inv_pos[i] = pos;
    }
    __syncthreads();
}

}  // namespace ftmoe

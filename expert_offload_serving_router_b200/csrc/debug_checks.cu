// Debug-bounds build (compiled with FT_DEBUG_BOUNDS=1 into libftmoe_debug.so): extra device
// checks after every counting sort and before the decode kernels read experts through a slot
// table.  A failed check raises the workspace status word (read by ft_moe_check as
// FT_ERR_DEVICE_CHECK); nothing traps and nothing waits.  In the normal build these launchers
// return at once and no kernel is compiled in.
#include "kernels.h"

namespace ftmoe {

#if FT_DEBUG_BOUNDS
// Permutation invariants: offsets start at 0, never decrease and end at the number of valid
// pairs; sorted_flat is injective into 0..R-1 with inv_pos its inverse; every pair sits in the
// group of its routed expert (the shared group E for the appended rows); flat indices ascend
// inside a group (stability).
__global__ void __launch_bounds__(1024) perm_check_kernel(const int32_t* idx, int T, int k, int E, int S, PermOut out) {
    const int P = T * k, R = P + (S ? T : 0);
    const int G = E + (S ? 1 : 0);
    const int n = out.offsets[G];
    bool bad = out.offsets[0] != 0 || n < 0 || n > R;
    for (int g = threadIdx.x; g < G && !bad; g += blockDim.x)
        if (out.offsets[g] > out.offsets[g + 1]) bad = true;
    if (!bad) {
        for (int r = threadIdx.x; r < n; r += blockDim.x) {
            const int p = out.sorted_flat[r];
            if (p < 0 || p >= R || out.inv_pos[p] != r) { bad = true; break; }
            int lo = 0, hi = G;                       // group of row r: largest g with offsets[g] <= r
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (out.offsets[mid] <= r) lo = mid; else hi = mid;
            }
            const int want = p < P ? idx[p] : E;
            if (want != lo) { bad = true; break; }
            if (r > out.offsets[lo] && out.sorted_flat[r - 1] >= p) { bad = true; break; }
        }
    }
    if (bad) atomicExch(out.err, kDevErrBounds);
}

// Every active routed group has its weight pointers in the slot table.
__global__ void slot_table_check_kernel(const int32_t* sched, int G, int E, const void* const* eptr, int mx,
                                        uint32_t* err) {
    const int n_active = sched[1];
    for (int i = threadIdx.x; i < n_active; i += blockDim.x) {
        const int g = sched[2 + (G + 1) + i];
        if (g < 0 || g >= G) { atomicExch(err, kDevErrBounds); continue; }
        if (g >= E) continue;                         // shared expert: not in the table
        if (!eptr[4 * g] || !eptr[4 * g + 2] || (mx && (!eptr[4 * g + 1] || !eptr[4 * g + 3])))
            atomicExch(err, kDevErrBounds);
    }
}
#endif

cudaError_t launch_perm_check(const int32_t* idx, int T, int k, int E, int S, const PermOut& out, cudaStream_t st) {
#if FT_DEBUG_BOUNDS
    if (T <= 0) return cudaSuccess;
    perm_check_kernel<<<1, 1024, 0, st>>>(idx, T, k, E, S, out);
    return cudaGetLastError();
#else
    (void)idx; (void)T; (void)k; (void)E; (void)S; (void)out; (void)st;
    return cudaSuccess;
#endif
}

cudaError_t launch_slot_table_check(const int32_t* sched, int G, int E, const void* const* eptr, int mx, uint32_t* err,
                                    cudaStream_t st) {
#if FT_DEBUG_BOUNDS
    if (!eptr) return cudaSuccess;
    slot_table_check_kernel<<<1, 256, 0, st>>>(sched, G, E, eptr, mx, err);
    return cudaGetLastError();
#else
    (void)sched; (void)G; (void)E; (void)eptr; (void)mx; (void)err; (void)st;
    return cudaSuccess;
#endif
}

}  // namespace ftmoe

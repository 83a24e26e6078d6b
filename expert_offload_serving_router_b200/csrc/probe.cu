// Diagnostic: a plain streaming read of device memory, for the bandwidth a kernel that does
// nothing but read reaches on transfers of a given size (the decode layer calls move 50-650 MB
// and cannot be held to the copy peak of gigabyte transfers).
#include "kernels.h"
#include "sm100.cuh"

namespace ftmoe {

// Grid-stride 16-byte loads around L1, four in flight per thread, folded into one word per
// CTA so the loads are not optimised away.
__global__ void __launch_bounds__(256) hbm_read_probe_kernel(const uint4* __restrict__ buf, size_t n16,
                                                             uint32_t* sink) {
    uint32_t acc = 0;
    const size_t stride = size_t(gridDim.x) * blockDim.x;
    size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x;
    for (; i + 3 * stride < n16; i += 4 * stride) {
        const uint4 a = ldg_nc_v4(buf + i), b = ldg_nc_v4(buf + i + stride);
        const uint4 c = ldg_nc_v4(buf + i + 2 * stride), d = ldg_nc_v4(buf + i + 3 * stride);
        acc ^= a.x ^ a.y ^ a.z ^ a.w ^ b.x ^ b.y ^ b.z ^ b.w ^ c.x ^ c.y ^ c.z ^ c.w ^ d.x ^ d.y ^ d.z ^ d.w;
    }
    for (; i < n16; i += stride) {
        const uint4 a = ldg_nc_v4(buf + i);
        acc ^= a.x ^ a.y ^ a.z ^ a.w;
    }
    acc = __reduce_xor_sync(0xffffffffu, acc);
    if ((threadIdx.x & 31) == 0 && acc == 0x9e3779b9u) atomicXor(sink, acc);   // practically never taken
}

}  // namespace ftmoe

using namespace ftmoe;

extern "C" ft_status ft_hbm_read_probe(const void* buf, size_t bytes, uint32_t* sink, int32_t ctas_per_sm,
                                       void* stream) {
    if (!buf || !sink || bytes == 0 || bytes % 16 || (reinterpret_cast<uintptr_t>(buf) & 15))
        return fail(FT_ERR_INVALID_ARG, "ft_hbm_read_probe: need a 16-byte aligned buffer, a sink and bytes %% 16 == 0");
    if (ctas_per_sm < 1 || ctas_per_sm > 8) return fail(FT_ERR_INVALID_ARG, "ft_hbm_read_probe: ctas_per_sm in 1..8");
    ft_status s = cuda_state();
    if (s) return s;
    hbm_read_probe_kernel<<<ctas_per_sm * num_sms(), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4*>(buf), bytes / 16, sink);
    return cuda_ok(cudaGetLastError(), "read probe launch");
}

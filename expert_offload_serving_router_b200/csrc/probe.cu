// Diagnostics.  hbm_read_probe: a plain streaming read of device memory, for the bandwidth a
// kernel that does nothing but read reaches on transfers of a given size (the decode layer calls
// move 50-650 MB and cannot be held to the copy peak of gigabyte transfers).  tma_read_probe:
// the rate of TMA loads of 128-byte rows into a shared-memory ring, as tiles or as row gathers
// (tile::gather4, the form a grouped GEMM would need to read token rows in place).
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

// One CTA per SM streams `tiles` tiles of 128 rows x 128 bytes through a 6-stage ring: mode 0 as
// one tile load per tile, mode 1 as 32 gather4 loads of consecutive rows, mode 2 as 32 gather4
// loads of hashed rows in [0, grows).  Only thread 0 issues and thread 32 consumes; every wait is
// bounded (a timeout sets *status and the thread returns).
constexpr int kTpSt = 6;
constexpr int kTpSlot = 16384;
__device__ __forceinline__ int tp_row(int k, int mode, int grows) {
    if (mode != 2) return k;
    uint32_t h = uint32_t(k) * 2654435761u;
    h ^= h >> 15;
    return int(h % uint32_t(grows));
}
__global__ void __launch_bounds__(64, 1) tma_read_probe_kernel(const __grid_constant__ CUtensorMap tm, int tiles, int mode,
                                                               int grows, uint32_t* status) {
    extern __shared__ __align__(1024) uint8_t tp_smem[];
    __shared__ __align__(8) uint64_t full[kTpSt], empty[kTpSt];
    uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tp_smem) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x;
    if (tid == 0) {
        for (int i = 0; i < kTpSt; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    const int row0 = blockIdx.x * tiles * 128;
    if (tid == 0) {
        for (int t = 0; t < tiles; ++t) {
            const int s = t % kTpSt;
            if (!mbar_wait(&empty[s], ((t / kTpSt) & 1) ^ 1, nullptr, 1000000000ull)) { atomicExch(status, 2u); return; }
            mbar_expect_tx(&full[s], 128u * 128u);
            uint8_t* dst = ring + s * kTpSlot;
            if (mode == 0) {
                tma_2d(&tm, &full[s], dst, 0, row0 + t * 128);
            } else {
                for (int g4 = 0; g4 < 32; ++g4) {
                    const int k = row0 + t * 128 + 4 * g4;
                    asm volatile(
                        "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
                        " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];"
                        ::"r"(su32(dst + 512 * g4)), "l"(&tm), "r"(0), "r"(tp_row(k, mode, grows)), "r"(tp_row(k + 1, mode, grows)),
                          "r"(tp_row(k + 2, mode, grows)), "r"(tp_row(k + 3, mode, grows)), "r"(su32(&full[s]))
                        : "memory");
                }
            }
        }
    } else if (tid == 32) {
        for (int t = 0; t < tiles; ++t) {
            const int s = t % kTpSt;
            if (!mbar_wait(&full[s], (t / kTpSt) & 1, nullptr, 1000000000ull)) { atomicExch(status, 3u); return; }
            mbar_arrive(&empty[s]);
        }
    }
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

extern "C" ft_status ft_tma_read_probe(int32_t mode, const void* buf, size_t bytes, size_t region_bytes, uint32_t* status,
                                       void* stream) {
    if (mode < 0 || mode > 2) return fail(FT_ERR_INVALID_ARG, "ft_tma_read_probe: mode 0 (tiles), 1 or 2 (gather4)");
    const size_t rows = bytes / 128;
    const int nsm = num_sms();
    if (!buf || !status || (reinterpret_cast<uintptr_t>(buf) & 15) || rows < size_t(128) * nsm || rows > (size_t(1) << 30))
        return fail(FT_ERR_INVALID_ARG, "ft_tma_read_probe: need a 16-byte aligned buffer of 128 x 128 x SMs .. 2^37 bytes");
    const size_t grows = region_bytes / 128;
    if (mode == 2 && (grows < 4 || grows > rows)) return fail(FT_ERR_INVALID_ARG, "ft_tma_read_probe: region within the buffer");
    ft_status s = cuda_state();
    if (s) return s;
    CUtensorMap tm{};
    uint64_t dims[2] = {128, uint64_t(rows)}, str[1] = {128};
    uint32_t box[2] = {128, mode == 0 ? 128u : 1u};     // gather4 takes a box one row high
    if (!make_map(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, buf, 2, dims, str, box))
        return fail(FT_ERR_INVALID_ARG, "ft_tma_read_probe: tensor map");
    const int tiles = int(rows / 128 / size_t(nsm));    // every CTA's rows lie inside the buffer
    const int smem = kTpSt * kTpSlot + 1024;
    static PerDeviceOnce attr;
    {
        const cudaError_t e = attr([&] { return cudaFuncSetAttribute(tma_read_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem); });
        if (e != cudaSuccess) return cuda_ok(e, "tma probe attribute");
    }
    tma_read_probe_kernel<<<nsm, 64, smem, static_cast<cudaStream_t>(stream)>>>(tm, tiles, mode, int(grows ? grows : 4), status);
    return cuda_ok(cudaGetLastError(), "tma probe launch");
}

// ft_moe_permute_noalloc: the permutation step for callers that cannot allocate
// device memory.
//
// Some callers never get to call cudaMalloc: serving engines that reserve nearly all of
// HBM for their own KV and expert pools at start-up (a later cudaMalloc would fail or
// fragment that reservation), plugins and backends that are handed only their input and
// output buffers by a host framework whose allocator owns the device, and code running
// under a fixed memory budget that must not grow.  ft_moe_permute needs a caller-sized
// workspace for its chunk counts, chunk bases and per-pair ranks; this variant keeps that
// scratch in one file-scope device array instead, so the caller passes only the inputs
// and outputs.
//
// The array (kNoAllocBytes, about 390 KB) is part of the library image: every GPU that
// loads libftmoe.so holds it until the process exits.  Its host-side name is only a
// stand-in for the symbol, never a device address: host code must not hand it to a
// kernel.  The first call on each device (with that device current) looks the device
// address up once with cudaGetSymbolAddress and caches it; make that first call before
// any stream capture.  All calls share the one array and it keeps the last call's
// contents, so calls whose work overlaps on the GPU (other streams, other host threads)
// race on it.  Nothing in it has to start at zero: every count, base, rank and schedule
// entry a call reads is written earlier in the same call.  The device status word inside the
// array (out-of-range ids, the debug-bounds build's permutation re-check) is never read back:
// on this entry point an out-of-range id shows only as offsets[E+S] < R.
#include <mutex>

#include "kernels.h"

namespace ftmoe {

constexpr int kNoAllocMaxRows = 65536;                        // T*k + S*T
constexpr int kNoAllocMaxGroups = kMaxExperts + 1;            // E + S
constexpr int kNoAllocMaxChunks = kNoAllocMaxRows / kPermChunk;
constexpr size_t kNaCnt = 0;
constexpr size_t kNaBase = kNaCnt + ((sizeof(int32_t) * kNoAllocMaxChunks * kNoAllocMaxGroups + 255) & ~size_t(255));
constexpr size_t kNaRank = kNaBase + ((sizeof(int32_t) * kNoAllocMaxChunks * kNoAllocMaxGroups + 255) & ~size_t(255));
constexpr size_t kNaSched = kNaRank + sizeof(int32_t) * kNoAllocMaxRows;
constexpr size_t kNaErr = kNaSched + ((sizeof(int32_t) * (2 + 2 * (kNoAllocMaxGroups + 1)) + 255) & ~size_t(255));
constexpr size_t kNoAllocBytes = kNaErr + 256;

static __device__ __align__(256) uint8_t g_permute_scratch[kNoAllocBytes];

constexpr int kNoAllocMaxDevices = 64;
static std::mutex g_scratch_mu;
static void* g_scratch_addr[kNoAllocMaxDevices] = {};

// Device address of g_permute_scratch on the current device, looked up once per device.  The
// cached address stays valid for the life of the device's primary context (a cudaDeviceReset
// would invalidate it).  A stream of another device than the current one is rejected: the
// address would belong to the wrong GPU.
static ft_status scratch_address(cudaStream_t stream, void** out) {
    int dev = 0;
    ft_status s = cuda_ok(cudaGetDevice(&dev), "cudaGetDevice");
    if (s) return s;
    if (stream) {
        int sdev = -1;
        if ((s = cuda_ok(cudaStreamGetDevice(stream, &sdev), "cudaStreamGetDevice"))) return s;
        if (sdev != dev)
            return fail(FT_ERR_INVALID_ARG, "ft_moe_permute_noalloc: the stream belongs to device %d but device %d is "
                        "current", sdev, dev);
    }
    if (dev < 0 || dev >= kNoAllocMaxDevices) return fail(FT_ERR_UNSUPPORTED, "device ordinal %d >= %d", dev, kNoAllocMaxDevices);
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        s = cuda_ok(cudaGetSymbolAddress(&p, g_permute_scratch), "cudaGetSymbolAddress(permute scratch)");
        if (s) return s;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return FT_OK;
}

}  // namespace ftmoe

using namespace ftmoe;

extern "C" ft_status ft_moe_permute_noalloc(const ft_moe_shape* shape, int32_t T, const int32_t* topk_idx, const void* x,
                                            int32_t* offsets, int32_t* sorted_flat, int32_t* inv_pos, void* x_sorted,
                                            void* stream) {
    ft_status s = check_shape(shape);
    if (s) return s;
    if (T < 0) return fail(FT_ERR_INVALID_ARG, "T < 0");
    const long long R = (long long)T * shape->top_k + (shape->num_shared ? T : 0);
    if (R > kNoAllocMaxRows)
        return fail(FT_ERR_UNSUPPORTED,
                    "ft_moe_permute_noalloc: %lld permuted rows exceed the static scratch limit of %d rows "
                    "(use ft_moe_permute with a workspace)", R, kNoAllocMaxRows);
    if (T == 0) return FT_OK;
    if (!topk_idx || !offsets || !sorted_flat || !inv_pos) return fail(FT_ERR_INVALID_ARG, "NULL permutation pointer");
    if (x_sorted && (!x || (reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(x_sorted) & 15)))
        return fail(FT_ERR_INVALID_ARG, "x_sorted needs a 16-byte aligned x and x_sorted");
    if ((s = cuda_state())) return s;
    void* base = nullptr;
    if ((s = scratch_address(static_cast<cudaStream_t>(stream), &base))) return s;
    PermOut po{offsets, sorted_flat, inv_pos, ws_at<int32_t>(base, kNaSched), ws_at<uint32_t>(base, kNaErr)};
    return cuda_ok(launch_permute(T, shape->top_k, shape->num_experts, shape->num_shared, shape->hidden, topk_idx,
                                  static_cast<const uint16_t*>(x), static_cast<uint16_t*>(x_sorted),
                                  ws_at<int32_t>(base, kNaCnt), ws_at<int32_t>(base, kNaBase),
                                  ws_at<int32_t>(base, kNaRank), po, static_cast<cudaStream_t>(stream)),
                   "permute (static scratch) launch");
}

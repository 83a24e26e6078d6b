// Internal launcher declarations shared by the kernel files and the C-ABI layer.
#pragma once
#include "common.cuh"
#include <nvtx3/nvToolsExt.h>
#include "permute_small.cuh"

namespace ftmoe {

// NVTX range around one public entry point (named in profiler timelines; no cost without a
// profiler attached).
struct TraceRange {
    explicit TraceRange(const char* name) { nvtxRangePushA(name); }
    ~TraceRange() { nvtxRangePop(); }
    TraceRange(const TraceRange&) = delete;
    TraceRange& operator=(const TraceRange&) = delete;
};
#define FT_TRACE(name) ::ftmoe::TraceRange ft_trace_range_(name)


struct DecodeArgs {
    int T, k, E, S, H, F, wdtype;
    const uint16_t* x;
    const int32_t* offsets;
    const int32_t* sorted_flat;
    const int32_t* sched;       // [1] n_active, active list at [2 + G + 1 ...]
    const uint8_t* w13;
    const uint8_t* w13s;
    const uint8_t* w2;
    const uint8_t* w2s;
    const void* const* eptr;    // optional [E][4] {w13, w13s, w2, w2s}
    const uint8_t* sw13;
    const uint8_t* sw13s;
    const uint8_t* sw2;
    const uint8_t* sw2s;
    uint16_t* h;                // [R, F]
    const int32_t* inv_pos;
    const float* topk_w;
    uint16_t* y;                // [T, H] or NULL
    uint16_t* o_sorted;         // [R, H] when y == NULL
    uint32_t* err;              // workspace device error flag
    uint16_t* o_ws;             // workspace [R, H] rows for the tensor-core decode's combine
    uint8_t* mx_ws;             // workspace scratch of the block-scaled MXFP4 decode (activation planes)
};

struct GemmLaunch {
    int mode;                 // 0 gate/up, 1 down
    int wdtype;
    int H, F, E, S, R;        // R = rows of the activation operand
    const void* w;            // bf16 weights or MXFP4 codes (routed)
    const uint8_t* wscale;
    const void* sw;           // shared expert weights / codes (S=1)
    const uint8_t* swscale;
    const void* act;          // x_sorted [R,H] (gate/up) or h [R,F] (down), bf16
    const int32_t* offsets;
    const int32_t* sched;
    uint16_t* out;
    uint32_t* err;
    int max_tiles;            // host upper bound on tiles (grid sizing)
};

template <class T> inline T* ws_at(void* ws, size_t off) { return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off); }

// host helpers of the C-ABI layer (api.cu)
ft_status fail(ft_status s, const char* fmt, ...);
ft_status check_shape(const ft_moe_shape* s);
ft_status cuda_ok(cudaError_t e, const char* what);
ft_status cuda_state();
DecodeArgs decode_args(const ft_moe_shape* s, int T, const ft_moe_weights* w, const void* x, const WsLayout& L,
                       void* ws, const int32_t* offsets, const int32_t* sorted_flat, const int32_t* inv_pos,
                       const float* topk_w, void* y, void* o_sorted);

// err: the workspace's device error word ([0] flag, [1] decode-router ticket); planes: the
// workspace's router-plane region and part its split-K partials (used when T > kSmallRoute).  `perm` (fused counting
// sort) is only taken by the decode-sized path.
cudaError_t launch_route(int T, int H, int E, int k, int S, const uint16_t* x, const float* wr, const float* bias,
                         int32_t* topk_idx, float* topk_w, float* logits, uint32_t* err, uint16_t* planes,
                         float* part, const PermOut* perm, cudaStream_t st);
cudaError_t launch_route_tc(int T, int H, int E, int k, const uint16_t* x, const float* wr, const float* bias,
                            int32_t* topk_idx, float* topk_w, float* logits, uint16_t* planes, float* part,
                            uint32_t* err, cudaStream_t st);
// debug-bounds build only (no-ops otherwise): permutation invariants, decode slot table
cudaError_t launch_perm_check(const int32_t* idx, int T, int k, int E, int S, const PermOut& out, cudaStream_t st);
cudaError_t launch_slot_table_check(const int32_t* sched, int G, int E, const void* const* eptr, int mx, uint32_t* err,
                                    cudaStream_t st);
cudaError_t launch_permute(int T, int k, int E, int S, int H, const int32_t* idx, const uint16_t* x,
                           uint16_t* x_sorted, int32_t* chunk_cnt, int32_t* chunk_base, int32_t* local_rank,
                           const PermOut& out, cudaStream_t st);
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st);
// the kernels launch_decode runs for a batch (decode.cu): one choice, used for the launch and for
// the kernel count ft_moe_decode_kernels reports
enum DecodePath { kDecodeGemv, kDecodeMma, kDecodeMxFused, kDecodeMxTwo };
DecodePath decode_path(const DecodeArgs& a);
int decode_path_kernels(DecodePath p, bool combine);   // kernels launched (combine: y != NULL)
// tensor-core decode (BF16, contiguous weights): false when the shape or weights do not qualify
bool decode_mma_eligible(const DecodeArgs& a);
cudaError_t launch_decode_mma(const DecodeArgs& a, cudaStream_t st);
// block-scaled MXFP4 decode on the tensor cores (decode_mx_mma.cu)
bool decode_mx_eligible(const DecodeArgs& a);
bool decode_mx_fused(const DecodeArgs& a);   // gate/up and down in one launch (else two)
cudaError_t launch_decode_mx(const DecodeArgs& a, cudaStream_t st);
bool block_scaled_decode(int T);   // api.cu: ft_set_block_scaled_decode
int launch_moe_gemm(const GemmLaunch& L, cudaStream_t st);
// bound (ns without progress) on each pipeline wait of the grouped GEMMs (api.cu)
unsigned long long gemm_wait_ns();
cudaError_t launch_combine(int T, int H, int k, int S, int R, const uint16_t* o, const int32_t* inv_pos,
                           const float* gw, uint16_t* y, cudaStream_t st);
cudaError_t launch_combine_dependent(int T, int H, int k, int S, int R, const uint16_t* o, const int32_t* inv_pos,
                           const float* gw, uint16_t* y, cudaStream_t st);   // PDL-launched after a decode expert kernel
cudaError_t launch_unit_rms(int T, int H, const uint16_t* in, uint16_t* out, float eps, cudaStream_t st);

}  // namespace ftmoe

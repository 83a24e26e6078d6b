// C-ABI entry points of libftmoe.so: argument validation on the host (before any CUDA
// call), workspace carving, and the launch order of the layer's kernels on the caller's
// stream.  No entry point allocates device memory or synchronises, except ft_moe_check.
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <string>

#include "kernels.h"
#include "sm100.cuh"

namespace ftmoe {

static thread_local std::string g_err;

ft_status fail(ft_status s, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return s;
}

static int init_decode_max() {
    const char* v = getenv("FT_DECODE_MAX_TOKENS");
    int d = 32;
    if (v && *v) {
        d = atoi(v);
        if (d < 0) d = 0;
        if (d > kSmallRoute) d = kSmallRoute;
    }
    return d;
}
static int g_decode_max = init_decode_max();
int decode_max() { return g_decode_max; }

// 0 never, 1 every eligible decode batch, 2 (default) eligible batches of kBlockScaledMinT+ tokens
static int g_block_scaled_decode = 2;
constexpr int kBlockScaledMinT = 4;
bool block_scaled_decode(int T) {
    return g_block_scaled_decode == 1 || (g_block_scaled_decode == 2 && T >= kBlockScaledMinT);
}

static unsigned long long g_gemm_wait_ns = kWaitNs;
unsigned long long gemm_wait_ns() { return g_gemm_wait_ns; }

static bool al(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

ft_status check_shape(const ft_moe_shape* s) {
    if (!s) return fail(FT_ERR_INVALID_ARG, "shape is NULL");
    if (s->hidden <= 0 || s->ffn <= 0 || s->num_experts <= 0 || s->top_k <= 0)
        return fail(FT_ERR_INVALID_ARG, "non-positive shape field (H=%d F=%d E=%d k=%d)", s->hidden, s->ffn,
                    s->num_experts, s->top_k);
    if (s->num_shared != 0 && s->num_shared != 1) return fail(FT_ERR_INVALID_ARG, "num_shared must be 0 or 1");
    if (s->wdtype != FT_W_BF16 && s->wdtype != FT_W_MXFP4) return fail(FT_ERR_INVALID_ARG, "unknown wdtype %d", s->wdtype);
    if (s->hidden % 128 || s->hidden > 16384) return fail(FT_ERR_UNSUPPORTED, "hidden %d: need H %% 128 == 0, H <= 16384", s->hidden);
    if (s->ffn % 64 || s->ffn > 4096) return fail(FT_ERR_UNSUPPORTED, "ffn %d: need F %% 64 == 0, F <= 4096", s->ffn);
    if (s->num_experts > kMaxExperts) return fail(FT_ERR_UNSUPPORTED, "num_experts %d > %d", s->num_experts, kMaxExperts);
    if (s->top_k > kMaxTopK || s->top_k > s->num_experts)
        return fail(FT_ERR_UNSUPPORTED, "top_k %d: need k <= 8 and k <= E", s->top_k);
    return FT_OK;
}

ft_status check_ws(const ft_moe_shape* s, int T, const void* ws, size_t ws_bytes, WsLayout* out) {
    WsLayout L = make_layout(*s, T);
    if (!ws) return fail(FT_ERR_INVALID_ARG, "workspace is NULL");
    if (!al(ws, 256)) return fail(FT_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    if (ws_bytes < L.total)
        return fail(FT_ERR_WORKSPACE, "workspace %zu bytes < %zu needed for T=%d", ws_bytes, L.total, T);
    if (out) *out = L;
    return FT_OK;
}

ft_status cuda_ok(cudaError_t e, const char* what) {
    if (e == cudaSuccess) return FT_OK;
    return fail(FT_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// a sticky error from earlier asynchronous work shows up here
ft_status cuda_state() {
    cudaError_t e = cudaGetLastError();
    return cuda_ok(e, "pending CUDA error");
}


ft_status check_weights(const ft_moe_shape* s, const ft_moe_weights* w, bool need_contig) {
    if (!w) return fail(FT_ERR_INVALID_ARG, "weights is NULL");
    const bool mx = s->wdtype == FT_W_MXFP4;
    if (w->expert_ptrs) {
        if (need_contig) return fail(FT_ERR_UNSUPPORTED, "expert_ptrs tables are only supported on the decode path");
        if (!al(w->expert_ptrs, 8)) return fail(FT_ERR_INVALID_ARG, "expert_ptrs must be 8-byte aligned");
    } else {
        if (!w->w13 || !w->w2) return fail(FT_ERR_INVALID_ARG, "w13/w2 are NULL");
        if (!al(w->w13, 16) || !al(w->w2, 16)) return fail(FT_ERR_INVALID_ARG, "w13/w2 must be 16-byte aligned");
        if (mx && (!w->w13_scale || !w->w2_scale)) return fail(FT_ERR_INVALID_ARG, "MXFP4 scales are NULL");
        if (mx && (!al(w->w13_scale, 2) || !al(w->w2_scale, 2))) return fail(FT_ERR_INVALID_ARG, "MXFP4 scales must be 2-byte aligned");
    }
    if (s->num_shared) {
        if (!w->shared_w13 || !w->shared_w2) return fail(FT_ERR_INVALID_ARG, "shared expert weights are NULL");
        if (!al(w->shared_w13, 16) || !al(w->shared_w2, 16)) return fail(FT_ERR_INVALID_ARG, "shared weights must be 16-byte aligned");
        if (mx && (!w->shared_w13_scale || !w->shared_w2_scale)) return fail(FT_ERR_INVALID_ARG, "shared MXFP4 scales are NULL");
    }
    return FT_OK;
}

DecodeArgs decode_args(const ft_moe_shape* s, int T, const ft_moe_weights* w, const void* x, const WsLayout& L,
                       void* ws, const int32_t* offsets, const int32_t* sorted_flat, const int32_t* inv_pos,
                       const float* topk_w, void* y, void* o_sorted) {
    DecodeArgs a{};
    a.T = T; a.k = s->top_k; a.E = s->num_experts; a.S = s->num_shared; a.H = s->hidden; a.F = s->ffn;
    a.wdtype = s->wdtype;
    a.x = static_cast<const uint16_t*>(x);
    a.offsets = offsets;
    a.sorted_flat = sorted_flat;
    a.sched = ws_at<int32_t>(ws, L.sched);
    a.w13 = static_cast<const uint8_t*>(w->w13);
    a.w13s = w->w13_scale;
    a.w2 = static_cast<const uint8_t*>(w->w2);
    a.w2s = w->w2_scale;
    a.eptr = w->expert_ptrs;
    a.sw13 = static_cast<const uint8_t*>(w->shared_w13);
    a.sw13s = w->shared_w13_scale;
    a.sw2 = static_cast<const uint8_t*>(w->shared_w2);
    a.sw2s = w->shared_w2_scale;
    a.h = ws_at<uint16_t>(ws, L.h);
    a.inv_pos = inv_pos;
    a.topk_w = topk_w;
    a.y = static_cast<uint16_t*>(y);
    a.o_sorted = static_cast<uint16_t*>(o_sorted);
    a.err = ws_at<uint32_t>(ws, L.err);
    a.o_ws = ws_at<uint16_t>(ws, L.o_sorted);
    a.mx_ws = ws_at<uint8_t>(ws, L.mx_decode);
    return a;
}

// one grouped GEMM stage: mode 0 gate/up (act = x_sorted, out = h), mode 1 down (act = h, out = o_sorted)
ft_status run_gemm_stage(int mode, const ft_moe_shape* s, const ft_moe_weights* w, const void* act,
                         const int32_t* offsets, void* out, const WsLayout& L, void* ws, cudaStream_t st) {
    GemmLaunch g{};
    g.mode = mode;
    g.wdtype = s->wdtype;
    g.H = s->hidden; g.F = s->ffn; g.E = s->num_experts; g.S = s->num_shared; g.R = L.R;
    g.offsets = offsets;
    g.sched = ws_at<int32_t>(ws, L.sched);
    g.err = ws_at<uint32_t>(ws, L.err);
    g.max_tiles = L.G + L.R / kGemmBN + 1;
    if (mode == 0) { g.w = w->w13; g.wscale = w->w13_scale; g.sw = w->shared_w13; g.swscale = w->shared_w13_scale; }
    else { g.w = w->w2; g.wscale = w->w2_scale; g.sw = w->shared_w2; g.swscale = w->shared_w2_scale; }
    g.act = act;
    g.out = static_cast<uint16_t*>(out);
    int r = launch_moe_gemm(g, st);
    if (r == 1) return fail(FT_ERR_CUDA, "cuTensorMapEncodeTiled failed (%s)", mode ? "down" : "gate/up");
    if (r) return cuda_ok(cudaGetLastError(), mode ? "down grouped GEMM launch" : "gate/up grouped GEMM launch");
    return FT_OK;
}

ft_status run_gemm_experts(const ft_moe_shape* s, const ft_moe_weights* w, const void* x_sorted,
                           const int32_t* offsets, void* o_sorted, const WsLayout& L, void* ws, cudaStream_t st) {
    uint16_t* h = ws_at<uint16_t>(ws, L.h);
    ft_status r = run_gemm_stage(0, s, w, x_sorted, offsets, h, L, ws, st);
    if (r) return r;
    return run_gemm_stage(1, s, w, h, offsets, o_sorted, L, ws, st);
}

}  // namespace ftmoe

using namespace ftmoe;

extern "C" {

const char* ft_last_error(void) { return g_err.c_str(); }

const char* ft_version(void) { return "ftmoe 0.1.0 (sm_100a: tcgen05 grouped GEMM, SIMT decode GEMV)"; }

int32_t ft_set_decode_max_tokens(int32_t t) {
    if (t < 0) return -1;
    int prev = g_decode_max;
    g_decode_max = t > kSmallRoute ? kSmallRoute : t;
    return prev;
}

int32_t ft_get_decode_max_tokens(void) { return g_decode_max; }

int32_t ft_set_block_scaled_decode(int32_t mode) {
    if (mode < 0 || mode > 2) return -1;
    const int32_t prev = g_block_scaled_decode;
    g_block_scaled_decode = mode;
    return prev;
}

int32_t ft_moe_decode_kernels(const ft_moe_shape* shape, int32_t T) {
    if (check_shape(shape) != FT_OK || T < 0) return -1;
    if (T == 0 || T > g_decode_max) return 0;
    DecodeArgs a{};
    a.T = T; a.k = shape->top_k; a.E = shape->num_experts; a.S = shape->num_shared;
    a.H = shape->hidden; a.F = shape->ffn; a.wdtype = shape->wdtype;
    int n = 1 + decode_path_kernels(decode_path(a), true);   // the router, then the experts
#if FT_DEBUG_BOUNDS
    n += 1;                                                  // the permutation check
#endif
    return n;
}

uint64_t ft_set_pipeline_wait_limit_ns(uint64_t ns) {
    const unsigned long long prev = g_gemm_wait_ns;
    g_gemm_wait_ns = ns ? ns : kWaitNs;
    return prev;
}

size_t ft_moe_workspace_bytes(const ft_moe_shape* shape, int32_t max_tokens) {
    if (check_shape(shape) != FT_OK || max_tokens < 0) return 0;
    return make_layout(*shape, max_tokens).total;
}

ft_status ft_moe_workspace_init(void* ws, size_t ws_bytes, void* stream) {
    if (!ws || ws_bytes < kWsHeaderBytes) return fail(FT_ERR_INVALID_ARG, "workspace NULL or smaller than its %zu-byte header", kWsHeaderBytes);
    if (!al(ws, 256)) return fail(FT_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    ft_status st = cuda_state();
    if (st) return st;
    return cuda_ok(cudaMemsetAsync(ws, 0, kWsHeaderBytes, static_cast<cudaStream_t>(stream)), "cudaMemsetAsync(ws header)");
}

ft_status ft_moe_check(void* ws, void* stream) {
    FT_TRACE("ft_moe_check");
    if (!ws) return fail(FT_ERR_INVALID_ARG, "workspace is NULL");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    ft_status s = cuda_ok(cudaStreamSynchronize(st), "stream synchronize");
    if (s) return s;
    uint32_t flag = 0;
    s = cuda_ok(cudaMemcpy(&flag, ws, sizeof flag, cudaMemcpyDeviceToHost), "read device status");
    if (s) return s;
    if (flag) {
        cudaMemset(ws, 0, sizeof flag);
        return fail(FT_ERR_DEVICE_CHECK, flag == kDevErrBadExpert ? "a routed expert id was outside [0, E)"
                                         : flag == kDevErrTimeout ? "a grouped-GEMM pipeline wait timed out"
                                         : flag == kDevErrBounds  ? "a debug-bounds check failed (permutation or slot table)"
                                                                  : "device check failed (code %u)", flag);
    }
    return FT_OK;
}

ft_status ft_moe_route(const ft_moe_shape* shape, int32_t T, const void* x, const float* w_router, const float* bias,
                       int32_t* topk_idx, float* topk_w, float* logits, void* ws, size_t ws_bytes, void* stream) {
    FT_TRACE("ft_moe_route");
    ft_status s = check_shape(shape);
    if (s) return s;
    if (T < 0) return fail(FT_ERR_INVALID_ARG, "T < 0");
    if (T == 0) return FT_OK;
    if (!x || !w_router || !topk_idx || !topk_w) return fail(FT_ERR_INVALID_ARG, "NULL input/output pointer");
    if (!al(x, 16) || !al(w_router, 16)) return fail(FT_ERR_INVALID_ARG, "x and w_router must be 16-byte aligned");
    WsLayout L;
    if ((s = check_ws(shape, T, ws, ws_bytes, &L))) return s;
    if ((s = cuda_state())) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t* err = ws_at<uint32_t>(ws, L.err);   // err[1]: decode-router ticket, zero between calls
    float* lg = logits ? logits : ws_at<float>(ws, L.logits);
    return cuda_ok(launch_route(T, shape->hidden, shape->num_experts, shape->top_k, shape->num_shared,
                                static_cast<const uint16_t*>(x), w_router, bias, topk_idx, topk_w, lg, err,
                                ws_at<uint16_t>(ws, L.wr_planes), ws_at<float>(ws, L.route_part), nullptr, st),
                   "route launch");
}

ft_status ft_moe_permute(const ft_moe_shape* shape, int32_t T, const int32_t* topk_idx, const void* x, int32_t* offsets,
                         int32_t* sorted_flat, int32_t* inv_pos, void* x_sorted, void* ws, size_t ws_bytes,
                         void* stream) {
    FT_TRACE("ft_moe_permute");
    ft_status s = check_shape(shape);
    if (s) return s;
    if (T < 0) return fail(FT_ERR_INVALID_ARG, "T < 0");
    if (T == 0) return FT_OK;
    if (!topk_idx || !offsets || !sorted_flat || !inv_pos) return fail(FT_ERR_INVALID_ARG, "NULL permutation pointer");
    if (x_sorted && (!x || !al(x, 16) || !al(x_sorted, 16)))
        return fail(FT_ERR_INVALID_ARG, "x_sorted needs a 16-byte aligned x and x_sorted");
    WsLayout L;
    if ((s = check_ws(shape, T, ws, ws_bytes, &L))) return s;
    if ((s = cuda_state())) return s;
    PermOut po{offsets, sorted_flat, inv_pos, ws_at<int32_t>(ws, L.sched), ws_at<uint32_t>(ws, L.err),
               ws_at<uint32_t>(ws, L.err) + kWsReady};
    return cuda_ok(launch_permute(T, shape->top_k, shape->num_experts, shape->num_shared, shape->hidden, topk_idx,
                                  static_cast<const uint16_t*>(x), static_cast<uint16_t*>(x_sorted),
                                  ws_at<int32_t>(ws, L.chunk_cnt), ws_at<int32_t>(ws, L.chunk_base),
                                  ws_at<int32_t>(ws, L.local_rank), po, static_cast<cudaStream_t>(stream)),
                   "permute launch");
}

ft_status ft_moe_experts(const ft_moe_shape* shape, int32_t T, const ft_moe_weights* weights, const void* x,
                         const void* x_sorted, const int32_t* offsets, const int32_t* sorted_flat, void* o_sorted,
                         void* ws, size_t ws_bytes, void* stream) {
    FT_TRACE("ft_moe_experts");
    ft_status s = check_shape(shape);
    if (s) return s;
    if (T < 0) return fail(FT_ERR_INVALID_ARG, "T < 0");
    if (T == 0) return FT_OK;
    const bool decode = T <= g_decode_max;
    if ((s = check_weights(shape, weights, !decode))) return s;
    if (!offsets || !sorted_flat || !o_sorted) return fail(FT_ERR_INVALID_ARG, "NULL permutation/output pointer");
    if (decode && (!x || !al(x, 16))) return fail(FT_ERR_INVALID_ARG, "decode path needs a 16-byte aligned x");
    if (!decode && (!x_sorted || !al(x_sorted, 16))) return fail(FT_ERR_INVALID_ARG, "grouped GEMM path needs x_sorted");
    if (!al(o_sorted, 16)) return fail(FT_ERR_INVALID_ARG, "o_sorted must be 16-byte aligned");
    WsLayout L;
    if ((s = check_ws(shape, T, ws, ws_bytes, &L))) return s;
    if ((s = cuda_state())) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (decode) {
        DecodeArgs a = decode_args(shape, T, weights, x, L, ws, offsets, sorted_flat, nullptr, nullptr, nullptr, o_sorted);
        return cuda_ok(launch_decode(a, st), "decode experts launch");
    }
    return run_gemm_experts(shape, weights, x_sorted, offsets, o_sorted, L, ws, st);
}

static ft_status gemm_stage_entry(int mode, const ft_moe_shape* shape, int32_t T, const ft_moe_weights* weights,
                                 const void* act, const int32_t* offsets, void* out, void* ws, size_t ws_bytes,
                                 void* stream) {
    ft_status s = check_shape(shape);
    if (s) return s;
    if (T < 0) return fail(FT_ERR_INVALID_ARG, "T < 0");
    if (T == 0) return FT_OK;
    if (T <= g_decode_max)
        return fail(FT_ERR_UNSUPPORTED, "grouped GEMM stages need T > decode threshold (%d); use ft_moe_experts", g_decode_max);
    if ((s = check_weights(shape, weights, true))) return s;
    if (!act || !offsets || !out || !al(act, 16) || !al(out, 16))
        return fail(FT_ERR_INVALID_ARG, "NULL or misaligned activation/offsets/output pointer");
    WsLayout L;
    if ((s = check_ws(shape, T, ws, ws_bytes, &L))) return s;
    if ((s = cuda_state())) return s;
    return run_gemm_stage(mode, shape, weights, act, offsets, out, L, ws, static_cast<cudaStream_t>(stream));
}

ft_status ft_moe_experts_gateup(const ft_moe_shape* shape, int32_t T, const ft_moe_weights* weights,
                                const void* x_sorted, const int32_t* offsets, void* h, void* ws, size_t ws_bytes,
                                void* stream) {
    FT_TRACE("ft_moe_experts_gateup");
    return gemm_stage_entry(0, shape, T, weights, x_sorted, offsets, h, ws, ws_bytes, stream);
}

ft_status ft_moe_experts_down(const ft_moe_shape* shape, int32_t T, const ft_moe_weights* weights, const void* h,
                              const int32_t* offsets, void* o_sorted, void* ws, size_t ws_bytes, void* stream) {
    FT_TRACE("ft_moe_experts_down");
    return gemm_stage_entry(1, shape, T, weights, h, offsets, o_sorted, ws, ws_bytes, stream);
}

ft_status ft_moe_combine(const ft_moe_shape* shape, int32_t T, const void* o_sorted, const int32_t* inv_pos,
                         const float* topk_w, void* y, void* stream) {
    FT_TRACE("ft_moe_combine");
    ft_status s = check_shape(shape);
    if (s) return s;
    if (T < 0) return fail(FT_ERR_INVALID_ARG, "T < 0");
    if (T == 0) return FT_OK;
    if (!o_sorted || !inv_pos || !topk_w || !y) return fail(FT_ERR_INVALID_ARG, "NULL pointer");
    if (!al(o_sorted, 16) || !al(y, 16)) return fail(FT_ERR_INVALID_ARG, "o_sorted and y must be 16-byte aligned");
    if ((s = cuda_state())) return s;
    const int R = T * shape->top_k + (shape->num_shared ? T : 0);
    return cuda_ok(launch_combine(T, shape->hidden, shape->top_k, shape->num_shared, R,
                                  static_cast<const uint16_t*>(o_sorted), inv_pos, topk_w, static_cast<uint16_t*>(y),
                                  static_cast<cudaStream_t>(stream)),
                   "combine launch");
}

ft_status ft_moe_layer_forward(const ft_moe_shape* shape, int32_t T, const void* x, const float* w_router,
                               const float* bias, const ft_moe_weights* weights, void* y, int32_t* topk_idx_out,
                               float* logits_out, void* ws, size_t ws_bytes, void* stream) {
    FT_TRACE("ft_moe_layer_forward");
    ft_status s = check_shape(shape);
    if (s) return s;
    if (T < 0) return fail(FT_ERR_INVALID_ARG, "T < 0");
    if (T == 0) return FT_OK;
    const bool decode = T <= g_decode_max;
    if (!x || !w_router || !y) return fail(FT_ERR_INVALID_ARG, "NULL x, w_router or y");
    if (!al(x, 16) || !al(w_router, 16) || !al(y, 16)) return fail(FT_ERR_INVALID_ARG, "x, w_router, y must be 16-byte aligned");
    if ((s = check_weights(shape, weights, !decode))) return s;
    WsLayout L;
    if ((s = check_ws(shape, T, ws, ws_bytes, &L))) return s;
    if ((s = cuda_state())) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int H = shape->hidden, E = shape->num_experts, k = shape->top_k, S = shape->num_shared;
    uint32_t* err = ws_at<uint32_t>(ws, L.err);
    int32_t* idx = topk_idx_out ? topk_idx_out : ws_at<int32_t>(ws, L.topk_idx);
    float* gw = ws_at<float>(ws, L.topk_w);
    float* lg = logits_out ? logits_out : ws_at<float>(ws, L.logits);
    int32_t* offsets = ws_at<int32_t>(ws, L.offsets);
    int32_t* sorted_flat = ws_at<int32_t>(ws, L.sorted_flat);
    int32_t* inv_pos = ws_at<int32_t>(ws, L.inv_pos);
    PermOut po{offsets, sorted_flat, inv_pos, ws_at<int32_t>(ws, L.sched), err, err + kWsReady};
    const uint16_t* xb = static_cast<const uint16_t*>(x);
    if (decode) {
        // route + top-k + permutation in one launch, then two weight-streaming kernels
        if ((s = cuda_ok(launch_route(T, H, E, k, S, xb, w_router, bias, idx, gw, lg, err, ws_at<uint16_t>(ws, L.wr_planes), ws_at<float>(ws, L.route_part), &po, st), "route launch")))
            return s;
        DecodeArgs a = decode_args(shape, T, weights, x, L, ws, offsets, sorted_flat, inv_pos, gw, y, nullptr);
        return cuda_ok(launch_decode(a, st), "decode experts launch");
    }
    if ((s = cuda_ok(launch_route(T, H, E, k, S, xb, w_router, bias, idx, gw, lg, err, ws_at<uint16_t>(ws, L.wr_planes), ws_at<float>(ws, L.route_part), nullptr, st), "route launch")))
        return s;
    uint16_t* xs = ws_at<uint16_t>(ws, L.x_sorted);
    if ((s = cuda_ok(launch_permute(T, k, E, S, H, idx, xb, xs, ws_at<int32_t>(ws, L.chunk_cnt),
                                    ws_at<int32_t>(ws, L.chunk_base), ws_at<int32_t>(ws, L.local_rank), po, st),
                     "permute launch")))
        return s;
    uint16_t* os = ws_at<uint16_t>(ws, L.o_sorted);
    if ((s = run_gemm_experts(shape, weights, xs, offsets, os, L, ws, st))) return s;
    return cuda_ok(launch_combine(T, H, k, S, L.R, os, inv_pos, gw, static_cast<uint16_t*>(y), st), "combine launch");
}

ft_status ft_moe_unit_rms(int32_t T, int32_t H, const void* in, void* out, float eps, void* stream) {
    FT_TRACE("ft_moe_unit_rms");
    if (T < 0 || H <= 0 || H % 8) return fail(FT_ERR_INVALID_ARG, "need T >= 0 and H a positive multiple of 8");
    if (T == 0) return FT_OK;
    if (!in || !out || !al(in, 16) || !al(out, 16)) return fail(FT_ERR_INVALID_ARG, "in/out NULL or not 16-byte aligned");
    ft_status s = cuda_state();
    if (s) return s;
    return cuda_ok(launch_unit_rms(T, H, static_cast<const uint16_t*>(in), static_cast<uint16_t*>(out), eps,
                                   static_cast<cudaStream_t>(stream)),
                   "unit_rms launch");
}

}  // extern "C"

/*
 * ftmoe.h -- C ABI of libftmoe.so: the forward pass of one sparse
 * Mixture-of-Experts FFN layer on one B200 (sm_100a), plus a host-resident
 * expert stream (double-buffered layer prefetch and an LRU expert-slot cache).
 *
 * What the layer computes (per token t, with T tokens, hidden size H, expert
 * FFN width F, E routed experts, top-k, S in {0,1} shared experts):
 *   1. route:   l[t,e] = sum_h x[t,h] * Wr[e,h] + b[e]  (fp32 accumulation);
 *               keep the k largest logits, ties to the lower expert index,
 *               slot order = descending logit;
 *               g[t,j] = softmax over the k kept logits (equal to the full
 *               softmax restricted to the k kept and renormalised).
 *   2. permute: stable counting sort of flat pairs p = t*k + j by expert;
 *               the shared expert (S = 1) is group E holding every token.
 *   3. experts: per expert e and routed row r: h = silu(Wg_e x) * (Wu_e x),
 *               o = Wd_e h  (SwiGLU; gate rows 0..F-1 of w13, up rows F..2F-1).
 *   4. combine: y[t] = sum_j g[t,j] * o[t,j] (+ o_shared[t]), fp32 in j order,
 *               one round-to-nearest-even to bf16.
 * The pages this library follows describe k-of-E routed experts ("6 of 256
 * routed experts in each of 43 layers": FreeToken write-up, aihot.vn, "The
 * gap it targets"), one shared expert beside 8 routed ones (TurboFieldfare
 * article, dothoosh.com, "Background: Gemma 4 26B A4B"), BF16 and MXFP4
 * expert weights (FreeToken article, dothoosh.com, "Benchmarks"), full-layer
 * double buffering during prefill and a router-following LRU expert cache in
 * decode that starts cold (FreeToken article, dothoosh.com, "FreeToken
 * architecture", mechanisms 2 and 3).  They print no formula for the layer;
 * the definitions above are the plain reading.  MXFP4 follows the OCP
 * Microscaling Formats v1.0 spec: E2M1 codes, one E8M0 scale per 32
 * consecutive elements along the contraction dimension.
 *
 * Conventions (every entry point):
 *   - Pointers marked "device" are CUDA device pointers, "host" are host
 *     pointers.  All buffers are owned by the caller; the library never
 *     allocates device memory.  Scratch is passed as (ws, ws_bytes), sized by
 *     ft_moe_workspace_bytes(); ws must be 256-byte aligned.
 *   - All work is enqueued on the caller's stream (`stream` is a
 *     cudaStream_t passed as void*; NULL = legacy default stream).  No call
 *     synchronises the host, except where stated.
 *   - Errors are return codes; ft_last_error() gives a thread-local message.
 *     Argument errors are detected on the host before any CUDA call.  An
 *     asynchronous CUDA error from earlier work surfaces as FT_ERR_CUDA.
 *   - Supported shapes: H % 128 == 0, H <= 16384, F % 64 == 0, F <= 4096,
 *     1 <= k <= 8, k <= E <= 256, S in {0, 1} (FT_ERR_UNSUPPORTED otherwise):
 *     the grouped GEMMs tile weights in groups of 128 rows (64 gate + 64 up
 *     rows for gate/up, 128 hidden rows for down).  MXFP4 additionally needs
 *     H % 32 == 0 and F % 32 == 0 (implied).  T may be 0 (nothing is
 *     launched).  Larger T than the max_tokens the workspace was sized for
 *     returns FT_ERR_WORKSPACE.
 *   - Activation precision: x, h and y are bf16 and every product is exact
 *     with fp32 accumulation, except on the decode path (T <= threshold) with
 *     MXFP4 weights, where the GEMVs multiply in f16: the activations (x, and
 *     h for the down projection) are rounded to f16 there, which is exact for
 *     2^-17 <= |v| <= 65504; |v| > 65504 becomes +-inf and below 2^-17 the
 *     absolute error is at most 2^-25.  The grouped GEMM path (prefill) keeps
 *     bf16 activations.
 *
 * Layouts (all row-major, innermost dimension last):
 *   x        [T, H]  bf16           topk_idx [T, k] int32     topk_w [T, k] fp32
 *   w_router [E, H]  fp32           bias     [E]    fp32 (or NULL)
 *   logits   [T, E]  fp32
 *   BF16 weights:  w13 [E, 2F, H] bf16, w2 [E, H, F] bf16
 *   MXFP4 weights: w13 codes [E, 2F, H/2] u8 + w13_scale [E, 2F, H/32] u8,
 *                  w2 codes [E, H, F/2] u8 + w2_scale [E, H, F/32] u8;
 *                  low nibble of a code byte = even index along the row.
 *   Shared expert: same layouts with leading dimension 1.
 *   R = T*k + S*T rows after permutation:
 *   offsets [E+S+1] int32, sorted_flat [R] int32, inv_pos [R] int32
 *   (flat id of the shared pair of token t is T*k + t),
 *   x_sorted [R, H] bf16, o_sorted [R, H] bf16, y [T, H] bf16.
 */
#ifndef FTMOE_H
#define FTMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FT_OK = 0,
    FT_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned buffer          */
    FT_ERR_UNSUPPORTED = 2,   /* shape outside the supported set                   */
    FT_ERR_CUDA = 3,          /* a CUDA runtime call failed (incl. earlier async)  */
    FT_ERR_WORKSPACE = 4,     /* ws too small for this call                        */
    FT_ERR_NOT_PINNED = 5,    /* host memory that must be pinned is not            */
    FT_ERR_TIMEOUT = 6,       /* a bounded host wait ran out                       */
    FT_ERR_DEVICE_CHECK = 7   /* a kernel reported an internal check failure       */
} ft_status;

typedef enum { FT_W_BF16 = 0, FT_W_MXFP4 = 1 } ft_wdtype;

typedef struct {
    int32_t hidden;       /* H */
    int32_t ffn;          /* F (per-expert SwiGLU width) */
    int32_t num_experts;  /* E routed experts */
    int32_t top_k;        /* k */
    int32_t num_shared;   /* S: 0 or 1 always-on shared expert */
    int32_t wdtype;       /* ft_wdtype of the expert weights */
} ft_moe_shape;

/* One layer's expert weights; device pointers, caller-owned.
 * expert_ptrs: optional device table of E entries x 4 pointers
 * {w13, w13_scale, w2, w2_scale} for one expert each (scales NULL for BF16),
 * used by the expert-slot cache; when non-NULL, w13/w2 are ignored for routed
 * experts.  Only the decode path (T <= ft_get_decode_max_tokens()) accepts a
 * table; the prefill grouped GEMM needs contiguous w13/w2. */
typedef struct {
    const void* w13;
    const uint8_t* w13_scale;
    const void* w2;
    const uint8_t* w2_scale;
    const void* const* expert_ptrs;
    const void* shared_w13;
    const uint8_t* shared_w13_scale;
    const void* shared_w2;
    const uint8_t* shared_w2_scale;
} ft_moe_weights;

/* Message for the last non-OK status returned on this thread ("" if none). */
const char* ft_last_error(void);

/* Library version string. */
const char* ft_version(void);

/* Token-count threshold of the decode path: T <= this uses the weight-streaming
 * decode kernels (the tcgen05 decode on BF16 or block-scaled MXFP4 weights for
 * batches that qualify, else the 128-bit GEMVs with the down projection and the
 * combine fused; ft_moe_decode_kernels tells which); larger T uses the tcgen05
 * grouped GEMM.  Default 32, or the environment variable FT_DECODE_MAX_TOKENS
 * read at load time.  Process-wide; returns the previous value.  Values < 0 are
 * rejected (returns -1). */
int32_t ft_set_decode_max_tokens(int32_t t);
int32_t ft_get_decode_max_tokens(void);

/* Block-scaled tensor-core decode for MXFP4 weights.  mode 0: never; 1: every
 * eligible decode batch; 2 (the default): eligible batches of 4 or more tokens
 * (on the DeepSeek-V4-Flash shape it is faster than the GEMVs from 4 tokens on,
 * slower for 1).  Process-wide; returns the previous mode, or -1 (and changes
 * nothing) for a mode outside 0..2.  Eligible: MXFP4 layers with contiguous
 * weights, no shared expert, H and F multiples of 512 and at most 4096.  The
 * experts then run as tcgen05.mma.kind::mxf8f6f4.block_scale MMAs: E2M1 weights
 * with their E8M0 scales straight from HBM (no dequantisation) times the
 * activations carried as two E4M3 planes (high plane and the plane of the
 * remainder, each with its own E8M0 scale per 32 elements; x before gate/up, h
 * before down).  Accuracy: under 1e-2 of max|y| against the exact layer (a third
 * of the 3e-2 MXFP4 tolerance); the GEMVs multiply the exactly decoded weights
 * in f16.  ft_moe_workspace_bytes reserves room for the planes on MXFP4 shapes. */
int32_t ft_set_block_scaled_decode(int32_t mode);

/* How many kernels one decode-sized ft_moe_layer_forward call (contiguous
 * weights) launches for this shape and T under the current settings
 * (ft_set_decode_max_tokens, ft_set_block_scaled_decode): the router (with the
 * fused top-k and counting sort), then the expert kernels of the path the call
 * takes -- BF16 tensor-core decode: 1 + the combine; block-scaled MXFP4: the x
 * planes, 1 (T <= 16, FFN <= 2048) or 3 (two projections and the h planes)
 * kernels, and the combine; the GEMVs: gate/up and down (combine fused).  The
 * debug-bounds build adds its permutation check.  Host-only, no CUDA call.
 * Returns 0 when T is 0 or above the decode threshold (the grouped-GEMM path),
 * -1 for an invalid shape or T < 0. */
int32_t ft_moe_decode_kernels(const ft_moe_shape* shape, int32_t T);

/* Bound on every pipeline wait of the grouped-GEMM kernels (steps 3 and 4 when
 * T > decode threshold): the time, in ns, a role waits for a stage without
 * progress before it gives up.  Default 4 s (4000000000); ns = 0 restores the
 * default.  Process-wide, applies to launches enqueued after the call; returns
 * the previous bound.  A wait that runs out makes the kernel give up cleanly:
 * it records a timeout in the workspace status word (ft_moe_check then
 * returns FT_ERR_DEVICE_CHECK), lets the copies and MMAs it issued finish,
 * frees its tensor memory and returns; that call's outputs are undefined and
 * the next call is unaffected.  Lets failure handling be tested without a
 * GPU fault (a bound too short for the pipeline makes the waits run out). */
uint64_t ft_set_pipeline_wait_limit_ns(uint64_t ns);

/* Bytes of scratch any call below needs for up to max_tokens tokens
 * (0 on invalid shape). */
size_t ft_moe_workspace_bytes(const ft_moe_shape* shape, int32_t max_tokens);

/* Clears the device status words at the start of a freshly allocated
 * workspace (ws: device, 256-byte aligned, >= 4096 bytes): the error flag and
 * the last-CTA tickets of the decode kernels, which every call leaves at zero
 * again.
 * Call once per workspace before its first use; enqueued on `stream`. */
ft_status ft_moe_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Synchronises `stream`, then reads and clears the device status word of ws.
 * FT_ERR_DEVICE_CHECK if a kernel since the last check saw a routed expert id
 * outside [0,E) or gave up a bounded wait (tcgen05 pipeline timeout);
 * FT_ERR_CUDA on an asynchronous CUDA error.  This is the only synchronising
 * call of the layer API. */
ft_status ft_moe_check(void* ws, void* stream);

/* Step 1 -- route.  x, w_router, bias (or NULL): device inputs.  topk_idx,
 * topk_w: device outputs.  logits: device output [T,E] fp32, or NULL.
 * ws: scratch (device) of ft_moe_workspace_bytes(shape, T) bytes or more. */
ft_status ft_moe_route(const ft_moe_shape* shape, int32_t T, const void* x, const float* w_router,
                       const float* bias, int32_t* topk_idx, float* topk_w, float* logits,
                       void* ws, size_t ws_bytes, void* stream);

/* Step 2 -- permute.  topk_idx: device input [T,k]; ids must lie in [0,E)
 * (an id outside is counted nowhere, its pair is dropped from the outputs
 * and ft_moe_check() then returns FT_ERR_DEVICE_CHECK).
 * offsets, sorted_flat, inv_pos: device outputs.  x_sorted: device output
 * [R,H] gather of x rows in sorted order, or NULL to skip the gather (the
 * decode path does not need it).  x may be NULL when x_sorted is NULL. */
ft_status ft_moe_permute(const ft_moe_shape* shape, int32_t T, const int32_t* topk_idx, const void* x,
                         int32_t* offsets, int32_t* sorted_flat, int32_t* inv_pos, void* x_sorted,
                         void* ws, size_t ws_bytes, void* stream);

/* Step 2 for callers that cannot allocate device memory (the source pages have
 * no counterpart to this entry point).  Same arithmetic, outputs and layouts
 * as ft_moe_permute, but no workspace argument: the scratch lives in one
 * static device array of the library (about 390 KB, held by every GPU that
 * loads the library until the process exits).  For callers that may not call
 * cudaMalloc: engines that reserve nearly all HBM for their own pools at
 * start-up, plugins handed only their input/output buffers by a framework
 * that owns the allocator, fixed-budget code that must not grow.
 * Limit: R = T*k + S*T <= 65536 rows, else FT_ERR_UNSUPPORTED before any
 * launch.  The first call on each device looks the array's device address up
 * (cudaGetSymbolAddress) and caches it; make that first call before any stream
 * capture.  The cached address lives as long as the device's context: do not
 * cudaDeviceReset that device after the first call.  `stream` must belong to
 * the current device (else FT_ERR_INVALID_ARG).  Every call shares the array
 * and it keeps the last call's contents: calls that overlap on the GPU race.
 * No allocation of any kind.  An id outside [0,E) drops its pair, and
 * offsets[E+S] < R is the only sign of it: the device status word that
 * ft_moe_check reads for a workspace (also the debug-bounds build's checks) is
 * not reported by this entry point.  The tile schedule that ft_moe_permute
 * leaves in its ws for ft_moe_experts is not produced for the caller here. */
ft_status ft_moe_permute_noalloc(const ft_moe_shape* shape, int32_t T, const int32_t* topk_idx, const void* x,
                                 int32_t* offsets, int32_t* sorted_flat, int32_t* inv_pos, void* x_sorted,
                                 void* stream);

/* Step 3 -- experts.  Computes o_sorted[r] = FFN_{group(r)}(x row of r) for
 * every permuted row r.  x: device [T,H]; x_sorted: device [R,H] as written
 * by ft_moe_permute (required when T > decode threshold, else may be NULL);
 * offsets, sorted_flat: as written by ft_moe_permute.  o_sorted: device
 * output [R,H] bf16.  The intermediate h = silu(a)*b is rounded to bf16. */
ft_status ft_moe_experts(const ft_moe_shape* shape, int32_t T, const ft_moe_weights* weights,
                         const void* x, const void* x_sorted, const int32_t* offsets,
                         const int32_t* sorted_flat, void* o_sorted, void* ws, size_t ws_bytes,
                         void* stream);

/* Step 3 split into its two grouped GEMMs (T > decode threshold only; they are
 * what ft_moe_experts runs there, one launch each):
 * gate/up: h[r,:] = bf16(silu(Wg x_r) * (Wu x_r)) for every permuted row r;
 *   x_sorted: device [R,H]; h: device output [R,F] bf16.
 * down:    o_sorted[r,:] = bf16(Wd h_r); h: device [R,F]; o_sorted: [R,H].
 * offsets and ws as for ft_moe_experts (ws carries the tile schedule written
 * by ft_moe_permute). */
ft_status ft_moe_experts_gateup(const ft_moe_shape* shape, int32_t T, const ft_moe_weights* weights,
                                const void* x_sorted, const int32_t* offsets, void* h, void* ws, size_t ws_bytes,
                                void* stream);
ft_status ft_moe_experts_down(const ft_moe_shape* shape, int32_t T, const ft_moe_weights* weights, const void* h,
                              const int32_t* offsets, void* o_sorted, void* ws, size_t ws_bytes, void* stream);

/* Step 4 -- combine.  y[t] = sum_j topk_w[t,j] * o_sorted[inv_pos[t*k+j]]
 * (+ o_sorted[inv_pos[T*k+t]] when S = 1); fp32 accumulation in j order,
 * shared term last, one RNE rounding to bf16.  All pointers device. */
ft_status ft_moe_combine(const ft_moe_shape* shape, int32_t T, const void* o_sorted, const int32_t* inv_pos,
                         const float* topk_w, void* y, void* stream);

/* Whole layer: steps 1-4 on one stream.  y: device output [T,H] bf16.
 * topk_idx_out: optional device output [T,k] (NULL: kept in ws only).
 * logits_out: optional device output [T,E] fp32. */
ft_status ft_moe_layer_forward(const ft_moe_shape* shape, int32_t T, const void* x, const float* w_router,
                               const float* bias, const ft_moe_weights* weights, void* y,
                               int32_t* topk_idx_out, float* logits_out, void* ws, size_t ws_bytes,
                               void* stream);

/* Chaining helper for stacked layers: out[t,:] = bf16(in[t,:] / sqrt(mean_h
 * in[t,h]^2 + eps)), computed in fp32.  in, out: device [T,H] bf16 (may alias). */
ft_status ft_moe_unit_rms(int32_t T, int32_t H, const void* in, void* out, float eps, void* stream);

/* ---------------------------------------------------------------------------
 * Host-resident experts: ft_expert_stream.
 * Every layer's routed experts live in pinned host memory (caller-owned).
 * prefill: streams whole layers host->HBM on `copy_stream` into two layer
 *   buffers (layer l+1 copies while layer l computes on `compute_stream`).
 * decode_step: per layer, routes on the GPU, reads the routed expert ids back
 *   (the only host synchronisation, a bounded wait), updates a per-layer LRU
 *   cache of `slots_per_layer` HBM expert slots on the host (hits first, then
 *   misses in ascending expert id, each into the lowest empty slot or the
 *   untouched slot with the oldest use), copies the missed experts host->HBM,
 *   and runs the experts through a device pointer table.  The cache starts
 *   cold.  Stacked layers are chained as x_{l+1} = ft_moe_unit_rms(y_l, 1e-6).
 *   cache_policy FT_CACHE_GLOBAL instead pools all num_layers * slots_per_layer
 *   slots into one LRU cache keyed by (layer, expert) -- the cross-layer cache of
 *   the FreeToken article (dothoosh.com, "Benchmarks and real performance":
 *   global LRU at equal capacity) -- with the same policy, one policy step per
 *   (decode step, layer) in execution order; a layer's misses may evict any
 *   layer's expert not touched in that policy step.
 * Shared experts and router weights are device-resident (caller-owned).
 * ------------------------------------------------------------------------- */
typedef struct ft_expert_stream ft_expert_stream;

typedef enum {
    FT_CACHE_PER_LAYER = 0,   /* slots_per_layer slots owned by each layer */
    FT_CACHE_GLOBAL = 1       /* num_layers * slots_per_layer slots shared by all layers */
} ft_cache_policy;

typedef struct {
    int32_t num_layers;
    int32_t slots_per_layer;            /* HBM expert slots per layer (>= k, <= E) */
    ft_moe_shape shape;
    const ft_moe_weights* host_layers;  /* host array [num_layers]; w13/w2(+scales) are
                                           pinned HOST pointers, contiguous per layer;
                                           shared_* are DEVICE pointers; expert_ptrs unused */
    void* hbm_arena;                    /* device, caller-owned, 256-byte aligned */
    size_t hbm_arena_bytes;             /* >= ft_expert_stream_arena_bytes(cfg) */
    int64_t host_wait_timeout_ms;       /* bound on every host wait (<= 0: 10000) */
    int32_t cache_policy;               /* ft_cache_policy; 0 (zero-initialised) = per layer */
} ft_stream_cfg;

/* Device bytes the stream needs in hbm_arena: two full-layer buffers plus
 * num_layers * slots_per_layer expert slots plus pointer tables. */
size_t ft_expert_stream_arena_bytes(const ft_stream_cfg* cfg);

/* Validates cfg (pinned-ness of every host pointer via cudaPointerGetAttributes:
 * FT_ERR_NOT_PINNED), creates events, returns an opaque handle. */
ft_status ft_expert_stream_create(const ft_stream_cfg* cfg, ft_expert_stream** out);

/* All layers over T tokens.  x: device [T,H] input of layer 0.
 * w_router / bias: HOST arrays of num_layers DEVICE pointers (bias entries may
 * be NULL; bias itself may be NULL).  y_layers: device [L,T,H] bf16 output of
 * every layer; x_layers: optional device [L,T,H] bf16, the input of every
 * layer.  ws: scratch of ft_moe_workspace_bytes(shape, T).  Returns after
 * enqueuing; the host waits (bounded) only for buffer reuse events. */
ft_status ft_expert_stream_prefill(ft_expert_stream* s, int32_t T, const void* x,
                                   const float* const* w_router, const float* const* bias,
                                   void* y_layers, void* x_layers, void* ws, size_t ws_bytes,
                                   void* compute_stream, void* copy_stream);

/* All layers over T tokens (T > decode threshold), streaming only the experts
 * each layer's router picks: per layer, route and permute on compute_stream,
 * read the group offsets back (one bounded host wait), copy the routed experts
 * host->HBM into their places in a layer buffer on copy_stream, then run the
 * experts and the combine.  Copies cannot overlap the layer's own compute (its
 * routing is needed first), so this pays off when a batch routes to a small
 * part of the expert set; the pages' prefill streams whole layers instead
 * ("full-layer double buffering": FreeToken article, dothoosh.com, "FreeToken
 * architecture", mechanism 2).  Same arguments and results as prefill (the
 * same kernels on the same data: bit-identical outputs). */
ft_status ft_expert_stream_prefill_routed(ft_expert_stream* s, int32_t T, const void* x,
                                          const float* const* w_router, const float* const* bias,
                                          void* y_layers, void* x_layers, void* ws, size_t ws_bytes,
                                          void* compute_stream, void* copy_stream);

/* One decode step over T tokens (T <= decode threshold), all layers, through
 * the LRU expert-slot cache.  Same arguments as prefill. */
ft_status ft_expert_stream_decode_step(ft_expert_stream* s, int32_t T, const void* x,
                                       const float* const* w_router, const float* const* bias,
                                       void* y_layers, void* x_layers, void* ws, size_t ws_bytes,
                                       void* compute_stream, void* copy_stream);

/* Counters of one layer (layer = -1: sum over layers):
 * out[0] hits, out[1] misses, out[2] host->device bytes, out[3] decode steps,
 * out[4] prefill layer copies, out[5] bounded-wait time in microseconds. */
ft_status ft_expert_stream_stats(const ft_expert_stream* s, int32_t layer, uint64_t out[6]);

/* Slot contents after the last step.  Per-layer cache: out[slots_per_layer]
 * expert ids of `layer` (-1 = empty).  Global cache: layer must be -1 and
 * out[num_layers * slots_per_layer] holds layer * E + expert (-1 = empty). */
ft_status ft_expert_stream_slots(const ft_expert_stream* s, int32_t layer, int32_t* out);

/* Empties every slot (next decode step starts cold) and zeroes the counters. */
ft_status ft_expert_stream_reset_cache(ft_expert_stream* s);

/* Elastic slot budget (FreeToken article, dothoosh.com, "FreeToken architecture",
 * mechanism 3: the GPU expert cache is rebuilt under a new VRAM budget at a safe point,
 * without restarting or reloading the host set).  Call between decode steps.  New
 * count in [k, cfg.slots_per_layer] (the arena was sized for cfg's count).  Growing adds
 * empty slots.  Shrinking keeps each cache's most recently used experts (per layer: the
 * slots_per_layer newest; global: num_layers * slots_per_layer newest), drops the rest,
 * and moves kept experts that sit above the new count into the lowest empty slots
 * (ascending old slot; ft_lru_resize).  The moves are device-to-device copies on
 * copy_stream, ordered after all work already enqueued on compute_stream and before
 * anything enqueued on it later.  Counters are kept. */
ft_status ft_expert_stream_set_slots(ft_expert_stream* s, int32_t slots_per_layer, void* compute_stream,
                                     void* copy_stream);

void ft_expert_stream_destroy(ft_expert_stream* s);

/* The host-side LRU policy of one layer's slot cache, one decode step (the
 * function ft_expert_stream_decode_step uses; host only, no CUDA call).
 * content[n_slots]: expert in each slot or -1; stamp[n_slots]: last use;
 * where[E]: slot of each expert or -1 -- all caller-owned host arrays, updated
 * in place (start: content = where = -1).  ids[n]: the step's routed experts,
 * sorted ascending, unique, n <= n_slots.  Every id already cached is a hit
 * and is touched first; then misses, in ascending id, each take the lowest
 * empty slot or else the slot not touched in this step with the smallest
 * stamp.  Stamp of ids[r] = step * E + r.  Outputs out_slot[n], out_hit[n].
 * The global cache calls it with E' = num_layers * E, ids layer * E + expert,
 * n_slots = num_layers * slots_per_layer and step = the policy-step count
 * (decode step * num_layers + layer). */
ft_status ft_lru_step(int32_t E, int32_t n_slots, int32_t* content, int64_t* stamp, int32_t* where,
                      int64_t step, const int32_t* ids, int32_t n, int32_t* out_slot, uint8_t* out_hit);

/* Resize of one LRU cache state from n_old to n_new slots (host only, no CUDA call; the
 * policy ft_expert_stream_set_slots applies).  content/stamp need room for
 * max(n_old, n_new) entries; where[E].  Growing: slots n_old..n_new-1 become empty.
 * Shrinking: the n_new occupied slots with the largest stamps are kept, the others
 * emptied (where = -1); then every kept expert in a slot >= n_new, in ascending slot
 * order, moves to the lowest empty slot < n_new; the moves are written to
 * move_from[i] -> move_to[i], i < *n_moves (capacity n_old). */
ft_status ft_lru_resize(int32_t E, int32_t n_old, int32_t n_new, int32_t* content, int64_t* stamp, int32_t* where,
                        int32_t* move_from, int32_t* move_to, int32_t* n_moves);

/* Diagnostic: a plain streaming read of `bytes` (a multiple of 16) of device
 * memory at `buf` (16-byte aligned) with 16-byte loads that bypass L1, four in
 * flight per thread, ctas_per_sm (1..8) CTAs of 256 threads per SM; `sink` is
 * one device word the kernel may write.  Enqueued on `stream`.  Time it with
 * events to see the bandwidth a kernel that only reads reaches for a transfer
 * of this size (decode layer calls move 50-650 MB, well below the sizes at
 * which HBM reaches its copy peak). */
ft_status ft_hbm_read_probe(const void* buf, size_t bytes, uint32_t* sink, int32_t ctas_per_sm, void* stream);

/* Diagnostic: TMA loads of 128-byte rows of `buf` into a 6-stage shared-memory ring, one CTA
 * per SM, nothing computed: mode 0 loads 128-row tiles; mode 1 the same rows as tile::gather4
 * loads (four rows per load); mode 2 gather4 loads of hashed rows inside the first
 * region_bytes (how a grouped GEMM would read permuted token rows in place).  Each CTA
 * streams bytes / (128 x 128 x SMs) tiles.  buf: device, 16-byte aligned, bytes >= 128 x 128
 * x SMs.  *status (device word, set to zero by the caller): 2 or 3 if a bounded wait ran out
 * (no fault is raised).  Time it with events on `stream`; returns after the launch. */
ft_status ft_tma_read_probe(int32_t mode, const void* buf, size_t bytes, size_t region_bytes, uint32_t* status,
                            void* stream);

/* Test hook for failure handling: make the n-th host->device expert copy
 * enqueue (counting from 1 after this call) report failure (n = 0 disables).
 * The failing decode step returns FT_ERR_CUDA and rolls the cache state of
 * that layer back to before the step. */
ft_status ft_expert_stream_inject_copy_failure(ft_expert_stream* s, int64_t n);

#ifdef __cplusplus
}
#endif

#endif /* FTMOE_H */

// ft_expert_stream: host-resident experts served from pinned memory.
//
// Prefill ("full-layer double buffering", FreeToken article, dothoosh.com, "FreeToken
// architecture", mechanism 2): two full-layer HBM buffers; the copy of layer l+1 runs on
// the copy stream while layer l computes on the compute stream.  Ordering is by CUDA
// events only (ready[b] after a layer's copies, free[b] after the layer's kernels); the
// host never waits.
//
// Decode (same passage: an LRU expert cache that follows the router; mechanism 3: the
// first request is served from a cold cache): per layer and step the router runs on the
// GPU, the routed ids come back through a pinned buffer (the one host wait, bounded), the
// host LRU policy (ft_lru_step) assigns slots, missed experts are copied host->HBM into
// their slots on the copy stream, a per-layer device pointer table is refreshed, and the
// decode kernels read the experts through the table.  The cache is either one LRU per
// layer or one LRU over all layers' slots keyed by (layer, expert) (global LRU at equal
// capacity: FreeToken article, dothoosh.com, "Benchmarks and real performance").  Any
// slot may be overwritten safely: the host has just waited for this layer's routed ids,
// which were produced after every earlier kernel on the compute stream finished reading.
#include <algorithm>
#include <chrono>
#include <cstring>
#include <new>
#include <thread>
#include <vector>

#include "kernels.h"


using namespace ftmoe;

extern "C" ft_status ft_lru_step(int32_t E, int32_t n_slots, int32_t* content, int64_t* stamp, int32_t* where,
                                 int64_t step, const int32_t* ids, int32_t n, int32_t* out_slot, uint8_t* out_hit) {
    if (E <= 0 || n_slots <= 0 || !content || !stamp || !where || (n > 0 && (!ids || !out_slot || !out_hit)))
        return fail(FT_ERR_INVALID_ARG, "ft_lru_step: bad arguments");
    if (n > n_slots) return fail(FT_ERR_INVALID_ARG, "ft_lru_step: %d ids > %d slots", n, n_slots);
    for (int r = 0; r < n; ++r)
        if (ids[r] < 0 || ids[r] >= E || (r > 0 && ids[r] <= ids[r - 1]))
            return fail(FT_ERR_INVALID_ARG, "ft_lru_step: ids must be sorted, unique, in [0, E)");
    std::vector<uint8_t> touched(size_t(n_slots), 0);
    // hits first: touch them with this step's stamps
    for (int r = 0; r < n; ++r) {
        int u = ids[r];
        int sl = where[u];
        if (sl >= 0) {
            touched[sl] = 1;
            stamp[sl] = step * E + r;
            out_slot[r] = sl;
            out_hit[r] = 1;
        }
    }
    // misses in ascending id: lowest empty slot, else the untouched slot used longest ago
    for (int r = 0; r < n; ++r) {
        int u = ids[r];
        if (where[u] >= 0 && touched[where[u]]) continue;
        int victim = -1;
        for (int i = 0; i < n_slots; ++i)
            if (content[i] < 0) { victim = i; break; }
        if (victim < 0)
            for (int i = 0; i < n_slots; ++i)
                if (!touched[i] && (victim < 0 || stamp[i] < stamp[victim])) victim = i;
        if (victim < 0) return fail(FT_ERR_INVALID_ARG, "ft_lru_step: no slot left");
        if (content[victim] >= 0) where[content[victim]] = -1;
        content[victim] = u;
        where[u] = victim;
        touched[victim] = 1;
        stamp[victim] = step * E + r;
        out_slot[r] = victim;
        out_hit[r] = 0;
    }
    return FT_OK;
}

extern "C" ft_status ft_lru_resize(int32_t E, int32_t n_old, int32_t n_new, int32_t* content, int64_t* stamp,
                                   int32_t* where, int32_t* move_from, int32_t* move_to, int32_t* n_moves) {
    if (E <= 0 || n_old <= 0 || n_new <= 0 || !content || !stamp || !where || !n_moves ||
        (n_new < n_old && (!move_from || !move_to)))
        return fail(FT_ERR_INVALID_ARG, "ft_lru_resize: bad arguments");
    *n_moves = 0;
    if (n_new >= n_old) {                          // grow: new slots start empty
        for (int i = n_old; i < n_new; ++i) { content[i] = -1; stamp[i] = -1; }
        return FT_OK;
    }
    // shrink: keep the n_new most recently used experts (stamps are unique)
    std::vector<int> occ;
    for (int i = 0; i < n_old; ++i)
        if (content[i] >= 0) occ.push_back(i);
    std::sort(occ.begin(), occ.end(), [&](int a, int b) { return stamp[a] > stamp[b]; });
    for (size_t r = size_t(n_new); r < occ.size(); ++r) {
        const int i = occ[r];
        where[content[i]] = -1;
        content[i] = -1;
        stamp[i] = -1;
    }
    // survivors above the new count move, in ascending old slot, to the lowest empty slot
    int free_slot = 0;
    for (int i = n_new; i < n_old; ++i) {
        if (content[i] < 0) continue;
        while (content[free_slot] >= 0) ++free_slot;   // exists: at most n_new survivors
        content[free_slot] = content[i];
        stamp[free_slot] = stamp[i];
        where[content[i]] = free_slot;
        move_from[*n_moves] = i;
        move_to[*n_moves] = free_slot;
        ++*n_moves;
        content[i] = -1;
        stamp[i] = -1;
    }
    return FT_OK;
}

struct LayerCache {
    std::vector<int32_t> content;   // [slots] expert id (global pool: layer * E + expert) or -1
    std::vector<int64_t> stamp;     // [slots]
    std::vector<int32_t> where;     // [E] (global pool: [L * E]) slot or -1
    uint64_t hits = 0, misses = 0, h2d = 0, steps = 0, prefill_copies = 0, wait_us = 0;
};

struct ft_expert_stream {
    ft_stream_cfg cfg;
    std::vector<ft_moe_weights> host;
    int L, S, E, k;
    int S_max;                      // slots per layer the arena holds (cfg.slots_per_layer)
    size_t b13, b13s, b2, b2s, expert_bytes, layer_bytes;
    uint8_t* buf[2];
    uint8_t* slots;                 // [L][S] expert slots, each [w13 | w13s | w2 | w2s]
    void** dtable;                  // device [L][E][4]
    void** htable;                  // pinned host mirror [L][E][4]
    int32_t* hids;                  // pinned [kSmallRoute * kMaxTopK]
    int32_t* hoff;                  // pinned [kMaxExperts + 2]: group offsets for routed-only prefill
    cudaEvent_t ready[2], freed[2], ids_ev, copy_ev;
    std::vector<LayerCache> cache;  // per-layer counters; per-layer policy: also the slot state
    bool global = false;            // FT_CACHE_GLOBAL: slot state lives in `pool`
    LayerCache pool;                // [L * S] slots shared by all layers
    int64_t policy_steps = 0;       // global policy steps taken (decode step * L + layer)
    int64_t timeout_ms;
    int64_t inject_at = 0;          // 0: off; else fail the n-th expert copy enqueue
    int64_t copy_count = 0;
};

static size_t a256(size_t v) { return (v + 255) & ~size_t(255); }

static void expert_sizes(const ft_moe_shape& s, size_t& b13, size_t& b13s, size_t& b2, size_t& b2s) {
    const size_t HF = size_t(s.hidden) * s.ffn;
    if (s.wdtype == FT_W_BF16) { b13 = 2 * HF * 2; b2 = HF * 2; b13s = b2s = 0; }
    else { b13 = 2 * HF / 2; b13s = 2 * HF / 32; b2 = HF / 2; b2s = HF / 32; }
}

static size_t arena_bytes(const ft_stream_cfg* c) {
    size_t b13, b13s, b2, b2s;
    expert_sizes(c->shape, b13, b13s, b2, b2s);
    const size_t E = size_t(c->shape.num_experts);
    const size_t layer = a256(E * b13) + a256(E * b13s) + a256(E * b2) + a256(E * b2s);
    const size_t expert = a256(b13) + a256(b13s) + a256(b2) + a256(b2s);
    return 2 * layer + size_t(c->num_layers) * c->slots_per_layer * expert +
           a256(size_t(c->num_layers) * E * 4 * sizeof(void*));
}

// empty every slot of the active policy's state (counters are left alone)
static void reset_slots(ft_expert_stream* st) {
    const size_t L = size_t(st->L), S = size_t(st->S), E = size_t(st->E);
    st->cache.resize(L);
    for (auto& c : st->cache) {
        c.content.assign(st->global ? 0 : S, -1);
        c.stamp.assign(st->global ? 0 : S, -1);
        c.where.assign(st->global ? 0 : E, -1);
    }
    st->pool.content.assign(st->global ? L * S : 0, -1);
    st->pool.stamp.assign(st->global ? L * S : 0, -1);
    st->pool.where.assign(st->global ? L * E : 0, -1);
    st->policy_steps = 0;
}

static bool is_pinned(const void* p) {
    if (!p) return false;
    cudaPointerAttributes at{};
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) { cudaGetLastError(); return false; }
    return at.type == cudaMemoryTypeHost;
}

extern "C" {

size_t ft_expert_stream_arena_bytes(const ft_stream_cfg* cfg) {
    if (!cfg || check_shape(&cfg->shape) != FT_OK || cfg->num_layers <= 0 || cfg->slots_per_layer <= 0) return 0;
    return arena_bytes(cfg);
}

ft_status ft_expert_stream_create(const ft_stream_cfg* cfg, ft_expert_stream** out) {
    if (!cfg || !out) return fail(FT_ERR_INVALID_ARG, "cfg/out is NULL");
    *out = nullptr;
    ft_status s = check_shape(&cfg->shape);
    if (s) return s;
    const int E = cfg->shape.num_experts, k = cfg->shape.top_k;
    if (cfg->num_layers <= 0) return fail(FT_ERR_INVALID_ARG, "num_layers must be > 0");
    if (cfg->slots_per_layer < k || cfg->slots_per_layer > E)
        return fail(FT_ERR_INVALID_ARG, "slots_per_layer %d must be in [k=%d, E=%d]", cfg->slots_per_layer, k, E);
    if (cfg->cache_policy != FT_CACHE_PER_LAYER && cfg->cache_policy != FT_CACHE_GLOBAL)
        return fail(FT_ERR_INVALID_ARG, "cache_policy %d is not a ft_cache_policy", cfg->cache_policy);
    if (!cfg->host_layers) return fail(FT_ERR_INVALID_ARG, "host_layers is NULL");
    if (!cfg->hbm_arena || (reinterpret_cast<uintptr_t>(cfg->hbm_arena) & 255))
        return fail(FT_ERR_INVALID_ARG, "hbm_arena NULL or not 256-byte aligned");
    if (cfg->hbm_arena_bytes < arena_bytes(cfg))
        return fail(FT_ERR_WORKSPACE, "hbm_arena %zu bytes < %zu needed", cfg->hbm_arena_bytes, arena_bytes(cfg));
    const bool mx = cfg->shape.wdtype == FT_W_MXFP4;
    for (int l = 0; l < cfg->num_layers; ++l) {
        const ft_moe_weights& w = cfg->host_layers[l];
        if (!w.w13 || !w.w2 || (mx && (!w.w13_scale || !w.w2_scale)))
            return fail(FT_ERR_INVALID_ARG, "layer %d: NULL host expert pointer", l);
        if (cfg->shape.num_shared && (!w.shared_w13 || !w.shared_w2))
            return fail(FT_ERR_INVALID_ARG, "layer %d: NULL shared expert pointer", l);
    }
    if ((s = cuda_state())) return s;
    for (int l = 0; l < cfg->num_layers; ++l) {
        const ft_moe_weights& w = cfg->host_layers[l];
        if (!is_pinned(w.w13) || !is_pinned(w.w2) || (mx && (!is_pinned(w.w13_scale) || !is_pinned(w.w2_scale))))
            return fail(FT_ERR_NOT_PINNED, "layer %d: host expert weights are not pinned (cudaHostAlloc/register them)", l);
    }
    ft_expert_stream* st = new (std::nothrow) ft_expert_stream();
    if (!st) return fail(FT_ERR_INVALID_ARG, "out of host memory");
    st->cfg = *cfg;
    st->host.assign(cfg->host_layers, cfg->host_layers + cfg->num_layers);
    st->cfg.host_layers = st->host.data();
    st->L = cfg->num_layers;
    st->S = cfg->slots_per_layer;
    st->S_max = cfg->slots_per_layer;
    st->E = E;
    st->k = k;
    expert_sizes(cfg->shape, st->b13, st->b13s, st->b2, st->b2s);
    st->expert_bytes = a256(st->b13) + a256(st->b13s) + a256(st->b2) + a256(st->b2s);
    st->layer_bytes = a256(E * st->b13) + a256(E * st->b13s) + a256(E * st->b2) + a256(E * st->b2s);
    uint8_t* base = static_cast<uint8_t*>(cfg->hbm_arena);
    st->buf[0] = base;
    st->buf[1] = base + st->layer_bytes;
    st->slots = base + 2 * st->layer_bytes;
    st->dtable = reinterpret_cast<void**>(st->slots + size_t(st->L) * st->S_max * st->expert_bytes);
    st->timeout_ms = cfg->host_wait_timeout_ms > 0 ? cfg->host_wait_timeout_ms : 10000;
    st->global = cfg->cache_policy == FT_CACHE_GLOBAL;
    reset_slots(st);
    cudaError_t e = cudaHostAlloc(reinterpret_cast<void**>(&st->htable), size_t(st->L) * E * 4 * sizeof(void*), cudaHostAllocDefault);
    if (e == cudaSuccess) e = cudaHostAlloc(reinterpret_cast<void**>(&st->hids), sizeof(int32_t) * kSmallRoute * kMaxTopK, cudaHostAllocDefault);
    if (e == cudaSuccess) e = cudaHostAlloc(reinterpret_cast<void**>(&st->hoff), sizeof(int32_t) * (kMaxExperts + 2), cudaHostAllocDefault);
    for (int i = 0; i < 2 && e == cudaSuccess; ++i) {
        e = cudaEventCreateWithFlags(&st->ready[i], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&st->freed[i], cudaEventDisableTiming);
    }
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&st->ids_ev, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&st->copy_ev, cudaEventDisableTiming);
    if (e != cudaSuccess) {
        ft_expert_stream_destroy(st);
        return cuda_ok(e, "expert stream setup");
    }
    std::memset(st->htable, 0, size_t(st->L) * E * 4 * sizeof(void*));
    *out = st;
    return FT_OK;
}

void ft_expert_stream_destroy(ft_expert_stream* s) {
    if (!s) return;
    for (int i = 0; i < 2; ++i) {
        if (s->ready[i]) cudaEventDestroy(s->ready[i]);
        if (s->freed[i]) cudaEventDestroy(s->freed[i]);
    }
    if (s->ids_ev) cudaEventDestroy(s->ids_ev);
    if (s->copy_ev) cudaEventDestroy(s->copy_ev);
    if (s->htable) cudaFreeHost(s->htable);
    if (s->hids) cudaFreeHost(s->hids);
    if (s->hoff) cudaFreeHost(s->hoff);
    delete s;
}

}  // extern "C"

// device layout of one full-layer buffer: [w13 all E | w13s all E | w2 all E | w2s all E]
static ft_moe_weights layer_view(const ft_expert_stream* s, int l, uint8_t* buf) {
    const size_t E = size_t(s->E);
    ft_moe_weights w = s->host[size_t(l)];   // shared_* (device) carried over
    w.w13 = buf;
    w.w13_scale = s->b13s ? buf + a256(E * s->b13) : nullptr;
    w.w2 = buf + a256(E * s->b13) + a256(E * s->b13s);
    w.w2_scale = s->b2s ? static_cast<const uint8_t*>(w.w2) + a256(E * s->b2) : nullptr;
    w.expert_ptrs = nullptr;
    return w;
}

static ft_status copy_layer(ft_expert_stream* s, int l, uint8_t* buf, cudaStream_t cs) {
    const ft_moe_weights& h = s->host[size_t(l)];
    const ft_moe_weights d = layer_view(s, l, buf);
    const size_t E = size_t(s->E);
    cudaError_t e = cudaMemcpyAsync(const_cast<void*>(d.w13), h.w13, E * s->b13, cudaMemcpyHostToDevice, cs);
    if (e == cudaSuccess && s->b13s)
        e = cudaMemcpyAsync(const_cast<uint8_t*>(d.w13_scale), h.w13_scale, E * s->b13s, cudaMemcpyHostToDevice, cs);
    if (e == cudaSuccess) e = cudaMemcpyAsync(const_cast<void*>(d.w2), h.w2, E * s->b2, cudaMemcpyHostToDevice, cs);
    if (e == cudaSuccess && s->b2s)
        e = cudaMemcpyAsync(const_cast<uint8_t*>(d.w2_scale), h.w2_scale, E * s->b2s, cudaMemcpyHostToDevice, cs);
    if (e != cudaSuccess) return cuda_ok(e, "layer host->device copy");
    s->cache[size_t(l)].prefill_copies += 1;
    s->cache[size_t(l)].h2d += E * (s->b13 + s->b13s + s->b2 + s->b2s);
    return FT_OK;
}

static ft_status check_common(ft_expert_stream* s, int T, const void* x, const float* const* w_router,
                              void* y_layers, void* x_layers, void* ws, size_t ws_bytes) {
    if (!s) return fail(FT_ERR_INVALID_ARG, "stream handle is NULL");
    if (T < 0) return fail(FT_ERR_INVALID_ARG, "T < 0");
    if (!x || !w_router || !y_layers || !x_layers) return fail(FT_ERR_INVALID_ARG, "NULL x, w_router, y_layers or x_layers");
    for (int l = 0; l < s->L; ++l)
        if (!w_router[l]) return fail(FT_ERR_INVALID_ARG, "w_router[%d] is NULL", l);
    if (!ws || ws_bytes < ft_moe_workspace_bytes(&s->cfg.shape, T))
        return fail(FT_ERR_WORKSPACE, "workspace too small for T=%d", T);
    return FT_OK;
}

extern "C" {

ft_status ft_expert_stream_prefill(ft_expert_stream* s, int32_t T, const void* x, const float* const* w_router,
                                   const float* const* bias, void* y_layers, void* x_layers, void* ws, size_t ws_bytes,
                                   void* compute_stream, void* copy_stream) {
    FT_TRACE("ft_expert_stream_prefill");
    ft_status st = check_common(s, T, x, w_router, y_layers, x_layers, ws, ws_bytes);
    if (st) return st;
    if (T == 0) return FT_OK;
    if (T <= ft_get_decode_max_tokens())
        return fail(FT_ERR_UNSUPPORTED, "prefill needs T > decode threshold (%d)", ft_get_decode_max_tokens());
    if ((st = cuda_state())) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(compute_stream), ps = static_cast<cudaStream_t>(copy_stream);
    const size_t TH = size_t(T) * s->cfg.shape.hidden;
    uint16_t* xl = static_cast<uint16_t*>(x_layers);
    uint16_t* yl = static_cast<uint16_t*>(y_layers);
    // layer 0 input
    if ((st = cuda_ok(cudaMemcpyAsync(xl, x, TH * 2, cudaMemcpyDeviceToDevice, cs), "copy x"))) return st;
    // buffers may still be read by an earlier call's kernels: copy stream waits for them
    for (int b = 0; b < 2; ++b)
        if ((st = cuda_ok(cudaStreamWaitEvent(ps, s->freed[b], 0), "wait freed"))) return st;
    if ((st = copy_layer(s, 0, s->buf[0], ps))) return st;
    if ((st = cuda_ok(cudaEventRecord(s->ready[0], ps), "record ready"))) return st;
    for (int l = 0; l < s->L; ++l) {
        const int b = l & 1;
        if (l + 1 < s->L) {
            const int nb = (l + 1) & 1;
            if (l >= 1 && (st = cuda_ok(cudaStreamWaitEvent(ps, s->freed[nb], 0), "wait freed"))) return st;
            if ((st = copy_layer(s, l + 1, s->buf[nb], ps))) return st;
            if ((st = cuda_ok(cudaEventRecord(s->ready[nb], ps), "record ready"))) return st;
        }
        if ((st = cuda_ok(cudaStreamWaitEvent(cs, s->ready[b], 0), "wait ready"))) return st;
        ft_moe_weights w = layer_view(s, l, s->buf[b]);
        st = ft_moe_layer_forward(&s->cfg.shape, T, xl + size_t(l) * TH, w_router[l], bias ? bias[l] : nullptr, &w,
                                  yl + size_t(l) * TH, nullptr, nullptr, ws, ws_bytes, cs);
        if (st) return st;
        if ((st = cuda_ok(cudaEventRecord(s->freed[b], cs), "record freed"))) return st;
        if (l + 1 < s->L) {
            st = ft_moe_unit_rms(T, s->cfg.shape.hidden, yl + size_t(l) * TH, xl + size_t(l + 1) * TH, 1e-6f, cs);
            if (st) return st;
        }
    }
    return FT_OK;
}

ft_status ft_expert_stream_prefill_routed(ft_expert_stream* s, int32_t T, const void* x, const float* const* w_router,
                                          const float* const* bias, void* y_layers, void* x_layers, void* ws,
                                          size_t ws_bytes, void* compute_stream, void* copy_stream) {
    FT_TRACE("ft_expert_stream_prefill_routed");
    ft_status st = check_common(s, T, x, w_router, y_layers, x_layers, ws, ws_bytes);
    if (st) return st;
    if (T == 0) return FT_OK;
    if (T <= ft_get_decode_max_tokens())
        return fail(FT_ERR_UNSUPPORTED, "prefill needs T > decode threshold (%d)", ft_get_decode_max_tokens());
    if ((st = cuda_state())) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(compute_stream), ps = static_cast<cudaStream_t>(copy_stream);
    const ft_moe_shape& sh = s->cfg.shape;
    const int E = s->E;
    const size_t TH = size_t(T) * sh.hidden;
    uint16_t* xl = static_cast<uint16_t*>(x_layers);
    uint16_t* yl = static_cast<uint16_t*>(y_layers);
    const WsLayout Lw = make_layout(sh, T);
    int32_t* idx = ws_at<int32_t>(ws, Lw.topk_idx);
    float* gw = ws_at<float>(ws, Lw.topk_w);
    int32_t* offsets = ws_at<int32_t>(ws, Lw.offsets);
    int32_t* sorted_flat = ws_at<int32_t>(ws, Lw.sorted_flat);
    int32_t* inv_pos = ws_at<int32_t>(ws, Lw.inv_pos);
    void* xs = ws_at<uint16_t>(ws, Lw.x_sorted);
    void* os = ws_at<uint16_t>(ws, Lw.o_sorted);
    if ((st = cuda_ok(cudaMemcpyAsync(xl, x, TH * 2, cudaMemcpyDeviceToDevice, cs), "copy x"))) return st;
    // buffer 0 may still be read by an earlier call's kernels
    if ((st = cuda_ok(cudaStreamWaitEvent(ps, s->freed[0], 0), "wait freed"))) return st;
    for (int l = 0; l < s->L; ++l) {
        LayerCache& c = s->cache[size_t(l)];
        const uint16_t* xcur = xl + size_t(l) * TH;
        // 1. route and permute on the GPU, read the group offsets back (the one host wait)
        if ((st = ft_moe_route(&sh, T, xcur, w_router[l], bias ? bias[l] : nullptr, idx, gw, nullptr, ws, ws_bytes, cs)))
            return st;
        if ((st = ft_moe_permute(&sh, T, idx, xcur, offsets, sorted_flat, inv_pos, xs, ws, ws_bytes, cs))) return st;
        if ((st = cuda_ok(cudaMemcpyAsync(s->hoff, offsets, sizeof(int32_t) * (E + 1), cudaMemcpyDeviceToHost, cs),
                          "offsets D2H")))
            return st;
        if ((st = cuda_ok(cudaEventRecord(s->ids_ev, cs), "record offsets"))) return st;
        const auto t0 = std::chrono::steady_clock::now();
        for (;;) {
            cudaError_t q = cudaEventQuery(s->ids_ev);
            if (q == cudaSuccess) break;
            if (q != cudaErrorNotReady) return cuda_ok(q, "wait for the group offsets");
            if (std::chrono::steady_clock::now() - t0 > std::chrono::milliseconds(s->timeout_ms))
                return fail(FT_ERR_TIMEOUT, "layer %d: group offsets not back within %lld ms", l, (long long)s->timeout_ms);
            std::this_thread::yield();
        }
        c.wait_us += uint64_t(std::chrono::duration_cast<std::chrono::microseconds>(std::chrono::steady_clock::now() - t0).count());
        // 2. copy only the routed experts into their places in the layer buffer.  Every kernel
        //    that read the buffer before (the previous layer) finished before this layer's
        //    routing ran, so the copies may start now.
        const ft_moe_weights& h = s->host[size_t(l)];
        const ft_moe_weights d = layer_view(s, l, s->buf[0]);
        uint64_t bytes = 0;
        for (int e = 0; e < E; ++e) {
            if (s->hoff[e + 1] == s->hoff[e]) continue;
            cudaError_t ce = cudaMemcpyAsync(static_cast<uint8_t*>(const_cast<void*>(d.w13)) + size_t(e) * s->b13,
                                             static_cast<const uint8_t*>(h.w13) + size_t(e) * s->b13, s->b13,
                                             cudaMemcpyHostToDevice, ps);
            if (ce == cudaSuccess && s->b13s)
                ce = cudaMemcpyAsync(const_cast<uint8_t*>(d.w13_scale) + size_t(e) * s->b13s, h.w13_scale + size_t(e) * s->b13s,
                                     s->b13s, cudaMemcpyHostToDevice, ps);
            if (ce == cudaSuccess)
                ce = cudaMemcpyAsync(static_cast<uint8_t*>(const_cast<void*>(d.w2)) + size_t(e) * s->b2,
                                     static_cast<const uint8_t*>(h.w2) + size_t(e) * s->b2, s->b2, cudaMemcpyHostToDevice, ps);
            if (ce == cudaSuccess && s->b2s)
                ce = cudaMemcpyAsync(const_cast<uint8_t*>(d.w2_scale) + size_t(e) * s->b2s, h.w2_scale + size_t(e) * s->b2s,
                                     s->b2s, cudaMemcpyHostToDevice, ps);
            if (ce != cudaSuccess) return cuda_ok(ce, "routed expert host->device copy");
            bytes += s->b13 + s->b13s + s->b2 + s->b2s;
        }
        c.h2d += bytes;
        c.prefill_copies += 1;
        if ((st = cuda_ok(cudaEventRecord(s->ready[0], ps), "record ready"))) return st;
        if ((st = cuda_ok(cudaStreamWaitEvent(cs, s->ready[0], 0), "wait ready"))) return st;
        // 3. experts and combine from the layer buffer
        if ((st = ft_moe_experts(&sh, T, &d, xcur, xs, offsets, sorted_flat, os, ws, ws_bytes, cs))) return st;
        if ((st = ft_moe_combine(&sh, T, os, inv_pos, gw, yl + size_t(l) * TH, cs))) return st;
        if (l + 1 < s->L) {
            st = ft_moe_unit_rms(T, sh.hidden, yl + size_t(l) * TH, xl + size_t(l + 1) * TH, 1e-6f, cs);
            if (st) return st;
        }
    }
    return cuda_ok(cudaEventRecord(s->freed[0], cs), "record freed");
}

ft_status ft_expert_stream_decode_step(ft_expert_stream* s, int32_t T, const void* x, const float* const* w_router,
                                       const float* const* bias, void* y_layers, void* x_layers, void* ws,
                                       size_t ws_bytes, void* compute_stream, void* copy_stream) {
    FT_TRACE("ft_expert_stream_decode_step");
    ft_status st = check_common(s, T, x, w_router, y_layers, x_layers, ws, ws_bytes);
    if (st) return st;
    if (T == 0) return FT_OK;
    if (T > ft_get_decode_max_tokens())
        return fail(FT_ERR_UNSUPPORTED, "decode step needs T <= decode threshold (%d)", ft_get_decode_max_tokens());
    if ((st = cuda_state())) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(compute_stream), ps = static_cast<cudaStream_t>(copy_stream);
    const ft_moe_shape& sh = s->cfg.shape;
    const int k = sh.top_k, E = s->E;
    const size_t TH = size_t(T) * sh.hidden;
    uint16_t* xl = static_cast<uint16_t*>(x_layers);
    uint16_t* yl = static_cast<uint16_t*>(y_layers);
    const WsLayout Lw = make_layout(sh, T);
    int32_t* d_idx = ws_at<int32_t>(ws, Lw.topk_idx);
    float* gw = ws_at<float>(ws, Lw.topk_w);
    float* lg = ws_at<float>(ws, Lw.logits);
    uint32_t* err = ws_at<uint32_t>(ws, Lw.err);
    PermOut po{ws_at<int32_t>(ws, Lw.offsets), ws_at<int32_t>(ws, Lw.sorted_flat), ws_at<int32_t>(ws, Lw.inv_pos),
               ws_at<int32_t>(ws, Lw.sched), err};
    if ((st = cuda_ok(cudaMemcpyAsync(xl, x, TH * 2, cudaMemcpyDeviceToDevice, cs), "copy x"))) return st;
    for (int l = 0; l < s->L; ++l) {
        LayerCache& c = s->cache[size_t(l)];
        // 1. route + top-k + permutation on the GPU (one launch), read the ids back: the one host wait
        const uint16_t* xcur = xl + size_t(l) * TH;
        if ((st = cuda_ok(launch_route(T, sh.hidden, E, k, sh.num_shared, xcur, w_router[l], bias ? bias[l] : nullptr,
                                       d_idx, gw, lg, err, ws_at<uint16_t>(ws, Lw.wr_planes), ws_at<float>(ws, Lw.route_part), &po, cs), "route launch")))
            return st;
        if ((st = cuda_ok(cudaMemcpyAsync(s->hids, d_idx, sizeof(int32_t) * T * k, cudaMemcpyDeviceToHost, cs), "ids D2H")))
            return st;
        if ((st = cuda_ok(cudaEventRecord(s->ids_ev, cs), "record ids"))) return st;
        const auto t0 = std::chrono::steady_clock::now();
        for (;;) {
            cudaError_t q = cudaEventQuery(s->ids_ev);
            if (q == cudaSuccess) break;
            if (q != cudaErrorNotReady) return cuda_ok(q, "wait for routed ids");
            if (std::chrono::steady_clock::now() - t0 > std::chrono::milliseconds(s->timeout_ms))
                return fail(FT_ERR_TIMEOUT, "layer %d: routed ids not back within %lld ms", l, (long long)s->timeout_ms);
            std::this_thread::yield();
        }
        c.wait_us += uint64_t(std::chrono::duration_cast<std::chrono::microseconds>(std::chrono::steady_clock::now() - t0).count());
        // 2. host LRU policy over the sorted unique routed ids
        std::vector<int32_t> ids(s->hids, s->hids + T * k);
        std::sort(ids.begin(), ids.end());
        ids.erase(std::unique(ids.begin(), ids.end()), ids.end());
        for (int32_t v : ids)
            if (v < 0 || v >= E) return fail(FT_ERR_DEVICE_CHECK, "layer %d: routed id %d outside [0, %d)", l, v, E);
        const int cap = s->global ? s->L * s->S : s->S;
        if (int(ids.size()) > cap)
            return fail(FT_ERR_UNSUPPORTED, "layer %d: %zu distinct experts in one step > %d slots", l, ids.size(), cap);
        // the policy's state: this layer's own slots, or the pool keyed by layer * E + expert
        LayerCache& pc = s->global ? s->pool : c;
        const int32_t key_base = s->global ? l * E : 0;
        const int32_t key_count = s->global ? s->L * E : E;
        const int32_t n_slots = s->global ? s->L * s->S : s->S;
        const int64_t pstep = s->global ? s->policy_steps : int64_t(c.steps);
        std::vector<int32_t> keys(ids);
        for (int32_t& v : keys) v += key_base;
        const std::vector<int32_t> bc = pc.content, bw = pc.where;
        const std::vector<int64_t> bs = pc.stamp;
        std::vector<int32_t> slot(ids.size());
        std::vector<uint8_t> hit(ids.size());
        if ((st = ft_lru_step(key_count, n_slots, pc.content.data(), pc.stamp.data(), pc.where.data(), pstep,
                              keys.data(), int32_t(ids.size()), slot.data(), hit.data())))
            return st;
        // 3. copy the misses into their slots (copy stream), refresh the pointer table
        void** ht = s->htable + size_t(l) * E * 4;
        std::vector<int> dirtied;
        uint64_t bytes = 0, nmiss = 0;
        for (size_t i = 0; i < ids.size(); ++i) {
            const int u = ids[i];
            uint8_t* sp = s->slots + ((s->global ? 0 : size_t(l) * s->S_max) + slot[i]) * s->expert_bytes;
            uint8_t* p13 = sp;
            uint8_t* p13s = sp + a256(s->b13);
            uint8_t* p2 = p13s + a256(s->b13s);
            uint8_t* p2s = p2 + a256(s->b2);
            if (!hit[i]) {
                ++s->copy_count;
                if (s->inject_at > 0 && s->copy_count == s->inject_at) {
                    // injected failure: undo this step's policy update; slots already being
                    // overwritten by enqueued copies no longer hold their old expert
                    pc.content = bc; pc.where = bw; pc.stamp = bs;
                    for (int d : dirtied) {
                        int old = pc.content[d];
                        if (old >= 0) pc.where[old] = -1;
                        pc.content[d] = -1;
                        pc.stamp[d] = -1;
                    }
                    return fail(FT_ERR_CUDA, "layer %d: injected host->device copy failure (copy %lld)", l,
                                (long long)s->copy_count);
                }
                const ft_moe_weights& h = s->host[size_t(l)];
                cudaError_t e = cudaMemcpyAsync(p13, static_cast<const uint8_t*>(h.w13) + size_t(u) * s->b13, s->b13,
                                                cudaMemcpyHostToDevice, ps);
                if (e == cudaSuccess && s->b13s)
                    e = cudaMemcpyAsync(p13s, h.w13_scale + size_t(u) * s->b13s, s->b13s, cudaMemcpyHostToDevice, ps);
                if (e == cudaSuccess)
                    e = cudaMemcpyAsync(p2, static_cast<const uint8_t*>(h.w2) + size_t(u) * s->b2, s->b2,
                                        cudaMemcpyHostToDevice, ps);
                if (e == cudaSuccess && s->b2s)
                    e = cudaMemcpyAsync(p2s, h.w2_scale + size_t(u) * s->b2s, s->b2s, cudaMemcpyHostToDevice, ps);
                if (e != cudaSuccess) return cuda_ok(e, "expert host->device copy");
                dirtied.push_back(slot[i]);
                bytes += s->b13 + s->b13s + s->b2 + s->b2s;
                ++nmiss;
            }
            ht[4 * u + 0] = p13;
            ht[4 * u + 1] = s->b13s ? p13s : nullptr;
            ht[4 * u + 2] = p2;
            ht[4 * u + 3] = s->b2s ? p2s : nullptr;
        }
        c.hits += ids.size() - nmiss;
        c.misses += nmiss;
        c.h2d += bytes;
        c.steps += 1;
        if (s->global) s->policy_steps += 1;
        if ((st = cuda_ok(cudaEventRecord(s->copy_ev, ps), "record copies"))) return st;
        if ((st = cuda_ok(cudaStreamWaitEvent(cs, s->copy_ev, 0), "wait copies"))) return st;
        void** dt = s->dtable + size_t(l) * E * 4;
        if ((st = cuda_ok(cudaMemcpyAsync(dt, ht, size_t(E) * 4 * sizeof(void*), cudaMemcpyHostToDevice, cs), "table H2D")))
            return st;
        // 4. experts through the slot table, down-projection fused with the combine
        ft_moe_weights w = s->host[size_t(l)];
        w.w13 = w.w2 = nullptr;
        w.w13_scale = w.w2_scale = nullptr;
        w.expert_ptrs = const_cast<const void* const*>(dt);
        DecodeArgs a = decode_args(&sh, T, &w, xcur, Lw, ws, po.offsets, po.sorted_flat, po.inv_pos, gw,
                                   yl + size_t(l) * TH, nullptr);
        if ((st = cuda_ok(launch_decode(a, cs), "decode experts launch"))) return st;
        if (l + 1 < s->L) {
            st = ft_moe_unit_rms(T, sh.hidden, yl + size_t(l) * TH, xl + size_t(l + 1) * TH, 1e-6f, cs);
            if (st) return st;
        }
    }
    return FT_OK;
}

ft_status ft_expert_stream_stats(const ft_expert_stream* s, int32_t layer, uint64_t out[6]) {
    if (!s || !out || layer < -1 || layer >= s->L) return fail(FT_ERR_INVALID_ARG, "bad stats arguments");
    for (int i = 0; i < 6; ++i) out[i] = 0;
    for (int l = 0; l < s->L; ++l) {
        if (layer >= 0 && l != layer) continue;
        const LayerCache& c = s->cache[size_t(l)];
        out[0] += c.hits; out[1] += c.misses; out[2] += c.h2d;
        out[3] += c.steps; out[4] += c.prefill_copies; out[5] += c.wait_us;
    }
    if (layer < 0) out[3] /= uint64_t(s->L);
    return FT_OK;
}

ft_status ft_expert_stream_slots(const ft_expert_stream* s, int32_t layer, int32_t* out) {
    if (!s || !out) return fail(FT_ERR_INVALID_ARG, "bad slots arguments");
    if (s->global) {
        if (layer != -1) return fail(FT_ERR_INVALID_ARG, "global cache: slots are read with layer = -1");
        std::copy(s->pool.content.begin(), s->pool.content.end(), out);
        return FT_OK;
    }
    if (layer < 0 || layer >= s->L) return fail(FT_ERR_INVALID_ARG, "bad slots arguments");
    const LayerCache& c = s->cache[size_t(layer)];
    for (int i = 0; i < s->S; ++i) out[i] = c.content[size_t(i)];
    return FT_OK;
}

ft_status ft_expert_stream_reset_cache(ft_expert_stream* s) {
    if (!s) return fail(FT_ERR_INVALID_ARG, "stream handle is NULL");
    for (auto& c : s->cache) c = LayerCache();
    reset_slots(s);
    s->copy_count = 0;
    return FT_OK;
}

ft_status ft_expert_stream_set_slots(ft_expert_stream* s, int32_t slots_per_layer, void* compute_stream,
                                     void* copy_stream) {
    FT_TRACE("ft_expert_stream_set_slots");
    if (!s) return fail(FT_ERR_INVALID_ARG, "stream handle is NULL");
    if (slots_per_layer < s->k || slots_per_layer > s->S_max)
        return fail(FT_ERR_INVALID_ARG, "slots_per_layer %d must be in [k=%d, %d (arena)]", slots_per_layer, s->k,
                    s->S_max);
    if (slots_per_layer == s->S) return FT_OK;
    ft_status st = cuda_state();
    if (st) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(compute_stream), ps = static_cast<cudaStream_t>(copy_stream);
    // the policy state: one per layer, or the pool (every layer's slots, layer-major)
    const int n_caches = s->global ? 1 : s->L;
    const int per = s->global ? s->L : 1;                     // slot counts scale by this
    std::vector<std::vector<int32_t>> from(static_cast<size_t>(n_caches)), to(static_cast<size_t>(n_caches));
    std::vector<int32_t> nmov(size_t(n_caches), 0);
    for (int q = 0; q < n_caches; ++q) {
        LayerCache& c = s->global ? s->pool : s->cache[size_t(q)];
        const int n_old = per * s->S, n_new = per * slots_per_layer;
        const int32_t keys = s->global ? s->L * s->E : s->E;
        c.content.resize(size_t(std::max(n_old, n_new)), -1);
        c.stamp.resize(size_t(std::max(n_old, n_new)), -1);
        from[size_t(q)].resize(size_t(n_old));
        to[size_t(q)].resize(size_t(n_old));
        if ((st = ft_lru_resize(keys, n_old, n_new, c.content.data(), c.stamp.data(), c.where.data(),
                                from[size_t(q)].data(), to[size_t(q)].data(), &nmov[size_t(q)])))
            return st;
        c.content.resize(size_t(n_new));
        c.stamp.resize(size_t(n_new));
    }
    s->S = slots_per_layer;
    // relocate the kept experts once every kernel already enqueued on the compute stream (which
    // may still read the old slots) is done; the next step's kernels wait for the copies
    bool any = false;
    for (int32_t n : nmov) any = any || n > 0;
    if (!any) return FT_OK;
    if ((st = cuda_ok(cudaEventRecord(s->ids_ev, cs), "record compute"))) return st;
    if ((st = cuda_ok(cudaStreamWaitEvent(ps, s->ids_ev, 0), "wait compute"))) return st;
    for (int q = 0; q < n_caches; ++q) {
        uint8_t* base = s->slots + (s->global ? 0 : size_t(q) * s->S_max) * s->expert_bytes;
        for (int m = 0; m < nmov[size_t(q)]; ++m) {
            cudaError_t e = cudaMemcpyAsync(base + size_t(to[size_t(q)][size_t(m)]) * s->expert_bytes,
                                            base + size_t(from[size_t(q)][size_t(m)]) * s->expert_bytes,
                                            s->expert_bytes, cudaMemcpyDeviceToDevice, ps);
            if (e != cudaSuccess) return cuda_ok(e, "slot relocation copy");
        }
    }
    if ((st = cuda_ok(cudaEventRecord(s->copy_ev, ps), "record relocation"))) return st;
    return cuda_ok(cudaStreamWaitEvent(cs, s->copy_ev, 0), "wait relocation");
}

ft_status ft_expert_stream_inject_copy_failure(ft_expert_stream* s, int64_t n) {
    if (!s || n < 0) return fail(FT_ERR_INVALID_ARG, "bad inject arguments");
    s->inject_at = n > 0 ? s->copy_count + n : 0;
    return FT_OK;
}

}  // extern "C"

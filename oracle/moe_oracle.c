/*
 * moe_oracle.c -- plain, slow, fp64 CPU restatement of the sparse-MoE FFN
 * forward pass and of the decode-time LRU expert cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark do.  It shares no code, header, table or constant with the
 * CUDA path.
 *
 * What the source pages fix, and what they leave open:
 *  - k-of-E expert routing per token: "6 of 256 routed experts in each of 43
 *    layers" (FreeToken write-up, aihot.vn, "The gap it targets"; also
 *    dothoosh.com FreeToken article, "FreeToken architecture").
 *  - one always-on shared expert next to 8 routed ones (TurboFieldfare
 *    article, dothoosh.com, "Background: Gemma 4 26B A4B").
 *  - BF16 and MXFP4 expert weights (dothoosh.com FreeToken article,
 *    "Benchmarks").  The E2M1 / E8M0 encodings follow the OCP Microscaling
 *    Formats (MX) v1.0 specification, section 5 (element and scale formats):
 *    E2M1 = 1 sign, 2 exponent (bias 1), 1 mantissa bit, no inf/NaN;
 *    E8M0 = 2^(b-127), 0xFF = NaN; one scale per 32 consecutive elements.
 *  - the offloaded computation is exact: CPU and GPU partial sums are merged
 *    without approximation and without changing the router (dothoosh.com
 *    FreeToken article, "FreeToken architecture", mechanism 1; ai4bro.com
 *    write-up, "Key points").  Hence the oracle is the plain definition.
 *  - decode uses an LRU expert cache that follows the router, starting cold
 *    (dothoosh.com FreeToken article, "FreeToken architecture", mechanisms 2
 *    and 3).
 * The pages print no formula for the layer itself.  The readings taken here:
 *  - logits l[t,e] = sum_h x[t,h] * Wr[e,h] + b[e];
 *  - top-k by (logit descending, expert index ascending), computed from the
 *    fp32 logits the caller passes in;
 *  - gate g = softmax over all E logits, restricted to the k selected and
 *    renormalised; identical to a softmax over the k selected logits;
 *  - expert FFN = SwiGLU: h = silu(Wg x) * (Wu x), o = Wd h, no biases,
 *    gate rows 0..F-1 of w13, up rows F..2F-1;
 *  - y[t] = sum_j g[t,j] * o_{t,j} + o_shared[t] (shared weight 1);
 *  - permutation = stable counting sort of flat pair p = t*k + j by expert,
 *    the shared group (if any) appended as group E in token order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------- exact decodes ---------------------------------------------- */

double oracle_bf16_to_f64(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP MX v1.0, E2M1: bits (s, e1, e0, m).  Normal (e != 0):
 * (-1)^s * 2^(e-1) * (1 + m/2).  Subnormal (e == 0): (-1)^s * 2^0 * (m/2). */
double oracle_e2m1_to_f64(uint8_t code)
{
    int s = (code >> 3) & 1;
    int e = (code >> 1) & 3;
    int m = code & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* OCP MX v1.0, E8M0: 2^(b - 127); 0xFF encodes NaN. */
double oracle_e8m0_to_f64(uint8_t b)
{
    if (b == 0xFF) return NAN;
    return ldexp(1.0, (int)b - 127);
}

/* OCP 8-bit float E4M3 (the MXFP8 element format, and NVFP4's block-scale format): bits
 * (s, e3 e2 e1 e0, m2 m1 m0), exponent bias 7, no infinities.  Normal (e != 0):
 * (-1)^s * 2^(e-7) * (1 + m/8); subnormal (e == 0): (-1)^s * 2^-6 * (m/8); S.1111.111 is NaN. */
double oracle_e4m3_to_f64(uint8_t b)
{
    int s = (b >> 7) & 1, e = (b >> 3) & 15, m = b & 7;
    if (e == 15 && m == 7) return NAN;
    double mag = e ? ldexp(1.0 + m / 8.0, e - 7) : ldexp(m / 8.0, -6);
    return s ? -mag : mag;
}

/* NVFP4 matrix [rows, cols] to fp64, exact (NVIDIA's 4-bit block format, named on the pages
 * only as the laptop build's: FreeToken article, dothoosh.com, editorial analysis; the layout
 * follows its public definition): E2M1 codes packed as for MXFP4 (codes[r][c/2], low nibble =
 * even c), one E4M3 scale per 16 consecutive elements of a row (scales[r][c/16]), one fp32
 * scale for the whole tensor; value = E2M1 * E4M3 * tensor_scale.  cols % 16 == 0. */
void oracle_decode_nvfp4(const uint8_t* codes, const uint8_t* scales, float tensor_scale, long rows, long cols,
                         double* out)
{
    for (long r = 0; r < rows; ++r)
        for (long c = 0; c < cols; ++c) {
            uint8_t byte = codes[r * (cols / 2) + c / 2];
            uint8_t code = (c & 1) ? (byte >> 4) : (byte & 15);
            out[r * cols + c] = oracle_e2m1_to_f64(code) * oracle_e4m3_to_f64(scales[r * (cols / 16) + c / 16]) *
                                (double)tensor_scale;
        }
}

/* element (r, c) of an MXFP4 matrix with `cols` columns:
 * codes[r][c/2] (low nibble = even c), scales[r][c/32]. */
static double mx_elem(const uint8_t* codes, const uint8_t* scales, long cols, long r, long c)
{
    uint8_t byte = codes[r * (cols / 2) + c / 2];
    uint8_t nib = (c & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);
    return oracle_e2m1_to_f64(nib) * oracle_e8m0_to_f64(scales[r * (cols / 32) + c / 32]);
}

/* decode a whole weight matrix [rows, cols] to fp64 (exact) */
void oracle_decode_matrix(int wdtype, const void* w, const uint8_t* scale, long rows, long cols, double* out)
{
    for (long r = 0; r < rows; ++r)
        for (long c = 0; c < cols; ++c)
            out[r * cols + c] = (wdtype == 0) ? oracle_bf16_to_f64(((const uint16_t*)w)[r * cols + c])
                                              : mx_elem((const uint8_t*)w, scale, cols, r, c);
}

/* ---------- step 1: router logits -------------------------------------- */

/* logits[t,e] = sum_h x[t,h]*Wr[e,h] + b[e] in fp64.  absdot[t,e] = sum_h |x*Wr|
 * (optional) feeds the fp32 dot-product error bound used by the tests. */
void oracle_router_logits(int T, int H, int E, const uint16_t* x, const float* w_router,
                          const float* bias, double* logits, double* absdot)
{
    for (int t = 0; t < T; ++t)
        for (int e = 0; e < E; ++e) {
            double s = 0.0, a = 0.0;
            for (int h = 0; h < H; ++h) {
                double p = oracle_bf16_to_f64(x[(long)t * H + h]) * (double)w_router[(long)e * H + h];
                s += p;
                a += fabs(p);
            }
            if (bias) s += (double)bias[e];
            logits[(long)t * E + e] = s;
            if (absdot) absdot[(long)t * E + e] = a;
        }
}

/* ---------- step 2: top-k + renormalised softmax ----------------------- */

typedef struct { float v; int i; } cand_t;

static int cand_cmp(const void* pa, const void* pb)
{
    const cand_t* a = (const cand_t*)pa;
    const cand_t* b = (const cand_t*)pb;
    if (a->v > b->v) return -1;          /* larger logit first            */
    if (a->v < b->v) return 1;
    return (a->i < b->i) ? -1 : (a->i > b->i); /* tie (incl. -0 == +0): lower index */
}

/* Full sort of all E candidates, first k kept (slot order = sort order).
 * g[t,j] = exp(l_j - l_0) / sum_i exp(l_i - l_0) over the k kept logits. */
void oracle_topk(int T, int E, int k, const float* logits32, int32_t* idx, double* g)
{
    cand_t* c = (cand_t*)malloc(sizeof(cand_t) * (size_t)E);
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) { c[e].v = logits32[(long)t * E + e]; c[e].i = e; }
        qsort(c, (size_t)E, sizeof(cand_t), cand_cmp);
        double l0 = (double)c[0].v, den = 0.0;
        for (int j = 0; j < k; ++j) den += exp((double)c[j].v - l0);
        for (int j = 0; j < k; ++j) {
            idx[(long)t * k + j] = c[j].i;
            g[(long)t * k + j] = exp((double)c[j].v - l0) / den;
        }
    }
    free(c);
}

/* ---------- step 3: permutation (textbook stable counting sort) -------- */

/* offsets[G+1] with G = E + S; sorted_flat / inv_pos have P + S*T entries
 * (P = T*k).  Flat id of the shared pair of token t is P + t. */
void oracle_permute(int T, int k, int E, int S, const int32_t* idx,
                    int32_t* offsets, int32_t* sorted_flat, int32_t* inv_pos)
{
    long P = (long)T * k;
    int G = E + (S ? 1 : 0);
    long* cursor = (long*)calloc((size_t)G + 1, sizeof(long));
    for (int gi = 0; gi <= G; ++gi) offsets[gi] = 0;
    for (long p = 0; p < P; ++p) offsets[idx[p] + 1] += 1;        /* histogram */
    if (S) offsets[E + 1] += T;
    for (int gi = 0; gi < G; ++gi) offsets[gi + 1] += offsets[gi]; /* prefix sum */
    for (int gi = 0; gi < G; ++gi) cursor[gi] = offsets[gi];
    for (long p = 0; p < P; ++p) {                                 /* stable scatter */
        long pos = cursor[idx[p]]++;
        sorted_flat[pos] = (int32_t)p;
        inv_pos[p] = (int32_t)pos;
    }
    if (S)
        for (int t = 0; t < T; ++t) {
            long pos = cursor[E]++;
            sorted_flat[pos] = (int32_t)(P + t);
            inv_pos[P + t] = (int32_t)pos;
        }
    free(cursor);
}

/* ---------- step 4: one token through one SwiGLU expert ---------------- */

static double w_elem(int wdtype, const void* w, const uint8_t* s, long cols, long r, long c)
{
    if (wdtype == 0) return oracle_bf16_to_f64(((const uint16_t*)w)[r * cols + c]);
    return mx_elem((const uint8_t*)w, s, cols, r, c);
}

/* x[H] -> o[H].  w13: [2F, H] (gate rows 0..F-1, up rows F..2F-1), w2: [H, F].
 * For MXFP4 the pointers are the packed codes and the E8M0 scale arrays. */
void oracle_expert_ffn(int H, int F, int wdtype, const void* w13, const uint8_t* w13_scale,
                       const void* w2, const uint8_t* w2_scale, const double* x, double* o)
{
    double* h = (double*)malloc(sizeof(double) * (size_t)F);
    for (int f = 0; f < F; ++f) {
        double a = 0.0, b = 0.0;
        for (int i = 0; i < H; ++i) {
            a += w_elem(wdtype, w13, w13_scale, H, f, i) * x[i];
            b += w_elem(wdtype, w13, w13_scale, H, F + f, i) * x[i];
        }
        h[f] = a / (1.0 + exp(-a)) * b;   /* silu(a) * b */
    }
    for (int i = 0; i < H; ++i) {
        double s = 0.0;
        for (int f = 0; f < F; ++f) s += w_elem(wdtype, w2, w2_scale, F, i, f) * h[f];
        o[i] = s;
    }
    free(h);
}

/* byte offset of expert e inside a stacked weight tensor */
static const void* expert_ptr(int wdtype, const void* base, long rows, long cols, int e, int is_scale)
{
    long per;
    if (is_scale) per = rows * (cols / 32);
    else per = (wdtype == 0) ? rows * cols * 2 : rows * (cols / 2);
    return (const void*)((const uint8_t*)base + (long)e * per);
}

/* ---------- step 5: the layer, for a list of tokens -------------------- */

/* y[n, H] (n = n_tokens, rows in list order) = sum_j g[t,j] * FFN_{idx[t,j]}(x_t)
 * + FFN_shared(x_t) when S = 1.  idx, g are the full [T, k] routing results.
 * tokens == NULL means all T tokens.  n_threads <= 0: library default. */
int oracle_moe_layer(int T, int H, int F, int E, int k, int S, int wdtype,
                     const int32_t* tokens, int n_tokens,
                     const uint16_t* x, const int32_t* idx, const double* g,
                     const void* w13, const uint8_t* w13_scale, const void* w2, const uint8_t* w2_scale,
                     const void* sw13, const uint8_t* sw13_scale, const void* sw2, const uint8_t* sw2_scale,
                     double* y, int n_threads)
{
    int n = tokens ? n_tokens : T;
    (void)E;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < n; ++r) {
        int t = tokens ? tokens[r] : r;
        if (t < 0 || t >= T) { bad = 1; continue; }
        double* xd = (double*)malloc(sizeof(double) * (size_t)H);
        double* o = (double*)malloc(sizeof(double) * (size_t)H);
        double* acc = y + (long)r * H;
        for (int i = 0; i < H; ++i) { xd[i] = oracle_bf16_to_f64(x[(long)t * H + i]); acc[i] = 0.0; }
        for (int j = 0; j < k; ++j) {
            int e = idx[(long)t * k + j];
            oracle_expert_ffn(H, F, wdtype,
                              expert_ptr(wdtype, w13, 2L * F, H, e, 0),
                              wdtype ? (const uint8_t*)expert_ptr(wdtype, w13_scale, 2L * F, H, e, 1) : NULL,
                              expert_ptr(wdtype, w2, H, F, e, 0),
                              wdtype ? (const uint8_t*)expert_ptr(wdtype, w2_scale, H, F, e, 1) : NULL,
                              xd, o);
            double gj = g[(long)t * k + j];
            for (int i = 0; i < H; ++i) acc[i] += gj * o[i];
        }
        if (S) {
            oracle_expert_ffn(H, F, wdtype, sw13, sw13_scale, sw2, sw2_scale, xd, o);
            for (int i = 0; i < H; ++i) acc[i] += o[i];
        }
        free(xd);
        free(o);
    }
    return bad ? -1 : 0;
}

/* ---------- error study: block-scaled (MXFP8) activations ------------- */

/* Nearest E4M3 value (OCP 8-bit float E4M3: 1 sign, 4 exponent bits with bias 7, 3 mantissa
 * bits, no infinities; largest normal 448 = 1.75 * 2^8, smallest normal 2^-6, subnormal step
 * 2^-9), ties to even, magnitudes above 448 saturated to 448 (the MX v1.0 spec leaves
 * overflow handling to the implementation; saturation is the conversion it recommends). */
double oracle_e4m3_round(double v)
{
    double a = fabs(v);
    if (a == 0.0) return 0.0 * v;
    int e = (int)floor(log2(a));
    if (e < -6) e = -6;                       /* subnormal range: fixed step 2^-9 */
    double step = ldexp(1.0, e - 3);
    double q = a / step;
    double r = floor(q);
    double d = q - r;
    if (d > 0.5 || (d == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
    double out = r * step;
    if (out > 448.0) out = 448.0;
    return v < 0 ? -out : out;
}

/* MXFP8 (E4M3) quantise-dequantise of n values in blocks of 32 (OCP Microscaling Formats
 * v1.0, conversion of a block of scalars to MX: shared scale X = 2^(floor(log2(max |v|)) -
 * emax_elem), emax_elem = 8 for E4M3; element P_i = round_E4M3(v_i / X); value = X * P_i).
 * A block of zeros keeps scale 1.  n % 32 == 0. */
void oracle_mxfp8_qdq(long n, const double* v, double* out)
{
    for (long b = 0; b < n; b += 32) {
        double amax = 0.0;
        for (int i = 0; i < 32; ++i) if (fabs(v[b + i]) > amax) amax = fabs(v[b + i]);
        double X = amax > 0.0 ? ldexp(1.0, (int)floor(log2(amax)) - 8) : 1.0;
        for (int i = 0; i < 32; ++i) out[b + i] = X * oracle_e4m3_round(v[b + i] / X);
    }
}

/* Two-plane MXFP8 split of n values: the high plane is the MXFP8 quantise-dequantise of v
 * (oracle_mxfp8_qdq), the low plane the same of the remainder v - high, each plane with its
 * own E8M0 block scales; the result is high + low, which is what a block-scaled MMA run once
 * per plane into one fp32 accumulator multiplies.  n % 32 == 0. */
void oracle_mxfp8x2_qdq(long n, const double* v, double* out)
{
    double* hi = (double*)malloc(sizeof(double) * (size_t)n);
    double* r = (double*)malloc(sizeof(double) * (size_t)n);
    oracle_mxfp8_qdq(n, v, hi);
    for (long i = 0; i < n; ++i) r[i] = v[i] - hi[i];
    oracle_mxfp8_qdq(n, r, out);
    for (long i = 0; i < n; ++i) out[i] += hi[i];
    free(hi);
    free(r);
}

/* The expert FFN of oracle_expert_ffn with both activation operands (x before gate/up, h
 * before down) passed through the MXFP8 quantiser of `planes` planes (1: oracle_mxfp8_qdq,
 * 2: oracle_mxfp8x2_qdq), as a block-scaled MMA with E4M3 activations would see them; products
 * and sums stay fp64.  H % 32 == 0, F % 32 == 0. */
void oracle_expert_ffn_mxfp8_planes(int planes, int H, int F, int wdtype, const void* w13, const uint8_t* w13_scale,
                                    const void* w2, const uint8_t* w2_scale, const double* x, double* o)
{
    double* xq = (double*)malloc(sizeof(double) * (size_t)H);
    double* h = (double*)malloc(sizeof(double) * (size_t)F);
    double* hq = (double*)malloc(sizeof(double) * (size_t)F);
    if (planes == 2) oracle_mxfp8x2_qdq(H, x, xq);
    else oracle_mxfp8_qdq(H, x, xq);
    for (int f = 0; f < F; ++f) {
        double a = 0.0, b = 0.0;
        for (int i = 0; i < H; ++i) {
            a += w_elem(wdtype, w13, w13_scale, H, f, i) * xq[i];
            b += w_elem(wdtype, w13, w13_scale, H, F + f, i) * xq[i];
        }
        h[f] = a / (1.0 + exp(-a)) * b;
    }
    if (planes == 2) oracle_mxfp8x2_qdq(F, h, hq);
    else oracle_mxfp8_qdq(F, h, hq);
    for (int i = 0; i < H; ++i) {
        double s = 0.0;
        for (int f = 0; f < F; ++f) s += w_elem(wdtype, w2, w2_scale, F, i, f) * hq[f];
        o[i] = s;
    }
    free(xq);
    free(h);
    free(hq);
}

/* One-plane form of oracle_expert_ffn_mxfp8_planes (E4M3 activations). */
void oracle_expert_ffn_mxfp8_act(int H, int F, int wdtype, const void* w13, const uint8_t* w13_scale,
                                 const void* w2, const uint8_t* w2_scale, const double* x, double* o)
{
    oracle_expert_ffn_mxfp8_planes(1, H, F, wdtype, w13, w13_scale, w2, w2_scale, x, o);
}

/* ---------- stacked-layer chaining ------------------------------------- */

/* x_next[t,:] = y[t,:] / sqrt(mean_h y[t,h]^2 + eps), fp64. */
void oracle_unit_rms(int T, int H, const double* y, double eps, double* out)
{
    for (int t = 0; t < T; ++t) {
        double ss = 0.0;
        for (int h = 0; h < H; ++h) ss += y[(long)t * H + h] * y[(long)t * H + h];
        double inv = 1.0 / sqrt(ss / H + eps);
        for (int h = 0; h < H; ++h) out[(long)t * H + h] = y[(long)t * H + h] * inv;
    }
}

/* ---------- decode-time LRU expert cache ------------------------------- */

/* One layer's cache of n_slots expert slots, cold at step 0.
 * ids: per step, the sorted unique experts the router picked (counts[s] of
 * them, concatenated).  Per step: every id already cached is a hit and is
 * touched; then misses are admitted in ascending id, each into an empty slot
 * (lowest index first) or else into the untouched slot with the oldest
 * last-use stamp.  Stamp of id u in step s = s*E + (rank of u in the step).
 * Outputs, aligned with ids: slot[] and hit[]; slot_expert[s][n_slots] is the
 * cache content after step s (-1 = empty).  Returns 0, or -1 if a step holds
 * more ids than slots or an id out of range. */
int oracle_lru_sim(int E, int n_slots, int n_steps, const int32_t* counts, const int32_t* ids,
                   int32_t* slot, uint8_t* hit, int32_t* slot_expert, int64_t* hits_out, int64_t* misses_out)
{
    int32_t* content = (int32_t*)malloc(sizeof(int32_t) * (size_t)n_slots);
    int64_t* stamp = (int64_t*)malloc(sizeof(int64_t) * (size_t)n_slots);
    int32_t* where = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
    uint8_t* touched = (uint8_t*)malloc((size_t)n_slots);
    int64_t hits = 0, misses = 0;
    int rc = 0;
    for (int i = 0; i < n_slots; ++i) { content[i] = -1; stamp[i] = -1; }
    for (int e = 0; e < E; ++e) where[e] = -1;
    long base = 0;
    for (int s = 0; s < n_steps && rc == 0; ++s) {
        int n = counts[s];
        if (n > n_slots) { rc = -1; break; }
        memset(touched, 0, (size_t)n_slots);
        for (int r = 0; r < n; ++r) {                      /* hits first */
            int u = ids[base + r];
            if (u < 0 || u >= E || (r > 0 && u <= ids[base + r - 1])) { rc = -1; break; }
            if (where[u] >= 0) {
                int sl = where[u];
                touched[sl] = 1;
                stamp[sl] = (int64_t)s * E + r;
                slot[base + r] = sl;
                hit[base + r] = 1;
                ++hits;
            }
        }
        for (int r = 0; r < n && rc == 0; ++r) {           /* then misses, ascending id */
            int u = ids[base + r];
            if (where[u] >= 0 && touched[where[u]]) continue;
            int victim = -1;
            for (int i = 0; i < n_slots; ++i)
                if (content[i] < 0) { victim = i; break; }
            if (victim < 0)
                for (int i = 0; i < n_slots; ++i)
                    if (!touched[i] && (victim < 0 || stamp[i] < stamp[victim])) victim = i;
            if (victim < 0) { rc = -1; break; }
            if (content[victim] >= 0) where[content[victim]] = -1;
            content[victim] = u;
            where[u] = victim;
            touched[victim] = 1;
            stamp[victim] = (int64_t)s * E + r;
            slot[base + r] = victim;
            hit[base + r] = 0;
            ++misses;
        }
        if (slot_expert)
            for (int i = 0; i < n_slots; ++i) slot_expert[(long)s * n_slots + i] = content[i];
        base += n;
    }
    if (hits_out) *hits_out = hits;
    if (misses_out) *misses_out = misses;
    free(content); free(stamp); free(where); free(touched);
    return rc;
}

/*
 * oracle.c -- plain, slow, obviously-correct CPU reference of one FreeToken-style
 * MoE layer (router, LRU expert-slot pool, FP4 SwiGLU expert FFN, weighted
 * combine) and of the q* bandwidth split.
 *
 * TEST INFRASTRUCTURE.  Only the test-suite, the smoke check and the benchmark's
 * CPU-baseline leg load this library.  It shares no code, header, table or
 * helper with the CUDA library; both sides only read the same input bytes made by
 * the seeded generator.  Compile with -O2 -ffp-contract=off (no fast-math), so
 * every float operation below is the single IEEE operation written.
 *
 * Sources (FreeToken write-ups, cited by page title or address and section):
 *  [q*]     post.smzdm.com/p/a825qpgl, section 二: misses split between PCIe
 *           transfer and CPU compute by q* = m * B_p / B_h; the four-machine table.
 *  [ratio]  "跑不快大模型，先别急着怪显卡", section 二 (q⋆): pull : compute =
 *           pcie_bw : (cpu_bw - pcie_bw).
 *  [split]  post.smzdm.com/p/a825qpgl, section 二: experts of a layer are cached
 *           hits, misses pulled to the GPU, or misses left to the CPU; results are
 *           merged by routing weight.
 *  [lru]    post.smzdm.com/p/aomxznrn, "FreeToken干的事": a global LRU expert-slot
 *           pool; recently used experts stay in VRAM, cold ones are evicted.
 *  [fmt]    post.smzdm.com/p/a825qpgl, section 一: MXFP4 expert weights
 *           (284B model) and an NVFP4 build of the 35B-A3B model.  The bit layouts
 *           are not on the pages; they follow the public OCP Microscaling v1.0
 *           spec (E2M1, E8M0) and NVIDIA's public NVFP4 description (E4M3 scale
 *           per 16 elements plus an FP32 tensor scale).
 *  [route]  "游戏电脑如何跑动2840亿参数大模型" (mubeitech): the router gate picks a
 *           few experts per token; post.smzdm.com/p/a825qpgl section 二: 256
 *           experts, 6 active.
 *
 * Readings where the pages are silent (each is a stated choice):
 *  - router logits: fp32, l[t,e] = tree(acc) + b[e], where lane j of 32 sums, with
 *    fmaf in ascending h, the 8-element chunks c = floor(h/8) with c mod 32 == j,
 *    and tree() adds lane j and lane j^off for off = 16, 8, 4, 2, 1;
 *  - top-k: descending logit, ties to the lower expert index;
 *  - weights: softmax over the k chosen logits (renormalize=1), or the full softmax
 *    over E read at the chosen experts (renormalize=0);
 *  - LRU: unique experts in ascending id; hits touched first, then each miss takes
 *    the lowest free slot, else the occupied unpinned slot with the oldest clock;
 *  - FFN: g = Wg x, u = Wu x, h = silu(g) * u, y_e = Wd h, accumulated in double;
 *  - prefill activations: x quantised to NVFP4 with a per-token FP32 scale
 *    amax(x_t)/(6*448); h quantised to NVFP4 with tensor scale 1.0;
 *  - q*: q_gpu = min(m, floor(m*B_p/B_h + 0.5)), q_cpu = m - q_gpu.
 *
 * Parity status: every function is pinned by tests against what the pages and the
 * mathematics fix: the codecs by the OCP tables and exhaustive byte sweeps, q* by
 * the pages' printed table, the router by an fp32 error bound around the exact dot
 * product and a full sort, the LRU by a textbook list LRU on random traces, the
 * expert FFN by closed forms on structured experts and by the sparse = dense
 * brute-force identity, the prefill path by closed forms on inputs NVFP4 holds
 * exactly.  The pages print no worked example of the FFN itself.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ codecs [fmt] */

/* E2M1 (OCP MX v1.0): sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0. */
double or_e2m1_value(int code)
{
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* E8M0: value 2^(b-127); 0xFF is NaN. */
double or_e8m0_value(int b)
{
    if ((b & 0xFF) == 0xFF) return NAN;
    return ldexp(1.0, (b & 0xFF) - 127);
}

/* E4M3 (FN variant, bias 7, no infinities, S.1111.111 is NaN, max 448). */
double or_e4m3_value(int b)
{
    int s = (b >> 7) & 1, e = (b >> 3) & 15, m = b & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) mag = ldexp(m / 8.0, -6);
    else mag = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* Nearest representable E2M1 to v, ties to the code with mantissa bit 0,
 * saturating at +-6; the sign of v (including -0) goes to bit 3. */
int or_e2m1_quantize(float v)
{
    double a = fabs((double)v), best_d = INFINITY;
    int best = 0;
    for (int c = 0; c < 8; c++) {
        double d = fabs(a - or_e2m1_value(c));
        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {
            best_d = d;
            best = c;
        }
    }
    if (a > 6.0) best = 7;
    return best | (signbit(v) ? 8 : 0);
}

/* Nearest finite non-negative E4M3 to v >= 0, ties to even mantissa, saturating at 448. */
int or_e4m3_quantize(float v)
{
    double a = (double)v, best_d = INFINITY;
    int best = 0;
    if (!(a > 0.0)) return 0;
    for (int c = 0; c < 127; c++) {
        double d = fabs(a - or_e4m3_value(c));
        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {
            best_d = d;
            best = c;
        }
    }
    if (a > 448.0) best = 126;
    return best;
}

static float bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* float -> bfloat16 bits, round to nearest even (inputs are finite). */
uint16_t or_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* fmt: 0 = MXFP4 (E8M0 per 32), 1 = NVFP4 (E4M3 per 16, times the tensor scale). */
static int block_of(int fmt) { return fmt == 0 ? 32 : 16; }

static float scale_value(int fmt, uint8_t s)
{
    return (float)(fmt == 0 ? or_e8m0_value(s) : or_e4m3_value(s));
}

/* One weight: (e2m1(c) * scale) * tensor_scale, two fp32 multiplies; for MXFP4 the
 * tensor scale is 1 and both products are exact. */
static float weight_value(int fmt, const uint8_t* codes, const uint8_t* scales, float ts,
                          int K, int r, int c)
{
    uint8_t byte = codes[(size_t)r * (K / 2) + c / 2];
    int code = (c & 1) ? (byte >> 4) : (byte & 15);
    float sv = scale_value(fmt, scales[(size_t)r * (K / block_of(fmt)) + c / block_of(fmt)]);
    float v = (float)or_e2m1_value(code) * sv;
    return fmt == 0 ? v : v * ts;
}

/* Dequantise a [rows, K] FP4 tensor in the canonical layout to fp32. */
void or_dequant(int fmt, const uint8_t* codes, const uint8_t* scales, float ts,
                int rows, int K, float* out)
{
    for (int r = 0; r < rows; r++)
        for (int c = 0; c < K; c++)
            out[(size_t)r * K + c] = weight_value(fmt, codes, scales, ts, K, r, c);
}

/* NVFP4 quantisation of one row of K values with tensor scale S (fp32 steps):
 * s_b = E4M3(amax_b / (6*S)); q = e4m3(s_b)*S; code = E2M1(v / q), 0 if q == 0. */
void or_nvfp4_quantize_row(const float* v, int K, float S, uint8_t* codes, uint8_t* scales)
{
    for (int b = 0; b < K / 16; b++) {
        float amax = 0.0f;
        for (int i = 0; i < 16; i++) {
            float a = fabsf(v[b * 16 + i]);
            if (a > amax) amax = a;
        }
        float denom = 6.0f * S;
        float ratio = amax / denom;
        int sc = or_e4m3_quantize(ratio);
        scales[b] = (uint8_t)sc;
        float q = (float)or_e4m3_value(sc) * S;
        for (int i = 0; i < 16; i += 2) {
            int c0 = 0, c1 = 0;
            if (q != 0.0f) {
                c0 = or_e2m1_quantize(v[b * 16 + i] / q);
                c1 = or_e2m1_quantize(v[b * 16 + i + 1] / q);
            }
            codes[(b * 16 + i) / 2] = (uint8_t)(c0 | (c1 << 4));
        }
    }
}

/* Per-token activation scale of the prefill path: amax(x_t) / (6*448), fp32. */
float or_token_scale(const float* v, int K)
{
    float amax = 0.0f;
    for (int i = 0; i < K; i++) {
        float a = fabsf(v[i]);
        if (a > amax) amax = a;
    }
    return amax / 2688.0f;
}

/* ------------------------------------------------------------------ router [route] */

/* Router logits in the fixed fp32 order stated in the header. */
void or_router_logits(const uint16_t* x, const uint16_t* wr, const float* bias, int T, int H,
                      int E, float* logits)
{
    for (int t = 0; t < T; t++)
        for (int e = 0; e < E; e++) {
            float acc[32], nxt[32];
            for (int j = 0; j < 32; j++) acc[j] = 0.0f;
            for (int h = 0; h < H; h++) {
                int lane = (h / 8) % 32;
                acc[lane] = fmaf(bf16_to_f32(x[(size_t)t * H + h]),
                                 bf16_to_f32(wr[(size_t)e * H + h]), acc[lane]);
            }
            for (int off = 16; off >= 1; off >>= 1) {
                for (int j = 0; j < 32; j++) nxt[j] = acc[j] + acc[j ^ off];
                for (int j = 0; j < 32; j++) acc[j] = nxt[j];
            }
            logits[(size_t)t * E + e] = acc[0] + (bias ? bias[e] : 0.0f);
        }
}

/* Top-k by descending logit, ties to the lower index (selection by repeated scan). */
void or_topk(const float* logits, int T, int E, int k, int32_t* idx)
{
    char* taken = (char*)malloc((size_t)E);
    for (int t = 0; t < T; t++) {
        const float* l = logits + (size_t)t * E;
        memset(taken, 0, (size_t)E);
        for (int j = 0; j < k; j++) {
            int best = -1;
            for (int e = 0; e < E; e++) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e;  /* strict: keeps lower index on ties */
            }
            taken[best] = 1;
            idx[(size_t)t * k + j] = best;
        }
    }
    free(taken);
}

/* Routing weights (double softmax). renormalize=1: softmax over the k chosen logits;
 * renormalize=0: the softmax over all E logits, read at the chosen experts. */
void or_route_weights(const float* logits, const int32_t* idx, int T, int E, int k,
                      int renormalize, float* w)
{
    for (int t = 0; t < T; t++) {
        const float* l = logits + (size_t)t * E;
        const int32_t* id = idx + (size_t)t * k;
        double mx = -INFINITY, den = 0.0;
        if (renormalize) {
            for (int j = 0; j < k; j++) mx = fmax(mx, (double)l[id[j]]);
            for (int j = 0; j < k; j++) den += exp((double)l[id[j]] - mx);
        } else {
            for (int e = 0; e < E; e++) mx = fmax(mx, (double)l[e]);
            for (int e = 0; e < E; e++) den += exp((double)l[e] - mx);
        }
        for (int j = 0; j < k; j++) w[(size_t)t * k + j] = (float)(exp((double)l[id[j]] - mx) / den);
    }
}

void or_route(const uint16_t* x, const uint16_t* wr, const float* bias, int T, int H, int E,
              int k, int renormalize, int32_t* idx, float* w, float* logits)
{
    or_router_logits(x, wr, bias, T, H, E, logits);
    or_topk(logits, T, E, k, idx);
    or_route_weights(logits, idx, T, E, k, renormalize, w);
}

/* --------------------------------------------------------------------- LRU [lru] */

typedef struct {
    int n_slots, n_keys;       /* n_keys = L * E */
    int32_t* slot_key;         /* slot -> layer*E + expert, -1 when empty */
    uint64_t* slot_clock;      /* last-touch clock per slot */
    int32_t* key_slot;         /* key -> slot, -1 when not resident */
    uint64_t clock;            /* global clock G */
} or_lru;

or_lru* or_lru_create(int n_slots, int n_keys)
{
    or_lru* p = (or_lru*)calloc(1, sizeof(or_lru));
    p->n_slots = n_slots;
    p->n_keys = n_keys;
    p->slot_key = (int32_t*)malloc(sizeof(int32_t) * (size_t)n_slots);
    p->slot_clock = (uint64_t*)calloc((size_t)n_slots, sizeof(uint64_t));
    p->key_slot = (int32_t*)malloc(sizeof(int32_t) * (size_t)n_keys);
    for (int s = 0; s < n_slots; s++) p->slot_key[s] = -1;
    for (int q = 0; q < n_keys; q++) p->key_slot[q] = -1;
    return p;
}

void or_lru_destroy(or_lru* p)
{
    if (!p) return;
    free(p->slot_key);
    free(p->slot_clock);
    free(p->key_slot);
    free(p);
}

void or_lru_state(const or_lru* p, int32_t* slot_key, uint64_t* slot_clock, int32_t* key_slot,
                  uint64_t* clock)
{
    memcpy(slot_key, p->slot_key, sizeof(int32_t) * (size_t)p->n_slots);
    memcpy(slot_clock, p->slot_clock, sizeof(uint64_t) * (size_t)p->n_slots);
    memcpy(key_slot, p->key_slot, sizeof(int32_t) * (size_t)p->n_keys);
    *clock = p->clock;
}

/* Resize the pool to n_new slots (post.smzdm.com/p/aomxznrn, "FreeToken干的事":
 * at run time the engine moves GPU memory between the expert cache and the KV
 * cache; read here as shrinking or growing the slot pool while keeping the LRU
 * order of what stays).  Shrinking evicts the residents with the oldest clocks until at
 * most n_new remain, then moves each survivor that sits in a slot >= n_new, in
 * ascending slot order, to the lowest free slot below n_new (its clock moves with
 * it).  Growing adds empty slots.  The global clock is unchanged.  Returns the
 * number of evictions, or -1 if n_new < 1. */
int or_lru_resize(or_lru* p, int n_new)
{
    if (n_new < 1) return -1;
    if (n_new > p->n_slots) {
        p->slot_key = (int32_t*)realloc(p->slot_key, sizeof(int32_t) * (size_t)n_new);
        p->slot_clock = (uint64_t*)realloc(p->slot_clock, sizeof(uint64_t) * (size_t)n_new);
        for (int s = p->n_slots; s < n_new; s++) {
            p->slot_key[s] = -1;
            p->slot_clock[s] = 0;
        }
        p->n_slots = n_new;
        return 0;
    }
    int resident = 0, evicted = 0;
    for (int s = 0; s < p->n_slots; s++) resident += p->slot_key[s] >= 0;
    while (resident > n_new) {          /* evict the least recently used */
        int v = -1;
        for (int s = 0; s < p->n_slots; s++)
            if (p->slot_key[s] >= 0 && (v < 0 || p->slot_clock[s] < p->slot_clock[v])) v = s;
        p->key_slot[p->slot_key[v]] = -1;
        p->slot_key[v] = -1;
        p->slot_clock[v] = 0;
        resident--;
        evicted++;
    }
    int free_slot = 0;
    for (int s = n_new; s < p->n_slots; s++) {
        if (p->slot_key[s] < 0) continue;
        while (p->slot_key[free_slot] >= 0) free_slot++;   /* exists: residents <= n_new */
        p->slot_key[free_slot] = p->slot_key[s];
        p->slot_clock[free_slot] = p->slot_clock[s];
        p->key_slot[p->slot_key[s]] = free_slot;
        p->slot_key[s] = -1;
        p->slot_clock[s] = 0;
    }
    p->n_slots = n_new;
    return evicted;
}

/* One (step, layer) lookup.  Outputs: slot_of[T*k]; uniq[] = sorted unique experts
 * with is_hit[] per entry (returns their count via *n_uniq); miss list
 * miss_expert[], miss_slot[], evicted_key[] (-1 when a free slot was used) in
 * ascending expert order (count via *n_miss).  Returns 0, or -1 if the pool is
 * smaller than the number of unique experts. */
int or_lru_step(or_lru* p, int layer, int E, const int32_t* idx, int T, int k, int32_t* slot_of,
                int32_t* uniq, int32_t* is_hit, int* n_uniq, int32_t* miss_expert,
                int32_t* miss_slot, int32_t* evicted_key, int* n_miss)
{
    char* used = (char*)calloc((size_t)E, 1);
    char* pinned = (char*)calloc((size_t)p->n_slots, 1);
    int nu = 0, nm = 0;
    for (int i = 0; i < T * k; i++) used[idx[i]] = 1;
    for (int e = 0; e < E; e++)
        if (used[e]) uniq[nu++] = e;
    if (nu > p->n_slots) {
        free(used);
        free(pinned);
        return -1;
    }
    /* hits first, ascending expert id */
    for (int u = 0; u < nu; u++) {
        int key = layer * E + uniq[u];
        int s = p->key_slot[key];
        is_hit[u] = s >= 0;
        if (s >= 0) {
            p->slot_clock[s] = ++p->clock;
            pinned[s] = 1;
        }
    }
    /* then misses, ascending expert id */
    for (int u = 0; u < nu; u++) {
        if (is_hit[u]) continue;
        int key = layer * E + uniq[u], s = -1;
        for (int q = 0; q < p->n_slots; q++)
            if (p->slot_key[q] < 0) { s = q; break; }
        int victim_key = -1;
        if (s < 0) {
            for (int q = 0; q < p->n_slots; q++) {
                if (pinned[q]) continue;
                if (s < 0 || p->slot_clock[q] < p->slot_clock[s]) s = q;
            }
            victim_key = p->slot_key[s];
            p->key_slot[victim_key] = -1;
        }
        p->slot_key[s] = key;
        p->key_slot[key] = s;
        p->slot_clock[s] = ++p->clock;
        pinned[s] = 1;
        miss_expert[nm] = uniq[u];
        miss_slot[nm] = s;
        evicted_key[nm] = victim_key;
        nm++;
    }
    for (int i = 0; i < T * k; i++) slot_of[i] = p->key_slot[layer * E + idx[i]];
    *n_uniq = nu;
    *n_miss = nm;
    free(used);
    free(pinned);
    return 0;
}

/* ------------------------------------------------------------------ FFN and combine */

/* One expert's FP4 tensors in the canonical layout. */
typedef struct {
    const uint8_t* codes[3];   /* gate [I,H/2], up [I,H/2], down [H,I/2] */
    const uint8_t* scales[3];  /* gate [I,H/bs], up [I,H/bs], down [H,I/bs] */
    float tscale[3];           /* FP32 tensor scales (NVFP4); 1 for MXFP4 */
} or_expert;

static double silu(double g) { return g / (1.0 + exp(-g)); }

/* y = Wd (silu(Wg x) * (Wu x)) for one token, x in fp32, accumulated in double. */
void or_expert_ffn(int fmt, int H, int I, const or_expert* ex, const float* x, double* y)
{
    double* h = (double*)malloc(sizeof(double) * (size_t)I);
    for (int i = 0; i < I; i++) {
        double g = 0.0, u = 0.0;
        for (int c = 0; c < H; c++) {
            g += (double)weight_value(fmt, ex->codes[0], ex->scales[0], ex->tscale[0], H, i, c) * x[c];
            u += (double)weight_value(fmt, ex->codes[1], ex->scales[1], ex->tscale[1], H, i, c) * x[c];
        }
        h[i] = silu(g) * u;
    }
    for (int r = 0; r < H; r++) {
        double acc = 0.0;
        for (int i = 0; i < I; i++)
            acc += (double)weight_value(fmt, ex->codes[2], ex->scales[2], ex->tscale[2], I, r, i) * h[i];
        y[r] = acc;
    }
    free(h);
}

/* Decode MoE layer for routed tokens: y[t] = sum_j w[t,j] * y_{idx[t,j]}(x_t) [split],
 * summed in double in rank order, then rounded to fp32 and to bf16.  experts[e] must
 * be valid for every chosen e. */
void or_moe_decode(int fmt, int H, int I, int T, int k, const uint16_t* x, const int32_t* idx,
                   const float* w, const or_expert* experts, float* y_f32, uint16_t* y_bf16)
{
    float* xf = (float*)malloc(sizeof(float) * (size_t)H);
    double* ye = (double*)malloc(sizeof(double) * (size_t)H);
    double* acc = (double*)malloc(sizeof(double) * (size_t)H);
    for (int t = 0; t < T; t++) {
        for (int c = 0; c < H; c++) xf[c] = bf16_to_f32(x[(size_t)t * H + c]);
        for (int c = 0; c < H; c++) acc[c] = 0.0;
        for (int j = 0; j < k; j++) {
            or_expert_ffn(fmt, H, I, &experts[idx[(size_t)t * k + j]], xf, ye);
            for (int c = 0; c < H; c++) acc[c] += (double)w[(size_t)t * k + j] * ye[c];
        }
        for (int c = 0; c < H; c++) {
            float f = (float)acc[c];
            y_f32[(size_t)t * H + c] = f;
            y_bf16[(size_t)t * H + c] = or_f32_to_bf16(f);
        }
    }
    free(xf);
    free(ye);
    free(acc);
}

/* Dense brute force for tiny shapes: every expert computed, y = sum_e m_e p_e y_e with
 * logits as plain double dot products, p the softmax, m the top-k mask and (when
 * renormalize) p renormalised over the mask. */
void or_moe_dense(int fmt, int H, int I, int E, int T, int k, int renormalize, const uint16_t* x,
                  const uint16_t* wr, const float* bias, const or_expert* experts, double* y,
                  int32_t* mask_out)
{
    float* xf = (float*)malloc(sizeof(float) * (size_t)H);
    double* l = (double*)malloc(sizeof(double) * (size_t)E);
    double* p = (double*)malloc(sizeof(double) * (size_t)E);
    double* ye = (double*)malloc(sizeof(double) * (size_t)H);
    int* m = (int*)malloc(sizeof(int) * (size_t)E);
    for (int t = 0; t < T; t++) {
        for (int c = 0; c < H; c++) xf[c] = bf16_to_f32(x[(size_t)t * H + c]);
        double mx = -INFINITY, den = 0.0;
        for (int e = 0; e < E; e++) {
            double s = 0.0;
            for (int c = 0; c < H; c++) s += (double)xf[c] * bf16_to_f32(wr[(size_t)e * H + c]);
            l[e] = s + (bias ? bias[e] : 0.0);
            mx = fmax(mx, l[e]);
        }
        for (int e = 0; e < E; e++) den += exp(l[e] - mx);
        for (int e = 0; e < E; e++) p[e] = exp(l[e] - mx) / den;
        /* mask: e is chosen iff fewer than k experts rank above it */
        double msum = 0.0;
        for (int e = 0; e < E; e++) {
            int above = 0;
            for (int f = 0; f < E; f++)
                if (l[f] > l[e] || (l[f] == l[e] && f < e)) above++;
            m[e] = above < k;
            if (m[e]) msum += p[e];
            mask_out[(size_t)t * E + e] = m[e];
        }
        for (int c = 0; c < H; c++) y[(size_t)t * H + c] = 0.0;
        for (int e = 0; e < E; e++) {
            or_expert_ffn(fmt, H, I, &experts[e], xf, ye);
            double coef = m[e] * (renormalize ? p[e] / msum : p[e]);
            for (int c = 0; c < H; c++) y[(size_t)t * H + c] += coef * ye[c];
        }
    }
    free(xf);
    free(l);
    free(p);
    free(ye);
    free(m);
}

/* Prefill activation quantisation of one token: S = amax(x_t)/(6*448), then NVFP4
 * with that tensor scale; returns S and writes codes [H/2], scales [H/16]. */
float or_prefill_quantize_x(const uint16_t* x_t, int H, uint8_t* codes, uint8_t* scales)
{
    float* xf = (float*)malloc(sizeof(float) * (size_t)H);
    for (int c = 0; c < H; c++) xf[c] = bf16_to_f32(x_t[c]);
    float S = or_token_scale(xf, H);
    or_nvfp4_quantize_row(xf, H, S, codes, scales);
    free(xf);
    return S;
}

/* Prefill token (activation-quantised path): x_t -> NVFP4 with the per-token scale,
 * g, u from the dequantised x; h = silu(g)*u rounded to fp32 and quantised to NVFP4
 * with tensor scale 1; y_e = Wd hq; y = sum_j w_j y_e (double) -> fp32 -> bf16. */
void or_moe_prefill_token(int H, int I, int k, const uint16_t* x_t, const int32_t* idx_t,
                          const float* w_t, const or_expert* experts, float* y_f32,
                          uint16_t* y_bf16)
{
    const int fmt = 1;
    float* xq = (float*)malloc(sizeof(float) * (size_t)H);
    uint8_t* xc = (uint8_t*)malloc((size_t)H / 2);
    uint8_t* xs = (uint8_t*)malloc((size_t)H / 16);
    float* hf = (float*)malloc(sizeof(float) * (size_t)I);
    float* hq = (float*)malloc(sizeof(float) * (size_t)I);
    uint8_t* hc = (uint8_t*)malloc((size_t)I / 2);
    uint8_t* hs = (uint8_t*)malloc((size_t)I / 16);
    double* acc = (double*)calloc((size_t)H, sizeof(double));
    float Sx = or_prefill_quantize_x(x_t, H, xc, xs);
    or_dequant(fmt, xc, xs, Sx, 1, H, xq);
    for (int j = 0; j < k; j++) {
        const or_expert* ex = &experts[idx_t[j]];
        for (int i = 0; i < I; i++) {
            double g = 0.0, u = 0.0;
            for (int c = 0; c < H; c++) {
                g += (double)weight_value(fmt, ex->codes[0], ex->scales[0], ex->tscale[0], H, i, c) * xq[c];
                u += (double)weight_value(fmt, ex->codes[1], ex->scales[1], ex->tscale[1], H, i, c) * xq[c];
            }
            hf[i] = (float)(silu(g) * u);
        }
        or_nvfp4_quantize_row(hf, I, 1.0f, hc, hs);
        or_dequant(fmt, hc, hs, 1.0f, 1, I, hq);
        for (int r = 0; r < H; r++) {
            double s = 0.0;
            for (int i = 0; i < I; i++)
                s += (double)weight_value(fmt, ex->codes[2], ex->scales[2], ex->tscale[2], I, r, i) * hq[i];
            acc[r] += (double)w_t[j] * s;
        }
    }
    for (int c = 0; c < H; c++) {
        float f = (float)acc[c];
        y_f32[c] = f;
        y_bf16[c] = or_f32_to_bf16(f);
    }
    free(xq); free(xc); free(xs);
    free(hf); free(hq); free(hc); free(hs);
    free(acc);
}

/* The h step of the prefill path for many rows at once: for every row r of the
 * [rows, I] double gate and up dot products, h = (float)(silu(g) * u), quantised
 * to NVFP4 with tensor scale 1 (the same steps as inside or_moe_prefill_token).
 * Writes codes [rows, I/2] and scales [rows, I/16]. */
void or_prefill_h_rows(const double* g, const double* u, int rows, int I, uint8_t* codes,
                       uint8_t* scales)
{
    float* hf = (float*)malloc(sizeof(float) * (size_t)I);
    for (int r = 0; r < rows; r++) {
        for (int i = 0; i < I; i++)
            hf[i] = (float)(silu(g[(size_t)r * I + i]) * u[(size_t)r * I + i]);
        or_nvfp4_quantize_row(hf, I, 1.0f, codes + (size_t)r * (I / 2), scales + (size_t)r * (I / 16));
    }
    free(hf);
}

/* ------------------------------------------------------------------------ q* [q*] */

/* q* = m * B_p / B_h misses go to the GPU; the rest would be computed by the CPU.
 * ratio = B_p / B_h (>= 1 means PCIe keeps up: every miss is pulled). */
int or_qstar_split(int m, double b_pcie, double b_host, int* q_gpu, int* q_cpu, double* ratio)
{
    if (m < 0 || !(b_pcie > 0.0) || !(b_host > 0.0)) return -1;
    double r = b_pcie / b_host;
    long long q = (long long)floor((double)m * r + 0.5);
    if (q > m) q = m;
    *q_gpu = (int)q;
    *q_cpu = m - (int)q;
    *ratio = r;
    return 0;
}

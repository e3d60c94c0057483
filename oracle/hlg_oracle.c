/*
 * hlg_oracle.c -- plain, slow fp64 CPU oracle for interleaved local/global
 * causal grouped-query attention with (proportional) RoPE, ring-buffer KV
 * slots and last-N-layer KV sharing.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the bench's
 * CPU-baseline leg load this library. The product path never links, imports
 * or calls it, and it shares no code, header or table with the CUDA library.
 *
 * Every function states the passage it follows. Page titles used below:
 *   [WALK]  "Gemma 4: End-to-End Architecture Walkthrough"
 *   [CORP]  "Gemma 4 Architecture Reference" (architecture fact sheet)
 *   [TALK]  "Gemma 4 Deep Dive -- Cassidy Hardin, Google DeepMind"
 *   [PLAY]  "Gemma 4: Architecture, Training and Local Deployment"
 *   [TECH]  "Gemma 4 Technical Report" (paper summary)
 *
 * Readings taken where the pages are silent (each is listed with its reason
 * in the design notes of the repository):
 *   - RoPE pairs are interleaved (2i, 2i+1); pair i turns by pos*theta^(-2i/D)
 *     using the full head dimension D; under p-RoPE only pairs
 *     i < floor(p*D/2) turn and the rest are the identity.
 *   - Rotation: y0 = x0 cos a - x1 sin a, y1 = x0 sin a + x1 cos a.
 *   - Positions are 0-based and absolute, on local layers too.
 *   - A window of W keys includes the query itself: key j is visible to the
 *     query at position p iff j <= p and (W == 0 or j > p - W).
 *   - The logit scale is passed in; there is no logit soft-capping.
 *   - Nothing is rounded: inputs are the bf16 values, all arithmetic fp64.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* bf16 bit pattern -> exact double (bf16 is the top half of an fp32). */
static double bf16_bits_to_double(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------ */
/* Layer schedule.                                                          */
/* [WALK] 3a "Interleaved Local/Global Attention": r local layers per global */
/* layer (4:1 small models, 5:1 larger ones) and the final layer is always  */
/* global. [CORP] "Attention Architecture" and [TALK] say the same; [PLAY]  */
/* 3.1 gives the 5:1 / 4:1 ratios.                                          */
/* Returns 1 for a global layer, 0 for a local one, -1 on a bad argument.   */
/* ------------------------------------------------------------------------ */
int hlg_layer_is_global(int n_layers, int ratio, int layer)
{
    if (n_layers <= 0 || ratio < 0 || layer < 0 || layer >= n_layers)
        return -1;
    if (layer == n_layers - 1)
        return 1;
    return ((layer + 1) % (ratio + 1)) == 0 ? 1 : 0;
}

/* ------------------------------------------------------------------------ */
/* KV sharing. [CORP] "Shared KV Cache": the last N layers reuse the K/V of */
/* earlier layers of the same attention type. The pages do not say which    */
/* earlier layer; the reading taken is the latest non-shared layer of the   */
/* same type. Returns the layer itself when it is not among the last N,     */
/* the source layer when one exists, -1 when a shared layer has no earlier  */
/* layer of its type (it then keeps its own cache), -2 on a bad argument.   */
/* ------------------------------------------------------------------------ */
int hlg_share_source(int n_layers, int ratio, int n_shared, int layer)
{
    if (n_shared < 0 || n_shared > n_layers)
        return -2;
    int type = hlg_layer_is_global(n_layers, ratio, layer);
    if (type < 0)
        return -2;
    int first_shared = n_layers - n_shared;
    if (layer < first_shared)
        return layer;
    for (int s = first_shared - 1; s >= 0; --s)
        if (hlg_layer_is_global(n_layers, ratio, s) == type)
            return s;
    return -1;
}

/* ------------------------------------------------------------------------ */
/* Cache slot of absolute position pos. [WALK] 3b: global layers cache K/V  */
/* for the whole context (slot = position); [TALK]: a local layer only      */
/* needs its window, kept as a ring of W slots (slot = pos mod W).          */
/* ------------------------------------------------------------------------ */
int64_t hlg_cache_slot(int64_t pos, int window)
{
    if (pos < 0)
        return -1;
    return window > 0 ? pos % window : pos;
}

/* ------------------------------------------------------------------------ */
/* Visible keys of the query at absolute position pos among keys            */
/* 0..n_keys-1. [WALK] 3a: a sliding-window token attends only to a fixed   */
/* recent window; a global token attends to the whole preceding context.    */
/* Writes the inclusive range [lo, hi] and returns the count (0 if empty).  */
/* ------------------------------------------------------------------------ */
int64_t hlg_visible_range(int64_t pos, int window, int64_t n_keys,
                          int64_t* lo, int64_t* hi)
{
    int64_t a = 0, b = pos;
    if (window > 0 && pos - window + 1 > 0)
        a = pos - window + 1;
    if (b > n_keys - 1)
        b = n_keys - 1;
    if (lo) *lo = a;
    if (hi) *hi = b;
    return b >= a ? b - a + 1 : 0;
}

/* ------------------------------------------------------------------------ */
/* (p-)RoPE of one D-vector at absolute position pos, in fp64.              */
/* [WALK] 3c "p-RoPE": standard RoPE turns every dimension pair by a        */
/* frequency that falls along the vector; p-RoPE (global layers) keeps the  */
/* rotation only on the first fraction p of the pairs (the high-frequency   */
/* ones) and leaves the rest unrotated. [CORP] "Positional Encoding: p-RoPE"*/
/* gives p = 0.25 and theta = 1e6 on global layers. Local layers use full   */
/* RoPE (rope_frac = 1).                                                    */
/* ------------------------------------------------------------------------ */
int hlg_rope_n_rotated_pairs(int head_dim, double rope_frac)
{
    return (int)floor(rope_frac * (double)(head_dim / 2));
}

void hlg_rope(const double* x, double* y, int head_dim, double rope_frac,
              double theta, int64_t pos)
{
    int n_rot = hlg_rope_n_rotated_pairs(head_dim, rope_frac);
    for (int i = 0; i < head_dim / 2; ++i) {
        double x0 = x[2 * i], x1 = x[2 * i + 1];
        if (i < n_rot) {
            double inv_freq = pow(theta, -2.0 * (double)i / (double)head_dim);
            double a = (double)pos * inv_freq;
            double c = cos(a), s = sin(a);
            y[2 * i] = x0 * c - x1 * s;
            y[2 * i + 1] = x0 * s + x1 * c;
        } else {
            y[2 * i] = x0;
            y[2 * i + 1] = x1;
        }
    }
}

/* Same, on bf16 input bits. */
void hlg_rope_bf16(const uint16_t* x_bits, double* y, int head_dim,
                   double rope_frac, double theta, int64_t pos)
{
    double* x = (double*)malloc(sizeof(double) * (size_t)head_dim);
    for (int d = 0; d < head_dim; ++d)
        x[d] = bf16_bits_to_double(x_bits[d]);
    hlg_rope(x, y, head_dim, rope_frac, theta, pos);
    free(x);
}

/* ------------------------------------------------------------------------ */
/* Attention rows.                                                          */
/*                                                                          */
/* For each requested row (b, h, i): the query sits at absolute position    */
/* p = q_pos0[b] + i, reads KV head g = h / (Hq / Hkv) ([WALK] 3b and       */
/* [CORP] "Attention Architecture": grouped-query attention, 2:1 on local   */
/* layers, 8:1 on global layers), and                                       */
/*     s_j = scale * <R_p(q), k~_j>       for every visible key j,          */
/*     o   = sum_j softmax(s)_j v_j,      lse = log sum_j exp(s_j)          */
/* where k~_j = R_j(k_j) for keys at positions >= rot_from[b] (keys given   */
/* pre-RoPE) and k~_j = k_j below it (keys that arrive already rotated, as  */
/* in a filled cache). V is never rotated.                                  */
/*                                                                          */
/* K = V ([WALK] 3b "K = V"; [TECH] "Core Model Architecture": global       */
/* layers cache only K and multiply the attention weights by K, which then  */
/* serves as V): pass v == NULL and v_j is the key as the cache holds it,   */
/* k~_j. Reading: the cache holds rotated keys, so the values are the       */
/* rotated keys.                                                            */
/*                                                                          */
/* Layouts: q [B][S][Hq][D], k and v [B][T][Hkv][D] in position order       */
/* (key j of batch b is row j), all bf16 bits. rows [n_rows][3] int32.      */
/* out [n_rows][D] fp64, lse [n_rows] fp64 (-inf when nothing is visible).  */
/* Returns 0, or -1 on a bad argument.                                      */
/* ------------------------------------------------------------------------ */
typedef struct {
    const uint16_t *q, *k, *v;
    const int64_t *q_pos0, *n_keys, *rot_from;
    int B, S, T, Hq, Hkv, D, window;
    double rope_frac, theta, scale;
    int64_t n_rows;
    const int32_t* rows;
    double *out, *lse;
} attn_args;

typedef struct {
    const attn_args* a;
    int b, g;
    double* krot;            /* [n_keys][D] rotated keys of (b, g) */
    const int64_t* row_ids;  /* rows of this (b, g) */
    int64_t n_ids;
    int64_t next;            /* work counter, atomically advanced */
    int64_t next_key;
    int phase;               /* 0 = rotate keys, 1 = rows */
} group_work;

static void rotate_keys_of_group(group_work* w, int64_t j)
{
    const attn_args* a = w->a;
    const uint16_t* src = a->k + (((size_t)w->b * a->T + (size_t)j) * a->Hkv + w->g) * a->D;
    double* dst = w->krot + (size_t)j * a->D;
    if (j >= a->rot_from[w->b]) {
        hlg_rope_bf16(src, dst, a->D, a->rope_frac, a->theta, j);
    } else {
        for (int d = 0; d < a->D; ++d)
            dst[d] = bf16_bits_to_double(src[d]);
    }
}

static void one_row(group_work* w, int64_t r, double* s, double* qrot)
{
    const attn_args* a = w->a;
    const int32_t* rw = a->rows + 3 * r;
    int b = rw[0], h = rw[1], i = rw[2];
    int64_t pos = a->q_pos0[b] + i;
    const uint16_t* qb = a->q + (((size_t)b * a->S + (size_t)i) * a->Hq + h) * a->D;
    hlg_rope_bf16(qb, qrot, a->D, a->rope_frac, a->theta, pos);

    int64_t lo, hi;
    int64_t cnt = hlg_visible_range(pos, a->window, a->n_keys[b], &lo, &hi);
    double* o = a->out + (size_t)r * a->D;
    for (int d = 0; d < a->D; ++d)
        o[d] = 0.0;
    if (cnt == 0) {
        a->lse[r] = -INFINITY;
        return;
    }
    double m = -INFINITY;
    for (int64_t j = lo; j <= hi; ++j) {
        const double* kj = w->krot + (size_t)j * a->D;
        double dot = 0.0;
        for (int d = 0; d < a->D; ++d)
            dot += qrot[d] * kj[d];
        s[j - lo] = a->scale * dot;
        if (s[j - lo] > m)
            m = s[j - lo];
    }
    double l = 0.0;
    for (int64_t j = lo; j <= hi; ++j) {
        double p = exp(s[j - lo] - m);
        s[j - lo] = p;
        l += p;
    }
    for (int64_t j = lo; j <= hi; ++j) {
        double p = s[j - lo] / l;
        if (a->v == NULL) {
            const double* kj = w->krot + (size_t)j * a->D;  /* K serves as V */
            for (int d = 0; d < a->D; ++d)
                o[d] += p * kj[d];
            continue;
        }
        const uint16_t* vj = a->v + (((size_t)b * a->T + (size_t)j) * a->Hkv + w->g) * a->D;
        for (int d = 0; d < a->D; ++d)
            o[d] += p * bf16_bits_to_double(vj[d]);
    }
    a->lse[r] = m + log(l);
}

static void* group_worker(void* arg)
{
    group_work* w = (group_work*)arg;
    const attn_args* a = w->a;
    if (w->phase == 0) {
        int64_t nk = a->n_keys[w->b];
        for (;;) {
            int64_t j = __atomic_fetch_add(&w->next_key, 1, __ATOMIC_RELAXED);
            if (j >= nk)
                break;
            rotate_keys_of_group(w, j);
        }
        return NULL;
    }
    double* s = (double*)malloc(sizeof(double) * (size_t)(a->T > 0 ? a->T : 1));
    double* qrot = (double*)malloc(sizeof(double) * (size_t)a->D);
    for (;;) {
        int64_t t = __atomic_fetch_add(&w->next, 1, __ATOMIC_RELAXED);
        if (t >= w->n_ids)
            break;
        one_row(w, w->row_ids[t], s, qrot);
    }
    free(s);
    free(qrot);
    return NULL;
}

static void run_threads(group_work* w, int n_threads)
{
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)n_threads);
    for (int t = 0; t < n_threads; ++t)
        pthread_create(&th[t], NULL, group_worker, w);
    for (int t = 0; t < n_threads; ++t)
        pthread_join(th[t], NULL);
    free(th);
}

int hlg_default_threads(void)
{
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

int hlg_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                  const int64_t* q_pos0, const int64_t* n_keys,
                  const int64_t* rot_from, int B, int S, int T, int Hq,
                  int Hkv, int D, int window, double rope_frac, double theta,
                  double scale, int64_t n_rows, const int32_t* rows,
                  double* out, double* lse, int n_threads)
{
    if (B <= 0 || S < 0 || T < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 ||
        D % 2 || Hq % Hkv || window < 0 || rope_frac < 0.0 || rope_frac > 1.0)
        return -1;
    for (int b = 0; b < B; ++b)
        if (n_keys[b] < 0 || n_keys[b] > T)
            return -1;
    for (int64_t r = 0; r < n_rows; ++r) {
        const int32_t* rw = rows + 3 * r;
        if (rw[0] < 0 || rw[0] >= B || rw[1] < 0 || rw[1] >= Hq || rw[2] < 0 || rw[2] >= S)
            return -1;
    }
    if (n_threads <= 0)
        n_threads = hlg_default_threads();

    attn_args a = {q, k, v, q_pos0, n_keys, rot_from, B, S, T, Hq, Hkv, D, window,
                   rope_frac, theta, scale, n_rows, rows, out, lse};
    int G = Hq / Hkv;
    int64_t* ids = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n_rows > 0 ? n_rows : 1));
    for (int b = 0; b < B; ++b) {
        for (int g = 0; g < Hkv; ++g) {
            int64_t n_ids = 0;
            for (int64_t r = 0; r < n_rows; ++r)
                if (rows[3 * r] == b && rows[3 * r + 1] / G == g)
                    ids[n_ids++] = r;
            if (n_ids == 0)
                continue;
            group_work w;
            memset(&w, 0, sizeof w);
            w.a = &a;
            w.b = b;
            w.g = g;
            w.row_ids = ids;
            w.n_ids = n_ids;
            w.krot = (double*)malloc(sizeof(double) * (size_t)(n_keys[b] > 0 ? n_keys[b] : 1) * (size_t)D);
            w.phase = 0;
            run_threads(&w, n_threads);
            w.phase = 1;
            run_threads(&w, n_threads);
            free(w.krot);
        }
    }
    free(ids);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Cache byte accounting.                                                   */
/* [WALK] 3b / [TECH] "Core Model Architecture": with K = V only one tensor */
/* is cached (the worked example caches 4 x 8 = 32 values instead of 64).   */
/* [CORP] "Shared KV Cache": a shared layer holds no cache of its own.      */
/* ------------------------------------------------------------------------ */
int64_t hlg_layer_cache_bytes(int64_t batch, int n_kv_heads, int64_t capacity,
                              int head_dim, int elem_bytes, int k_equals_v)
{
    int64_t one = batch * (int64_t)n_kv_heads * capacity * (int64_t)head_dim * elem_bytes;
    return k_equals_v ? one : 2 * one;
}

/* Total cache bytes of an n_layers stack; which = 0 all layers, 1 local    */
/* only, 2 global only. A shared layer with a source holds nothing.         */
int64_t hlg_stack_cache_bytes(int n_layers, int ratio, int n_shared,
                              int64_t batch, int elem_bytes,
                              int local_kv_heads, int local_head_dim, int64_t local_capacity,
                              int global_kv_heads, int global_head_dim, int64_t global_capacity,
                              int global_k_equals_v, int which)
{
    int64_t total = 0;
    for (int l = 0; l < n_layers; ++l) {
        int g = hlg_layer_is_global(n_layers, ratio, l);
        int src = hlg_share_source(n_layers, ratio, n_shared, l);
        if (g < 0 || src == -2)
            return -1;
        if (src >= 0 && src != l)
            continue;
        if ((which == 1 && g) || (which == 2 && !g))
            continue;
        total += g ? hlg_layer_cache_bytes(batch, global_kv_heads, global_capacity,
                                           global_head_dim, elem_bytes, global_k_equals_v)
                   : hlg_layer_cache_bytes(batch, local_kv_heads, local_capacity,
                                           local_head_dim, elem_bytes, 0);
    }
    return total;
}

/* ------------------------------------------------------------------------ */
/* int8 KV cache rows. "Gemma 4 Technical Report", Quantization and        */
/* Efficiency: a quantizer maps a channel's [min, max] onto the 2^b codes   */
/* with scale = (2^b - 1) / (max - min) and code = round((x - min) * scale),*/
/* and the dequantizer returns min + code / scale; Table 3 lists int8 KV    */
/* caching. Reading: b = 8, one (min, step) pair per cached row (one token, */
/* one KV head, all D channels), codes 0..255, round half to even, every    */
/* step of the code decision in fp32, step = (max - min) / 255 stored for   */
/* the dequantizer (min + code * step), and a constant row gets codes 0 and */
/* step 0. Inputs are bf16 (the rounded rotated keys, or the values).       */
/* ------------------------------------------------------------------------ */
int hlg_quantize_rows_u8(const uint16_t* x_bits, int64_t n_rows, int D, uint8_t* codes,
                         float* lo_out, float* step_out)
{
    if (!x_bits || !codes || !lo_out || !step_out || n_rows < 0 || D <= 0)
        return 1;
    for (int64_t r = 0; r < n_rows; ++r) {
        const uint16_t* x = x_bits + r * D;
        float lo = (float)bf16_bits_to_double(x[0]), hi = lo;
        for (int d = 1; d < D; ++d) {
            float v = (float)bf16_bits_to_double(x[d]);
            if (v < lo) lo = v;
            if (v > hi) hi = v;
        }
        volatile float range = hi - lo;      /* fp32, rounded once */
        if (range > 0.0f) {
            volatile float scale = 255.0f / range;
            for (int d = 0; d < D; ++d) {
                volatile float off = (float)bf16_bits_to_double(x[d]) - lo;
                volatile float t = off * scale;
                float c = nearbyintf(t);     /* default rounding: to nearest, ties to even */
                if (c < 0.0f) c = 0.0f;
                if (c > 255.0f) c = 255.0f;
                codes[r * D + d] = (uint8_t)c;
            }
            step_out[r] = range / 255.0f;
        } else {
            for (int d = 0; d < D; ++d)
                codes[r * D + d] = 0;
            step_out[r] = 0.0f;
        }
        lo_out[r] = lo;
    }
    return 0;
}

/* The dequantized row, in fp64: min + code * step. */
void hlg_dequantize_rows_u8(const uint8_t* codes, const float* lo, const float* step,
                            int64_t n_rows, int D, double* out)
{
    for (int64_t r = 0; r < n_rows; ++r)
        for (int d = 0; d < D; ++d)
            out[r * D + d] = (double)lo[r] + (double)codes[r * D + d] * (double)step[r];
}

/* Attention of one query row over a given list of keys and values (fp64,   */
/* already rotated), the definition written out ("Gemma 4: End-to-End       */
/* Architecture Walkthrough", 3a): s_j = scale <q, k_j>, out = sum_j        */
/* softmax(s)_j v_j, lse = log sum_j exp(s_j). Row r reads keys             */
/* key_begin[r] .. key_begin[r] + key_count[r] - 1 of k and v ([n][D]).     */
int hlg_attend_rows(const double* q, const double* k, const double* v, int64_t n_keys_total,
                    const int64_t* key_begin, const int64_t* key_count, int64_t n_rows, int D,
                    double scale, double* out, double* lse)
{
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t b = key_begin[r], n = key_count[r];
        if (b < 0 || n < 1 || b + n > n_keys_total)
            return 1;
        double* s = (double*)malloc((size_t)n * sizeof(double));
        if (!s)
            return 2;
        double m = -INFINITY;
        for (int64_t j = 0; j < n; ++j) {
            double acc = 0.0;
            for (int d = 0; d < D; ++d)
                acc += q[r * D + d] * k[(b + j) * D + d];
            s[j] = scale * acc;
            if (s[j] > m)
                m = s[j];
        }
        double z = 0.0;
        for (int64_t j = 0; j < n; ++j)
            z += exp(s[j] - m);
        for (int d = 0; d < D; ++d) {
            double acc = 0.0;
            for (int64_t j = 0; j < n; ++j)
                acc += exp(s[j] - m) * v[(b + j) * D + d];
            out[r * D + d] = acc / z;
        }
        lse[r] = m + log(z);
        free(s);
    }
    return 0;
}

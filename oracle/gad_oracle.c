/*
 * gad_oracle.c - CPU oracle for one step of gated grouped-query attention
 * decode over a paged FP8 E4M3 KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously-correct
 * definition that the CUDA path is checked against.  Only the tests, the
 * smoke check and the benchmark's CPU-baseline arm may load it.  It shares no
 * code, header, table or helper with the CUDA library, and the library never
 * calls it.
 *
 * Source of the method: the task page "Gated attention decode
 * (muse_attention_decode)", section "What to compute" (the six-line formula),
 * section "Shapes" (16 query heads, 2 KV heads, q_len 1 or 8 causal, sliding
 * window of the last 2,048 tokens with RoPE, or full attention without RoPE,
 * page size 1 or 64, cache scales 1 or 1/64) and section "Correctness" (the
 * reference attends to the step's own new FP8 entries).
 *
 * Everything is evaluated in double precision, literally:
 *   q, k, v, gate = split(qkv[t])
 *   q = rmsnorm(q) * 5.473 ; k = rmsnorm(k)             (per 64-wide head)
 *   q, k = rope(q, p), rope(k, p)                        (sliding layers)
 *   cache[cache_loc[t]] = fp8(k / k_scale), fp8(v / v_scale)
 *   a = softmax(q . K^T / 8) . V   over keys lo..p       (no tiling, no online softmax)
 *   out = rmsnorm(a) * sigmoid(gate)                     (per 64-wide head) -> bf16
 *
 * Readings where the page is silent (each is listed in the design notes):
 *   - rmsnorm: eps 1e-6, unit weights, over each 64-wide head.
 *   - rope: NeoX half-split pairs (i, i+32), angle p * 10000^(-2i/64).
 *   - window W: token at position p attends keys i with p-W < i <= p.
 *   - q head h reads KV head h / (hq / hkv); with 16 and 2 heads, h / 8.
 *   - qkv columns, for hq query and hkv KV heads of 64 dims:
 *     q[0, 64hq) | k[64hq, 64(hq+hkv)) | v[.., 64(hq+2hkv)) | gate[.., 64(2hq+2hkv)),
 *     i.e. q[0,1024) | k[1024,1152) | v[1152,1280) | gate[1280,2304) at 16 and 2.
 *   - "heads tp8" is 16 query and 2 KV heads per GPU (the page's section
 *     "Shapes"); "heads dp" gives each GPU all heads of the layer, 8 times
 *     as many: 128 and 16.  The step itself is the same formula.
 *   - a cache row holds the hkv heads' 64 codes each: 64 * hkv bytes.
 *   - cache scale: stored code = E4M3(x / scale), dequantised = code * scale.
 *   - fp8(): double -> float (round to nearest even), then float -> E4M3
 *     (round to nearest even, saturating to +-448, NaN kept).
 *   - All of the step's cache writes happen before any attention read.
 *
 * Blocks of more than 8 new tokens per request (the page "Prefill layer
 * (muse_prefill_layer)", q_len 753 and 16,384, section "What to compute")
 * are the same formula, causal within the block: token j at position p sees
 * the cached keys and the block's keys up to p (inside the window when there
 * is one); the code below is written for any L.
 *
 * The file also holds the output projection that follows the step in the
 * decoder layer (gado_oproj, at the end).
 *
 * Parity pins: tests/test_oracle_pins.py checks every function here against
 * closed forms, library routines and invariants that do not come from this
 * file.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GADO_HQ 16   /* query heads of the page's per-GPU shapes ("heads tp8") */
#define GADO_HKV 2   /* key/value heads of those shapes */
#define GADO_D 64

/* ------------------------------------------------------------------------- */
/* Number formats                                                             */
/* ------------------------------------------------------------------------- */

/* OCP FP8 E4M3 ("e4m3fn"): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits,
 * no infinities, NaN = S.1111.111, largest finite 448. */
double gado_e4m3_decode(uint8_t code) {
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 15;
    int m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);               /* subnormal: m * 2^-6 / 8 */
    else
        v = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -v : v;
}

/* float -> E4M3, round to nearest even, saturating: any magnitude that would
 * round past 448 becomes 448.  NaN maps to 0x7F.  -0 keeps its sign (0x80). */
uint8_t gado_e4m3_encode(float xf) {
    double x = (double)xf;
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs(x);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    int e;
    if (a < ldexp(1.0, -6)) {
        e = -6;                                  /* subnormal range shares 2^-9 spacing */
    } else {
        frexp(a, &e);
        e -= 1;                                  /* a in [2^e, 2^(e+1)) */
    }
    double quantum = ldexp(1.0, e - 3);          /* 3 mantissa bits */
    double n = nearbyint(a / quantum);           /* exact division; ties to even */
    double v = n * quantum;
    if (v == 0.0) return sign;
    if (v < ldexp(1.0, -6)) return (uint8_t)(sign | (int)(v / ldexp(1.0, -9)));
    frexp(v, &e);
    e -= 1;
    int m = (int)(v / ldexp(1.0, e - 3)) - 8;
    return (uint8_t)(sign | ((e + 7) << 3) | m);
}

double gado_bf16_decode(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* double -> bfloat16, one rounding, to nearest even. */
uint16_t gado_bf16_encode(double x) {
    if (isnan(x)) return 0x7FC0;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (a == 0.0) return sign;
    int e;
    if (a < ldexp(1.0, -126)) {
        e = -126;
    } else {
        frexp(a, &e);
        e -= 1;
    }
    double quantum = ldexp(1.0, e - 7);          /* 8 significant bits */
    double v = nearbyint(a / quantum) * quantum;
    if (v >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80);
    float f = (float)v;                          /* exact */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(sign | ((u >> 16) & 0x7FFF));
}

/* ------------------------------------------------------------------------- */
/* Per-head transforms                                                        */
/* ------------------------------------------------------------------------- */

/* y = x / sqrt(mean(x^2) + eps), unit weights. */
void gado_rmsnorm(const double* x, double* y, int n, double eps) {
    double ss = 0.0;
    for (int i = 0; i < n; ++i) ss += x[i] * x[i];
    double r = sqrt(ss / n + eps);
    for (int i = 0; i < n; ++i) y[i] = x[i] / r;
}

/* NeoX half-split rotary embedding, in place: dims (i, i + d/2) rotate by
 * angle pos * theta^(-2i/d). */
void gado_rope_neox(double* u, int d, double pos, double theta) {
    int half = d / 2;
    for (int i = 0; i < half; ++i) {
        double inv_freq = pow(theta, -2.0 * i / d);
        double phi = pos * inv_freq;
        double c = cos(phi), s = sin(phi);
        double x0 = u[i], x1 = u[i + half];
        u[i] = x0 * c - x1 * s;
        u[i + half] = x1 * c + x0 * s;
    }
}

static double gado_sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* ------------------------------------------------------------------------- */
/* The whole step                                                             */
/* ------------------------------------------------------------------------- */

enum {
    GADO_OK = 0,
    GADO_ERR_ARG = -1,
    GADO_ERR_PAGE = -2,    /* a key's page index is beyond the page-table row */
    GADO_ERR_ROW = -3,     /* a cache row is outside the cache */
    GADO_ERR_NOMEM = -4,
};

typedef struct {
    /* inputs */
    const int64_t* positions;
    const int32_t* page_table;
    const uint8_t* k_cache;
    const uint8_t* v_cache;
    const uint16_t* qkv;
    double k_scale, v_scale;
    int B, L, max_pages, page_size, window;
    int hq, hkv;            /* query heads, key/value heads */
    int64_t num_rows;
    const uint8_t* want;
    const double* qn;       /* [T, hq, 64] normalised (and rotated) queries */
    /* outputs */
    uint16_t* out;
    double* out_exact;
    double* attn_out;
    /* work split */
    int tid, nthreads;
    int status;
} gado_job;

/* Cache row holding key i of request b: page_table[b][i / ps] * ps + i % ps. */
static int gado_row(const gado_job* J, int b, int64_t i, int64_t* row) {
    int64_t page_idx = i / J->page_size;
    if (page_idx < 0 || page_idx >= J->max_pages) return GADO_ERR_PAGE;
    int64_t page = J->page_table[(int64_t)b * J->max_pages + page_idx];
    int64_t r = page * J->page_size + i % J->page_size;
    if (r < 0 || r >= J->num_rows) return GADO_ERR_ROW;
    *row = r;
    return GADO_OK;
}

/* softmax(q.K^T/8).V for one (token, query head), then the gated output norm. */
static int gado_one_head(gado_job* J, int t, int h, double* logits, int64_t cap) {
    const int b = t / J->L;
    const int hq = J->hq, hkv = J->hkv;
    const int g = h / (hq / hkv);
    const int64_t row_bytes = (int64_t)hkv * GADO_D;
    const int64_t p = J->positions[t];
    int64_t lo = 0;
    if (J->window > 0) {
        lo = p - J->window + 1;
        if (lo < 0) lo = 0;
    }
    const int64_t n = p - lo + 1;
    if (n <= 0 || n > cap) return GADO_ERR_ARG;
    const double* q = J->qn + ((int64_t)t * hq + h) * GADO_D;

    /* logits s_i = q . K_i / 8, K_i dequantised from the cache */
    double smax = -INFINITY;
    for (int64_t i = lo; i <= p; ++i) {
        int64_t row;
        int st = gado_row(J, b, i, &row);
        if (st) return st;
        const uint8_t* kr = J->k_cache + row * row_bytes + g * GADO_D;
        double dot = 0.0;
        for (int d = 0; d < GADO_D; ++d) dot += q[d] * (gado_e4m3_decode(kr[d]) * J->k_scale);
        double s = dot / 8.0;
        logits[i - lo] = s;
        if (s > smax) smax = s;
    }
    /* a = sum_i e^(s_i - max) V_i / sum_i e^(s_i - max) */
    double a[GADO_D];
    for (int d = 0; d < GADO_D; ++d) a[d] = 0.0;
    double den = 0.0;
    for (int64_t i = lo; i <= p; ++i) {
        int64_t row = 0;
        gado_row(J, b, i, &row);  /* checked by the first pass over the keys */
        const uint8_t* vr = J->v_cache + row * row_bytes + g * GADO_D;
        double w = exp(logits[i - lo] - smax);
        den += w;
        for (int d = 0; d < GADO_D; ++d) a[d] += w * (gado_e4m3_decode(vr[d]) * J->v_scale);
    }
    for (int d = 0; d < GADO_D; ++d) a[d] /= den;

    /* out = rmsnorm(a) * sigmoid(gate) */
    double an[GADO_D];
    gado_rmsnorm(a, an, GADO_D, 1e-6);
    const int64_t qkv_cols = (int64_t)(2 * hq + 2 * hkv) * GADO_D;
    const int64_t gate_off = (int64_t)(hq + 2 * hkv) * GADO_D;
    const uint16_t* row_qkv = J->qkv + (int64_t)t * qkv_cols;
    for (int d = 0; d < GADO_D; ++d) {
        double gate = gado_bf16_decode(row_qkv[gate_off + h * GADO_D + d]);
        double y = an[d] * gado_sigmoid(gate);
        int64_t o = (int64_t)t * ((int64_t)hq * GADO_D) + h * GADO_D + d;
        J->out[o] = gado_bf16_encode(y);
        if (J->out_exact) J->out_exact[o] = y;
        if (J->attn_out) J->attn_out[o] = a[d];
    }
    return GADO_OK;
}

static void* gado_worker(void* arg) {
    gado_job* J = (gado_job*)arg;
    const int T = J->B * J->L;
    /* longest key range of any token */
    int64_t cap = 1;
    for (int t = 0; t < T; ++t) {
        int64_t p = J->positions[t];
        int64_t n = (J->window > 0 && p + 1 > J->window) ? J->window : p + 1;
        if (n > cap) cap = n;
    }
    double* logits = (double*)malloc(sizeof(double) * (size_t)cap);
    if (!logits) {
        J->status = GADO_ERR_NOMEM;
        return NULL;
    }
    for (int64_t w = J->tid; w < (int64_t)T * J->hq; w += J->nthreads) {
        if (J->want && !J->want[w]) continue;
        int st = gado_one_head(J, (int)(w / J->hq), (int)(w % J->hq), logits, cap);
        if (st) {
            J->status = st;
            break;
        }
    }
    free(logits);
    return NULL;
}

/*
 * The whole step on host memory, for hq query heads and hkv key/value heads
 * of 64 dims (hq a positive multiple of hkv).
 *   qkv        bf16 bits [T, 64 * (2 hq + 2 hkv)], T = B * L, token t = b * L + j
 *   positions  [T]   position p of each token (attends keys lo..p)
 *   page_table [B, max_pages]
 *   cache_loc  [T]   cache row receiving token t's k and v
 *   k_cache, v_cache [num_rows, hkv, 64] E4M3 codes; rows cache_loc[] are written
 *   k_scale, v_scale  the cache scales (float, as the device holds them)
 *   window     > 0: sliding window size; <= 0: full attention
 *   use_rope   1: rotate q and k by their positions
 *   want       [T * hq] or NULL: compute only (t, h) with want[t*hq+h] != 0
 *   out        bf16 bits [T, 64 * hq]
 *   out_exact  [T, 64 * hq] or NULL: the output before bf16 rounding
 *   attn_out   [T, 64 * hq] or NULL: a = softmax(...) . V before the output norm
 * Returns 0, or a negative GADO_ERR_* code.
 */
int gado_attn_decode_heads(const uint16_t* qkv, const int64_t* positions, const int32_t* page_table,
                           const int64_t* cache_loc, uint8_t* k_cache, uint8_t* v_cache,
                           float k_scale, float v_scale, int B, int L, int hq, int hkv,
                           int max_pages, int64_t num_rows, int page_size, int window,
                           int use_rope, const uint8_t* want, uint16_t* out, double* out_exact,
                           double* attn_out, int nthreads) {
    if (B <= 0 || L <= 0 || max_pages <= 0 || num_rows <= 0 || page_size <= 0) return GADO_ERR_ARG;
    if (hq <= 0 || hkv <= 0 || hq % hkv != 0) return GADO_ERR_ARG;
    if (!(k_scale > 0.0f) || !(v_scale > 0.0f)) return GADO_ERR_ARG;
    if (nthreads < 1) nthreads = 1;
    const int T = B * L;
    const double ks = (double)k_scale, vs = (double)v_scale;
    const int64_t qkv_cols = (int64_t)(2 * hq + 2 * hkv) * GADO_D;
    const int64_t k_off = (int64_t)hq * GADO_D, v_off = (int64_t)(hq + hkv) * GADO_D;
    const int64_t row_bytes = (int64_t)hkv * GADO_D;

    double* qn = (double*)malloc(sizeof(double) * (size_t)T * hq * GADO_D);
    if (!qn) return GADO_ERR_NOMEM;

    /* Pass 1: split, QK-norm, RoPE, quantise and write this step's k, v. */
    for (int t = 0; t < T; ++t) {
        const uint16_t* row_qkv = qkv + (int64_t)t * qkv_cols;
        const double p = (double)positions[t];
        double u[GADO_D];
        for (int h = 0; h < hq; ++h) {
            for (int d = 0; d < GADO_D; ++d) u[d] = gado_bf16_decode(row_qkv[h * GADO_D + d]);
            double* qh = qn + ((int64_t)t * hq + h) * GADO_D;
            gado_rmsnorm(u, qh, GADO_D, 1e-6);
            for (int d = 0; d < GADO_D; ++d) qh[d] *= 5.473;
            if (use_rope) gado_rope_neox(qh, GADO_D, p, 10000.0);
        }
        int64_t row = cache_loc[t];
        if (row < 0 || row >= num_rows) {
            free(qn);
            return GADO_ERR_ROW;
        }
        for (int g = 0; g < hkv; ++g) {
            double kh[GADO_D];
            for (int d = 0; d < GADO_D; ++d) u[d] = gado_bf16_decode(row_qkv[k_off + g * GADO_D + d]);
            gado_rmsnorm(u, kh, GADO_D, 1e-6);
            if (use_rope) gado_rope_neox(kh, GADO_D, p, 10000.0);
            for (int d = 0; d < GADO_D; ++d) {
                double vv = gado_bf16_decode(row_qkv[v_off + g * GADO_D + d]);
                k_cache[row * row_bytes + g * GADO_D + d] = gado_e4m3_encode((float)(kh[d] / ks));
                v_cache[row * row_bytes + g * GADO_D + d] = gado_e4m3_encode((float)(vv / vs));
            }
        }
    }

    /* Pass 2: attention and the gated output norm, one (token, head) at a time. */
    gado_job* jobs = (gado_job*)calloc((size_t)nthreads, sizeof(gado_job));
    pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !th) {
        free(qn);
        free(jobs);
        free(th);
        return GADO_ERR_NOMEM;
    }
    for (int i = 0; i < nthreads; ++i) {
        gado_job* J = &jobs[i];
        J->positions = positions;
        J->page_table = page_table;
        J->k_cache = k_cache;
        J->v_cache = v_cache;
        J->qkv = qkv;
        J->k_scale = ks;
        J->v_scale = vs;
        J->B = B;
        J->L = L;
        J->max_pages = max_pages;
        J->page_size = page_size;
        J->window = window;
        J->hq = hq;
        J->hkv = hkv;
        J->num_rows = num_rows;
        J->want = want;
        J->qn = qn;
        J->out = out;
        J->out_exact = out_exact;
        J->attn_out = attn_out;
        J->tid = i;
        J->nthreads = nthreads;
        J->status = GADO_OK;
    }
    int status = GADO_OK;
    if (nthreads == 1) {
        gado_worker(&jobs[0]);
    } else {
        for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, gado_worker, &jobs[i]);
        for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    }
    for (int i = 0; i < nthreads; ++i)
        if (jobs[i].status) status = jobs[i].status;
    free(jobs);
    free(th);
    free(qn);
    return status;
}

/* The page's per-GPU shapes: 16 query heads and 2 key/value heads. */
int gado_attn_decode(const uint16_t* qkv, const int64_t* positions, const int32_t* page_table,
                     const int64_t* cache_loc, uint8_t* k_cache, uint8_t* v_cache, float k_scale,
                     float v_scale, int B, int L, int max_pages, int64_t num_rows, int page_size,
                     int window, int use_rope, const uint8_t* want, uint16_t* out, double* out_exact,
                     double* attn_out, int nthreads) {
    return gado_attn_decode_heads(qkv, positions, page_table, cache_loc, k_cache, v_cache, k_scale,
                                  v_scale, B, L, GADO_HQ, GADO_HKV, max_pages, num_rows, page_size,
                                  window, use_rope, want, out, out_exact, attn_out, nthreads);
}

/* ------------------------------------------------------------------------- */
/* Output projection                                                          */
/* ------------------------------------------------------------------------- */

typedef struct {
    const uint16_t *out, *o;
    int T, K, N;
    uint16_t* a;
    double* a_exact;
    int tid, nthreads;
} gado_oproj_job;

static void* gado_oproj_worker(void* arg) {
    gado_oproj_job* J = (gado_oproj_job*)arg;
    for (int n = J->tid; n < J->N; n += J->nthreads) {
        const uint16_t* orow = J->o + (int64_t)n * J->K;
        for (int t = 0; t < J->T; ++t) {
            const uint16_t* xrow = J->out + (int64_t)t * J->K;
            double acc = 0.0;
            for (int k = 0; k < J->K; ++k) acc += gado_bf16_decode(xrow[k]) * gado_bf16_decode(orow[k]);
            const int64_t i = (int64_t)t * J->N + n;
            J->a[i] = gado_bf16_encode(acc);
            if (J->a_exact) J->a_exact[i] = acc;
        }
    }
    return NULL;
}

/*
 * The projection that follows the attention in the decoder layer (the pages
 * "Decode layer (muse_decode_layer)" and "Prefill layer (muse_prefill_layer)",
 * section "What to compute": a = (rmsnorm(attention(q)) * sigmoid(g)) @ o.T,
 * the all-reduce after it being the identity on one GPU):
 *   a[t][n] = sum_k out[t][k] * o[n][k]
 * in double, k in index order, then one rounding to bf16.
 *   out      bf16 bits [T, K]  the attention step's output
 *   o        bf16 bits [N, K]  the projection weight (row n = hidden unit n)
 *   a        bf16 bits [T, N]
 *   a_exact  [T, N] or NULL: before the bf16 rounding
 * Returns 0, or GADO_ERR_ARG / GADO_ERR_NOMEM.
 */
int gado_oproj(const uint16_t* out, const uint16_t* o, int T, int K, int N, uint16_t* a,
               double* a_exact, int nthreads) {
    if (T <= 0 || K <= 0 || N <= 0 || !out || !o || !a) return GADO_ERR_ARG;
    if (nthreads < 1) nthreads = 1;
    gado_oproj_job* jobs = (gado_oproj_job*)calloc((size_t)nthreads, sizeof(gado_oproj_job));
    pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !th) {
        free(jobs);
        free(th);
        return GADO_ERR_NOMEM;
    }
    for (int i = 0; i < nthreads; ++i) {
        gado_oproj_job* J = &jobs[i];
        J->out = out;
        J->o = o;
        J->T = T;
        J->K = K;
        J->N = N;
        J->a = a;
        J->a_exact = a_exact;
        J->tid = i;
        J->nthreads = nthreads;
    }
    if (nthreads == 1) {
        gado_oproj_worker(&jobs[0]);
    } else {
        for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, gado_oproj_worker, &jobs[i]);
        for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    }
    free(jobs);
    free(th);
    return GADO_OK;
}


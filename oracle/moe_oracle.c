/*
 * moe_oracle.c -- plain fp64 CPU oracle of the K2-style MoE FFN layer forward.
 * TEST INFRASTRUCTURE ONLY (see moe_oracle.h): tests, the smoke check and the
 * benchmark's CPU-baseline leg load it; the CUDA library never does.
 *
 * Every function follows the step it names, in the pages' order and notation;
 * loops are written out plainly, with no blocking, fusion or reordering beyond
 * the definitions.  Threads (pthreads) only split independent tokens.
 */
#include "moe_oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- numbers */

double oracle_bf16_to_f64(uint16_t v) {
    uint32_t bits = ((uint32_t)v) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* One rounding from double to bf16 (8 significant bits), nearest-even.
 * rint() rounds to nearest, ties to even, in the default rounding mode. */
uint16_t oracle_f64_to_bf16(double v) {
    if (isnan(v)) return 0x7FC0;
    double a = fabs(v);
    double r;
    if (a == 0.0 || isinf(v)) {
        r = v;
    } else if (a < 0x1p-126) {                 /* bf16 subnormal: quantum 2^-133 */
        r = rint(v * 0x1p133) * 0x1p-133;
    } else {
        int e;
        double m = frexp(v, &e);               /* v = m * 2^e, 0.5 <= |m| < 1 */
        r = ldexp(rint(ldexp(m, 8)), e - 8);   /* keep 8 significant bits */
    }
    if (fabs(r) > 0x1.FEp127) r = copysign(INFINITY, v);   /* above max bf16 */
    float f = (float)r;                        /* exact: r is a bf16 value */
    uint32_t bits;
    memcpy(&bits, &f, sizeof bits);
    return (uint16_t)(bits >> 16);
}

void oracle_round_bf16(const double* in, uint16_t* out, size_t n) {
    for (size_t i = 0; i < n; ++i) out[i] = oracle_f64_to_bf16(in[i]);
}

/* scoring_func = sigmoid ("Kimi K2.5 deep dive", CH4.2) */
double oracle_sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

/* SiLU inside SwiGLU ("Kimi K2.5 Q&A", Q8.3 step 5: gate+up -> SiLU -> x -> down) */
double oracle_silu(double z) { return z / (1.0 + exp(-z)); }

/* ------------------------------------------------------------ thread pool */

typedef void (*oracle_task_fn)(void* ctx, int begin, int end);
typedef struct { oracle_task_fn fn; void* ctx; int begin, end; } oracle_span;

static void* oracle_span_main(void* p) {
    oracle_span* s = (oracle_span*)p;
    s->fn(s->ctx, s->begin, s->end);
    return NULL;
}

/* Split [0, n) into nthreads contiguous spans and run fn on each. */
static void oracle_parallel_for(int n, int nthreads, oracle_task_fn fn, void* ctx) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > n) nthreads = n;
    if (nthreads <= 1) {
        if (n > 0) fn(ctx, 0, n);
        return;
    }
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
    oracle_span* sp = (oracle_span*)malloc(sizeof(oracle_span) * (size_t)nthreads);
    int started = 0;
    for (int i = 0; i < nthreads; ++i) {
        sp[i].fn = fn;
        sp[i].ctx = ctx;
        sp[i].begin = (int)((long long)n * i / nthreads);
        sp[i].end = (int)((long long)n * (i + 1) / nthreads);
        if (pthread_create(&th[i], NULL, oracle_span_main, &sp[i]) == 0) {
            started = i + 1;
        } else {                                /* no thread: run it here */
            oracle_span_main(&sp[i]);
            th[i] = (pthread_t)0;
        }
    }
    for (int i = 0; i < started; ++i)
        if (th[i]) pthread_join(th[i], NULL);
    free(th);
    free(sp);
}

/* ----------------------------------------------------------------- router */

typedef struct {
    const uint16_t* x; const uint16_t* w_router; const float* bias;
    int d, E, k; double scale;
    int32_t* topk_idx; double* topk_w; double* scores; double* gap;
} route_ctx;

static void route_tokens(void* p, int t0, int t1) {
    route_ctx* c = (route_ctx*)p;
    const int d = c->d, E = c->E, k = c->k;
    double* s = (double*)malloc(sizeof(double) * (size_t)E);
    double* b = (double*)malloc(sizeof(double) * (size_t)E);
    unsigned char* taken = (unsigned char*)malloc((size_t)E);
    for (int t = t0; t < t1; ++t) {
        const uint16_t* xt = c->x + (size_t)t * d;
        /* 1. logits = x . W_router^T, s = sigmoid(logits) */
        for (int e = 0; e < E; ++e) {
            const uint16_t* we = c->w_router + (size_t)e * d;
            double acc = 0.0;
            for (int i = 0; i < d; ++i)
                acc += oracle_bf16_to_f64(xt[i]) * oracle_bf16_to_f64(we[i]);
            s[e] = oracle_sigmoid(acc);
            /* 2. biased score, used for selection only */
            b[e] = s[e] + (double)c->bias[e];
            taken[e] = 0;
        }
        /* 3. top-k of b: k rounds of "largest remaining, lowest index on ties" */
        double kth = 0.0;
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || b[e] > b[best]) best = e;
            }
            taken[best] = 1;
            c->topk_idx[(size_t)t * k + j] = best;
            kth = b[best];
        }
        /* sum of the unbiased scores over the selected SET (taken in expert
         * order, so it depends on the set only, not on the slot order) */
        double sum = 0.0;
        for (int e = 0; e < E; ++e)
            if (taken[e]) sum += s[e];
        if (c->gap) {
            double next = -INFINITY;
            for (int e = 0; e < E; ++e)
                if (!taken[e] && b[e] > next) next = b[e];
            c->gap[t] = (k < E) ? (kth - next) : INFINITY;
        }
        /* 4. weights from the UNBIASED scores, renormalised, then scaled */
        for (int j = 0; j < k; ++j) {
            int e = c->topk_idx[(size_t)t * k + j];
            c->topk_w[(size_t)t * k + j] = c->scale * (s[e] / sum);
        }
        if (c->scores) memcpy(c->scores + (size_t)t * E, s, sizeof(double) * (size_t)E);
    }
    free(s);
    free(b);
    free(taken);
}

int oracle_route(const uint16_t* x, const uint16_t* w_router, const float* bias,
                 int T, int d, int E, int k, double scale,
                 int32_t* topk_idx, double* topk_w, double* scores, double* gap,
                 int nthreads) {
    if (T < 0 || d <= 0 || E <= 0 || k <= 0 || k > E) return -1;
    if (T == 0) return 0;
    if (!x || !w_router || !bias || !topk_idx || !topk_w) return -1;
    route_ctx c = {x, w_router, bias, d, E, k, scale, topk_idx, topk_w, scores, gap};
    oracle_parallel_for(T, nthreads, route_tokens, &c);
    return 0;
}

/* ------------------------------------------------------------ permutation */

int oracle_permute(const int32_t* topk_idx, int T, int E, int k,
                   int32_t* counts, int32_t* offsets, int32_t* row_token, int32_t* slot_row) {
    if (T < 0 || E <= 0 || k <= 0) return -1;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    /* per-expert histogram */
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int e = topk_idx[(size_t)t * k + j];
            if (e < 0 || e >= E) return -1;
            for (int jj = 0; jj < j; ++jj)
                if (topk_idx[(size_t)t * k + jj] == e) return -1;
            counts[e] += 1;
        }
    /* exclusive prefix sum */
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    /* the pages' per-expert mask: for expert e, visit tokens in order */
    for (int e = 0; e < E; ++e) {
        int row = offsets[e];
        for (int t = 0; t < T; ++t)
            for (int j = 0; j < k; ++j)
                if (topk_idx[(size_t)t * k + j] == e) {
                    row_token[row] = t;
                    slot_row[(size_t)t * k + j] = row;
                    ++row;
                }
    }
    return 0;
}

/* ---------------------------------------------------------- SwiGLU expert */

void oracle_swiglu_row(const uint16_t* xrow, const uint16_t* w_gate_up, const uint16_t* w_down,
                       int d, int inter, double* y, double* act) {
    double* a = act ? act : (double*)malloc(sizeof(double) * (size_t)inter);
    for (int n = 0; n < inter; ++n) {
        const uint16_t* wg = w_gate_up + (size_t)n * d;             /* gate_proj row n */
        const uint16_t* wu = w_gate_up + (size_t)(inter + n) * d;   /* up_proj row n */
        double g = 0.0, u = 0.0;
        for (int i = 0; i < d; ++i) {
            double xi = oracle_bf16_to_f64(xrow[i]);
            g += oracle_bf16_to_f64(wg[i]) * xi;
            u += oracle_bf16_to_f64(wu[i]) * xi;
        }
        a[n] = oracle_silu(g) * u;
    }
    for (int o = 0; o < d; ++o) {                                    /* down_proj */
        const uint16_t* wd = w_down + (size_t)o * inter;
        double acc = 0.0;
        for (int n = 0; n < inter; ++n) acc += oracle_bf16_to_f64(wd[n]) * a[n];
        y[o] = acc;
    }
    if (!act) free(a);
}

/* ---------------------------------------------------------------- combine */

void oracle_combine(const double* y, const double* y_shared, const double* topk_w,
                    const int32_t* slot_row, int T, int d, int k, double* out) {
    for (int t = 0; t < T; ++t) {
        double* o = out + (size_t)t * d;
        for (int i = 0; i < d; ++i) o[i] = y_shared ? y_shared[(size_t)t * d + i] : 0.0;
        for (int j = 0; j < k; ++j) {
            double w = topk_w[(size_t)t * k + j];
            const double* yr = y + (size_t)slot_row[(size_t)t * k + j] * d;
            for (int i = 0; i < d; ++i) o[i] += w * yr[i];
        }
    }
}

/* ------------------------------------------------------------ whole layer */

typedef struct {
    const uint16_t* x; int d, k, inter;
    const int32_t* topk_idx; const double* topk_w;
    const uint16_t* const* egu; const uint16_t* const* edn;
    const uint16_t* sgu; const uint16_t* sdn;
    const int32_t* tokens; double* out;
} rows_ctx;

static void rows_tokens(void* p, int r0, int r1) {
    rows_ctx* c = (rows_ctx*)p;
    const int d = c->d, k = c->k;
    double* y = (double*)malloc(sizeof(double) * (size_t)d);
    for (int r = r0; r < r1; ++r) {
        int t = c->tokens ? c->tokens[r] : r;
        const uint16_t* xt = c->x + (size_t)t * d;
        double* o = c->out + (size_t)r * d;
        /* step 5: shared expert, every token, unscaled */
        oracle_swiglu_row(xt, c->sgu, c->sdn, d, c->inter, o, NULL);
        /* steps 6-7: routed experts, weighted and added */
        for (int j = 0; j < k; ++j) {
            int e = c->topk_idx[(size_t)t * k + j];
            double w = c->topk_w[(size_t)t * k + j];
            oracle_swiglu_row(xt, c->egu[e], c->edn[e], d, c->inter, y, NULL);
            for (int i = 0; i < d; ++i) o[i] += w * y[i];
        }
    }
    free(y);
}

int oracle_moe_rows(const uint16_t* x, int T, int d, int E, int k, int inter,
                    const int32_t* topk_idx, const double* topk_w,
                    const uint16_t* const* expert_gate_up, const uint16_t* const* expert_down,
                    const uint16_t* shared_gate_up, const uint16_t* shared_down,
                    const int32_t* tokens, int n_tokens, double* out, int nthreads) {
    if (!shared_gate_up || !shared_down) return -1;
    if (!tokens) n_tokens = T;
    for (int r = 0; r < n_tokens; ++r) {
        int t = tokens ? tokens[r] : r;
        if (t < 0 || t >= T) return -1;
        for (int j = 0; j < k; ++j) {
            int e = topk_idx[(size_t)t * k + j];
            if (e < 0 || e >= E || !expert_gate_up[e] || !expert_down[e]) return -1;
        }
    }
    rows_ctx c = {x, d, k, inter, topk_idx, topk_w, expert_gate_up, expert_down,
                  shared_gate_up, shared_down, tokens, out};
    oracle_parallel_for(n_tokens, nthreads, rows_tokens, &c);
    return 0;
}

/* ------------------------------------------------------- FP8 (E4M3) storage */

uint8_t oracle_e4m3_encode(double v) {
    if (isnan(v)) return 0x7F;
    const uint8_t sign = signbit(v) ? 0x80 : 0x00;
    const double a = fabs(v);
    if (a >= 448.0) return sign | 0x7E;                 /* largest finite: 1.75 * 2^8 */
    if (a < 0x1p-6) {                                   /* subnormal range: step 2^-9 */
        const double m = rint(a * 0x1p9);               /* 0 .. 8, ties to even */
        return sign | (uint8_t)m;                       /* m == 8 is the code of 2^-6 */
    }
    int e = ilogb(a);                                   /* 2^e <= a < 2^(e+1), -6 <= e <= 8 */
    double m = rint(ldexp(a, 3 - e));                   /* 8 .. 16: 1.mmm scaled by 8 */
    if (m == 16.0) {
        m = 8.0;
        e += 1;
    }
    if (e > 8 || (e == 8 && m > 14.0)) return sign | 0x7E;
    return sign | (uint8_t)(((e + 7) << 3) | ((int)m - 8));
}

double oracle_e4m3_decode(uint8_t code) {
    const int ex = (code >> 3) & 0xF, man = code & 0x7;
    if (ex == 0xF && man == 0x7) return NAN;
    const double mag = ex == 0 ? ldexp((double)man, -9) : ldexp(1.0 + man / 8.0, ex - 7);
    return (code & 0x80) ? -mag : mag;
}

int oracle_fp8_block_exponent(double amax) {
    if (!(amax > 0.0)) return 0;
    int s = ilogb(amax) - 8;                            /* amax < 2^(s+9) */
    if (amax > ldexp(448.0, s)) s += 1;                 /* now amax <= 448 * 2^s */
    while (s > -1000 && amax <= ldexp(448.0, s - 1)) s -= 1;   /* smallest such s */
    if (s < -124) s = -124;
    if (s > 127) s = 127;
    return s;
}

int oracle_quantize_fp8(const uint16_t* w, int64_t rows, int64_t cols, uint8_t* q, int8_t* sexp) {
    if (rows <= 0 || cols <= 0 || rows % 128 || cols % 128) return -1;
    const int64_t bc = cols / 128;
    for (int64_t br = 0; br < rows / 128; ++br)
        for (int64_t bk = 0; bk < bc; ++bk) {
            double amax = 0.0;
            for (int64_t r = br * 128; r < br * 128 + 128; ++r)
                for (int64_t c = bk * 128; c < bk * 128 + 128; ++c) {
                    const double a = fabs(oracle_bf16_to_f64(w[r * cols + c]));
                    if (a > amax) amax = a;
                }
            const int s = oracle_fp8_block_exponent(amax);
            sexp[br * bc + bk] = (int8_t)s;
            for (int64_t r = br * 128; r < br * 128 + 128; ++r)
                for (int64_t c = bk * 128; c < bk * 128 + 128; ++c)
                    q[r * cols + c] = oracle_e4m3_encode(ldexp(oracle_bf16_to_f64(w[r * cols + c]), -s));
        }
    return 0;
}

int oracle_dequantize_fp8(const uint8_t* q, const int8_t* sexp, int64_t rows, int64_t cols,
                          uint16_t* w_out) {
    if (rows <= 0 || cols <= 0 || rows % 128 || cols % 128) return -1;
    const int64_t bc = cols / 128;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            w_out[r * cols + c] = oracle_f64_to_bf16(
                ldexp(oracle_e4m3_decode(q[r * cols + c]), sexp[(r / 128) * bc + c / 128]));
    return 0;
}

/* ------------------------------------------------------------ load balance */

void oracle_bias_update(const int32_t* counts, int T, int E, int k, float gamma, float* bias) {
    const long long total = (long long)T * k;
    for (int e = 0; e < E; ++e) {
        const long long scaled = (long long)counts[e] * E;     /* load vs mean, exactly */
        float b = bias[e];
        if (scaled > total)
            b = b - gamma;                                    /* over-loaded: lower */
        else if (scaled < total)
            b = b + gamma;                                    /* under-loaded: raise */
        bias[e] = b;
    }
}

void oracle_seq_aux_loss(const double* scores, const int32_t* topk_idx, int B, int S, int E,
                         int k, double alpha, double* loss, double* f, double* p) {
    double* fb = (double*)calloc((size_t)E, sizeof(double));
    double* pb = (double*)calloc((size_t)E, sizeof(double));
    for (int b = 0; b < B; ++b) {
        for (int i = 0; i < E; ++i) fb[i] = pb[i] = 0.0;
        for (int t = b * S; t < (b + 1) * S; ++t) {
            for (int j = 0; j < k; ++j) fb[topk_idx[(size_t)t * k + j]] += 1.0;
            double tot = 0.0;
            for (int i = 0; i < E; ++i) tot += scores[(size_t)t * E + i];
            for (int i = 0; i < E; ++i) pb[i] += scores[(size_t)t * E + i] / tot;
        }
        double l = 0.0;
        for (int i = 0; i < E; ++i) {
            fb[i] *= (double)E / ((double)k * S);
            pb[i] /= S;
            l += fb[i] * pb[i];
            if (f) f[(size_t)b * E + i] = fb[i];
            if (p) p[(size_t)b * E + i] = pb[i];
        }
        loss[b] = alpha * l;
    }
    free(fb);
    free(pb);
}

/* ------------------------------------------------------------- FP8 compute */

/* quantize n values (bf16 bits, or doubles already bf16-exact) with one exponent */
static int quantize_row_f64(const double* v, int64_t n, uint8_t* q) {
    double amax = 0.0;
    for (int64_t i = 0; i < n; ++i)
        if (fabs(v[i]) > amax) amax = fabs(v[i]);
    const int s = oracle_fp8_block_exponent(amax);
    for (int64_t i = 0; i < n; ++i) q[i] = oracle_e4m3_encode(ldexp(v[i], -s));
    return s;
}

void oracle_quantize_fp8_rows(const uint16_t* w, int64_t rows, int64_t cols, uint8_t* q,
                              int8_t* sexp) {
    double* v = (double*)calloc((size_t)cols, sizeof(double));
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t c = 0; c < cols; ++c) v[c] = oracle_bf16_to_f64(w[r * cols + c]);
        sexp[r] = (int8_t)quantize_row_f64(v, cols, q + r * cols);
    }
    free(v);
}

void oracle_swiglu_row_fp8(const uint16_t* xrow, const uint8_t* wq_gu, const int8_t* s_gu,
                           const uint8_t* wq_dn, const int8_t* s_dn, int d, int inter, double* y) {
    double* xv = (double*)calloc((size_t)d, sizeof(double));
    uint8_t* xq = (uint8_t*)malloc((size_t)d);
    double* h = (double*)calloc((size_t)inter, sizeof(double));
    uint8_t* hq = (uint8_t*)malloc((size_t)inter);
    double* xd = (double*)malloc(sizeof(double) * (size_t)d);
    double* hd = (double*)malloc(sizeof(double) * (size_t)inter);
    for (int i = 0; i < d; ++i) xv[i] = oracle_bf16_to_f64(xrow[i]);
    const int sx = quantize_row_f64(xv, d, xq);
    for (int i = 0; i < d; ++i) xd[i] = oracle_e4m3_decode(xq[i]);
    for (int n = 0; n < inter; ++n) {
        const uint8_t* wg = wq_gu + (size_t)n * d;
        const uint8_t* wu = wq_gu + (size_t)(inter + n) * d;
        double g = 0.0, u = 0.0;
        for (int i = 0; i < d; ++i) {
            g += oracle_e4m3_decode(wg[i]) * xd[i];
            u += oracle_e4m3_decode(wu[i]) * xd[i];
        }
        g = ldexp(g, s_gu[n] + sx);
        u = ldexp(u, s_gu[inter + n] + sx);
        /* the stored intermediate is bf16 */
        h[n] = oracle_bf16_to_f64(oracle_f64_to_bf16(oracle_silu(g) * u));
    }
    const int sh = quantize_row_f64(h, inter, hq);
    for (int n = 0; n < inter; ++n) hd[n] = oracle_e4m3_decode(hq[n]);
    for (int o = 0; o < d; ++o) {
        const uint8_t* wd = wq_dn + (size_t)o * inter;
        double acc = 0.0;
        for (int n = 0; n < inter; ++n) acc += oracle_e4m3_decode(wd[n]) * hd[n];
        y[o] = ldexp(acc, s_dn[o] + sh);
    }
    free(xv); free(xq); free(h); free(hq); free(xd); free(hd);
}

typedef struct {
    const uint16_t* x; int d, k, inter;
    const int32_t* topk_idx; const double* topk_w;
    const uint8_t* const* egq; const int8_t* const* egs;
    const uint8_t* const* edq; const int8_t* const* eds;
    const uint8_t* sgq; const int8_t* sgs; const uint8_t* sdq; const int8_t* sds;
    const int32_t* tokens; double* out;
} rows8_ctx;

static void rows8_tokens(void* p, int r0, int r1) {
    rows8_ctx* c = (rows8_ctx*)p;
    const int d = c->d, k = c->k;
    double* y = (double*)malloc(sizeof(double) * (size_t)d);
    for (int r = r0; r < r1; ++r) {
        int t = c->tokens ? c->tokens[r] : r;
        const uint16_t* xt = c->x + (size_t)t * d;
        double* o = c->out + (size_t)r * d;
        oracle_swiglu_row_fp8(xt, c->sgq, c->sgs, c->sdq, c->sds, d, c->inter, o);
        for (int j = 0; j < k; ++j) {
            int e = c->topk_idx[(size_t)t * k + j];
            double w = c->topk_w[(size_t)t * k + j];
            oracle_swiglu_row_fp8(xt, c->egq[e], c->egs[e], c->edq[e], c->eds[e], d, c->inter, y);
            for (int i = 0; i < d; ++i) o[i] += y[i] * w;
        }
    }
    free(y);
}

int oracle_moe_rows_fp8(const uint16_t* x, int T, int d, int E, int k, int inter,
                        const int32_t* topk_idx, const double* topk_w,
                        const uint8_t* const* egu_q, const int8_t* const* egu_s,
                        const uint8_t* const* edn_q, const int8_t* const* edn_s,
                        const uint8_t* sgu_q, const int8_t* sgu_s, const uint8_t* sdn_q,
                        const int8_t* sdn_s, const int32_t* tokens, int n_tokens, double* out,
                        int nthreads) {
    if (!sgu_q || !sgu_s || !sdn_q || !sdn_s) return -1;
    if (!tokens) n_tokens = T;
    for (int r = 0; r < n_tokens; ++r) {
        int t = tokens ? tokens[r] : r;
        if (t < 0 || t >= T) return -1;
        for (int j = 0; j < k; ++j) {
            int e = topk_idx[(size_t)t * k + j];
            if (e < 0 || e >= E || !egu_q[e] || !egu_s[e] || !edn_q[e] || !edn_s[e]) return -1;
        }
    }
    rows8_ctx c = {x, d, k, inter, topk_idx, topk_w, egu_q, egu_s, edn_q, edn_s,
                   sgu_q, sgu_s, sdn_q, sdn_s, tokens, out};
    oracle_parallel_for(n_tokens, nthreads, rows8_tokens, &c);
    return 0;
}

/* ------------------------------------------------------------ INT4 storage */

int oracle_quantize_int4(const uint16_t* w, int64_t rows, int64_t cols, int8_t* q,
                         uint16_t* scale) {
    if (rows < 0 || cols < 0 || cols % 32 != 0) return -1;
    const int64_t groups = cols / 32;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t g = 0; g < groups; ++g) {
            const uint16_t* wg = w + r * cols + g * 32;
            int8_t* qg = q + r * cols + g * 32;
            double amax = 0.0;
            for (int i = 0; i < 32; ++i) {
                const double v = fabs(oracle_bf16_to_f64(wg[i]));
                if (v > amax) amax = v;
            }
            const uint16_t sb = oracle_f64_to_bf16(amax / 7.0);
            scale[r * groups + g] = sb;
            const double sv = oracle_bf16_to_f64(sb);
            for (int i = 0; i < 32; ++i) {
                double n = 0.0;
                if (sv != 0.0) {
                    n = rint(oracle_bf16_to_f64(wg[i]) / sv);      /* ties to even */
                    if (n > 7.0) n = 7.0;
                    if (n < -8.0) n = -8.0;
                }
                qg[i] = (int8_t)n;
            }
        }
    }
    return 0;
}

int oracle_dequantize_int4(const int8_t* q, const uint16_t* scale, int64_t rows, int64_t cols,
                           uint16_t* w_out) {
    if (rows < 0 || cols < 0 || cols % 32 != 0) return -1;
    const int64_t groups = cols / 32;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            w_out[r * cols + c] = oracle_f64_to_bf16(
                (double)q[r * cols + c] * oracle_bf16_to_f64(scale[r * groups + c / 32]));
    return 0;
}

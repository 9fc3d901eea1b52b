/*
 * g4attn_oracle.c -- plain fp64 CPU oracle (test infrastructure only; see the header).
 *
 * Written from the method's definitions, step by step, with no blocking, fusion or
 * online-softmax rewrite: each query row builds its full score vector, takes the
 * max, exponentiates, normalises and sums the values.  Host threads only split the
 * independent (head, row) work items.
 */
#include "g4attn_oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdatomic.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* bf16 bits -> double: a bf16 value is the top half of an IEEE binary32. */
static double bf16_to_double(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int g4o_rope_pairs(int head_dim, double rope_p) {
    /* Only the first fraction p of the d/2 rotary pairs carry position
     * (Gemma 4 report section 2: p-RoPE with p = 0.25 on global layers;
     *  explainer "p-RoPE": the first 25% of pairs rotate, the rest do not). */
    double r = floor(rope_p * (double)head_dim / 2.0);
    if (r < 0) r = 0;
    if (r > head_dim / 2) r = head_dim / 2;
    return (int)r;
}

void g4o_rmsnorm(const double* x, const double* gamma, int d, double eps, double* y) {
    /* QKNorm = RMSNorm over head_dim with a learned per-dim gain
     * (Gemma 4 report section 2: pre-norm, post-norm and QKNorm, all RMSNorm). */
    double ss = 0.0;
    for (int c = 0; c < d; ++c) ss += x[c] * x[c];
    double inv = 1.0 / sqrt(ss / (double)d + eps);
    for (int c = 0; c < d; ++c) y[c] = x[c] * inv * (gamma ? gamma[c] : 1.0);
}

void g4o_rope(const double* x, int d, int R, double base, int64_t pos, double* y) {
    /* RoPE cuts the vector into pairs and turns each pair by an angle that shrinks
     * from the first pair to the last (explainer "p-RoPE" section).  Pair i is
     * (x_i, x_{i+d/2}); angle phi_i = pos * base^(-2i/d); direction (cos -sin; sin cos).
     * Pairs i >= R keep angle 0 (p-RoPE: the low-frequency pairs carry no position). */
    int half = d / 2;
    if (y != x) memcpy(y, x, sizeof(double) * (size_t)d);
    for (int i = 0; i < R; ++i) {
        double theta = pow(base, -2.0 * (double)i / (double)d);
        double phi = (double)pos * theta;
        double c = cos(phi), s = sin(phi);
        double a = x[i], b = x[i + half];
        y[i] = a * c - b * s;
        y[i + half] = a * s + b * c;
    }
}

static int cfg_valid(const g4o_cfg* cfg) {
    if (!cfg) return 0;
    if (cfg->n_q_heads <= 0 || cfg->n_kv_heads <= 0) return 0;
    if (cfg->n_q_heads % cfg->n_kv_heads != 0) return 0;
    if (cfg->head_dim <= 0 || (cfg->head_dim & 1)) return 0;
    if (cfg->window < 0) return 0;
    if (cfg->kv_is_k < 0 || cfg->kv_is_k > 2) return 0;
    return 1;
}

static int online_cores(int nthreads) {
    if (nthreads > 0) return nthreads;
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

/* Load one row of bf16 bits, normalise it (when QKNorm is on) into y. */
static void load_norm(const uint16_t* src, const double* gamma, const g4o_cfg* cfg,
                      double* tmp, double* y) {
    int d = cfg->head_dim;
    for (int c = 0; c < d; ++c) tmp[c] = bf16_to_double(src[c]);
    if (cfg->qk_norm)
        g4o_rmsnorm(tmp, gamma, d, cfg->qk_norm_eps, y);
    else
        memcpy(y, tmp, sizeof(double) * (size_t)d);
}

int g4o_qknorm_rope(const uint16_t* q_in, const uint16_t* k_in,
                    const float* gamma_q, const float* gamma_k,
                    int B, int T, int64_t pos0, const g4o_cfg* cfg,
                    double* q_out, double* k_out, double* krot_out) {
    if (!cfg_valid(cfg) || B < 0 || T < 0) return -1;
    int d = cfg->head_dim, Hq = cfg->n_q_heads, Hkv = cfg->n_kv_heads;
    int R = g4o_rope_pairs(d, cfg->rope_p);
    double* gq = malloc(sizeof(double) * (size_t)d);
    double* gk = malloc(sizeof(double) * (size_t)d);
    double* tmp = malloc(sizeof(double) * (size_t)d);
    double* y = malloc(sizeof(double) * (size_t)d);
    for (int c = 0; c < d; ++c) {
        gq[c] = gamma_q ? (double)gamma_q[c] : 1.0;
        gk[c] = gamma_k ? (double)gamma_k[c] : 1.0;
    }
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t) {
            int64_t pos = pos0 + t;
            if (q_in && q_out)
                for (int h = 0; h < Hq; ++h) {
                    size_t off = (((size_t)b * T + t) * Hq + h) * (size_t)d;
                    load_norm(q_in + off, gq, cfg, tmp, y);
                    g4o_rope(y, d, R, cfg->rope_base, pos, q_out + off);
                }
            if (k_in)
                for (int g = 0; g < Hkv; ++g) {
                    size_t off = (((size_t)b * T + t) * Hkv + g) * (size_t)d;
                    load_norm(k_in + off, gk, cfg, tmp, y);
                    if (k_out) memcpy(k_out + off, y, sizeof(double) * (size_t)d);
                    if (krot_out) g4o_rope(y, d, R, cfg->rope_base, pos, krot_out + off);
                }
        }
    free(gq); free(gk); free(tmp); free(y);
    return 0;
}

/* ------------------------------------------------------------------------------ */
/* One query row against an explicit list of key/value rows: the attention sum.   */
/* ------------------------------------------------------------------------------ */
static void attend_row(const double* qr, const double* krot, const double* vals,
                       int64_t lo, int64_t hi, int d, double scale, double* s,
                       double* out, double* lse) {
    /* keys lo..hi inclusive; krot/vals are indexed by key position */
    double m = -INFINITY;
    for (int64_t j = lo; j <= hi; ++j) {
        const double* kj = krot + (size_t)j * d;
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += qr[c] * kj[c];
        s[j - lo] = scale * acc;
        if (s[j - lo] > m) m = s[j - lo];
    }
    for (int c = 0; c < d; ++c) out[c] = 0.0;
    if (hi < lo) { if (lse) *lse = -INFINITY; return; }
    double l = 0.0;
    for (int64_t j = lo; j <= hi; ++j) l += exp(s[j - lo] - m);
    for (int64_t j = lo; j <= hi; ++j) {
        double w = exp(s[j - lo] - m) / l;
        const double* vj = vals + (size_t)j * d;
        for (int c = 0; c < d; ++c) out[c] += w * vj[c];
    }
    if (lse) *lse = m + log(l);
}

typedef struct {
    /* shared, read-only */
    const uint16_t* q;
    const double* gq;
    const g4o_cfg* cfg;
    const double* krot;   /* [T, d] for this (b, g) */
    const double* vals;   /* [T, d] */
    const int32_t* rows;
    int nrows, B, T, b, g, G, R;
    double* out;
    double* lse;
    atomic_long next;     /* work item counter over (h_local, row) */
} prefill_job;

static void* prefill_worker(void* arg) {
    prefill_job* J = (prefill_job*)arg;
    const g4o_cfg* cfg = J->cfg;
    int d = cfg->head_dim, Hq = cfg->n_q_heads;
    double* tmp = malloc(sizeof(double) * (size_t)d);
    double* qn = malloc(sizeof(double) * (size_t)d);
    double* qr = malloc(sizeof(double) * (size_t)d);
    double* s = malloc(sizeof(double) * (size_t)(J->T > 0 ? J->T : 1));
    long total = (long)J->G * J->nrows;
    for (;;) {
        long it = atomic_fetch_add(&J->next, 1);
        if (it >= total) break;
        int hl = (int)(it / J->nrows), ri = (int)(it % J->nrows);
        int h = J->g * J->G + hl;
        int64_t i = J->rows[ri];
        size_t qoff = (((size_t)J->b * J->T + (size_t)i) * Hq + h) * (size_t)d;
        load_norm(J->q + qoff, J->gq, cfg, tmp, qn);
        g4o_rope(qn, d, J->R, cfg->rope_base, i, qr);
        int64_t lo = 0;
        if (cfg->window > 0 && i - cfg->window + 1 > 0) lo = i - cfg->window + 1;
        double* o = J->out + (((size_t)J->b * J->nrows + ri) * Hq + h) * (size_t)d;
        double* l = J->lse ? J->lse + ((size_t)J->b * Hq + h) * J->nrows + ri : NULL;
        attend_row(qr, J->krot, J->vals, lo, i, d, cfg->scale, s, o, l);
    }
    free(tmp); free(qn); free(qr); free(s);
    return NULL;
}

typedef struct {
    const uint16_t* k;
    const uint16_t* v;
    const double* gk;
    const g4o_cfg* cfg;
    int T, b, g, R, Hkv;
    int64_t jmax;
    double* khat;
    double* krot;
    double* vals;
    atomic_long next;
} keyprep_job;

static void* keyprep_worker(void* arg) {
    keyprep_job* J = (keyprep_job*)arg;
    const g4o_cfg* cfg = J->cfg;
    int d = cfg->head_dim;
    double* tmp = malloc(sizeof(double) * (size_t)d);
    for (;;) {
        long j = atomic_fetch_add(&J->next, 1);
        if (j > J->jmax) break;
        size_t off = (((size_t)J->b * J->T + (size_t)j) * J->Hkv + J->g) * (size_t)d;
        double* kh = J->khat + (size_t)j * d;
        load_norm(J->k + off, J->gk, cfg, tmp, kh);
        g4o_rope(kh, d, J->R, cfg->rope_base, j, J->krot + (size_t)j * d);
        if (cfg->kv_is_k == 0) {
            double* vv = J->vals + (size_t)j * d;
            for (int c = 0; c < d; ++c) vv[c] = bf16_to_double(J->v[off + c]);
        }
    }
    free(tmp);
    return NULL;
}

int g4o_prefill_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                     const float* gamma_q, const float* gamma_k,
                     int B, int T, const g4o_cfg* cfg,
                     const int32_t* rows, int nrows, int nthreads,
                     double* out, double* lse) {
    if (!cfg_valid(cfg) || B < 0 || T < 0 || nrows < 0) return -1;
    if (cfg->kv_is_k == 0 && !v) return -1;
    if (B == 0 || nrows == 0) return 0;
    if (!q || !k || !rows || !out) return -1;
    int32_t rmax = -1;
    for (int r = 0; r < nrows; ++r) {
        if (rows[r] < 0 || rows[r] >= T) return -1;
        if (rows[r] > rmax) rmax = rows[r];
    }
    int d = cfg->head_dim, Hkv = cfg->n_kv_heads, G = cfg->n_q_heads / cfg->n_kv_heads;
    int R = g4o_rope_pairs(d, cfg->rope_p);
    int nt = online_cores(nthreads);
    double* gq = malloc(sizeof(double) * (size_t)d);
    double* gk = malloc(sizeof(double) * (size_t)d);
    for (int c = 0; c < d; ++c) {
        gq[c] = gamma_q ? (double)gamma_q[c] : 1.0;
        gk[c] = gamma_k ? (double)gamma_k[c] : 1.0;
    }
    size_t nkeys = (size_t)rmax + 1;
    double* khat = malloc(sizeof(double) * nkeys * d);
    double* krot = malloc(sizeof(double) * nkeys * d);
    double* vsep = cfg->kv_is_k == 0 ? malloc(sizeof(double) * nkeys * d) : NULL;
    pthread_t* th = malloc(sizeof(pthread_t) * (size_t)nt);
    if (!khat || !krot || (cfg->kv_is_k == 0 && !vsep)) {
        free(gq); free(gk); free(khat); free(krot); free(vsep); free(th);
        return -2;
    }
    for (int b = 0; b < B; ++b)
        for (int g = 0; g < Hkv; ++g) {
            keyprep_job KJ = {k, v, gk, cfg, T, b, g, R, Hkv, rmax, khat, krot, vsep, 0};
            for (int t = 0; t < nt; ++t) pthread_create(&th[t], NULL, keyprep_worker, &KJ);
            for (int t = 0; t < nt; ++t) pthread_join(th[t], NULL);
            const double* vals = cfg->kv_is_k == 1 ? khat : cfg->kv_is_k == 2 ? krot : vsep;
            prefill_job PJ = {q, gq, cfg, krot, vals, rows, nrows, B, T, b, g, G, R, out, lse, 0};
            for (int t = 0; t < nt; ++t) pthread_create(&th[t], NULL, prefill_worker, &PJ);
            for (int t = 0; t < nt; ++t) pthread_join(th[t], NULL);
        }
    free(gq); free(gk); free(khat); free(krot); free(vsep); free(th);
    return 0;
}

/* ------------------------------------------------------------------------------ */
/* Decode                                                                          */
/* ------------------------------------------------------------------------------ */
typedef struct {
    const uint16_t* q;
    const uint16_t* kc;
    const uint16_t* vc;
    const int8_t* kq;   /* int8 cache (kq != NULL): element = scale of its row * code */
    const float* ks;
    const int8_t* vq;
    const float* vs;
    const g4o_cfg* cfg;
    const int32_t* bg;  /* optional list of b * Hkv + g items; NULL = all */
    int nbg, B, L, R;
    double* out;
    double* lse;
    atomic_long next;
} decode_job;

/* Row (b, j, g) of the key (v = 0) or value (v = 1) cache, widened exactly to double: a bf16
 * element, or the row's fp32 scale times an int8 code. */
static void cache_row(const decode_job* J, int v, int b, int g, int64_t j, double* dst) {
    int d = J->cfg->head_dim, Hkv = J->cfg->n_kv_heads;
    size_t row = ((size_t)b * J->L + (size_t)j) * Hkv + g;
    size_t off = row * (size_t)d;
    if (J->kq) {
        const int8_t* code = v ? J->vq : J->kq;
        double sc = (double)(v ? J->vs : J->ks)[row];
        for (int c = 0; c < d; ++c) dst[c] = sc * (double)code[off + c];
    } else {
        const uint16_t* src = v ? J->vc : J->kc;
        for (int c = 0; c < d; ++c) dst[c] = bf16_to_double(src[off + c]);
    }
}

/* Key j of the cache, as the score side (rotated to position j) and the value side. */
static void decode_key(const decode_job* J, int b, int g, int64_t j, double* kh, double* kr) {
    const g4o_cfg* cfg = J->cfg;
    cache_row(J, 0, b, g, j, kh);
    g4o_rope(kh, cfg->head_dim, J->R, cfg->rope_base, j, kr);
}

static void* decode_worker(void* arg) {
    decode_job* J = (decode_job*)arg;
    const g4o_cfg* cfg = J->cfg;
    int d = cfg->head_dim, Hq = cfg->n_q_heads, Hkv = cfg->n_kv_heads, G = Hq / Hkv;
    size_t nk = J->L > 0 ? (size_t)J->L : 1;
    double* s = malloc(sizeof(double) * nk * (size_t)G);   /* scores [G, L] */
    double* qd = malloc(sizeof(double) * (size_t)d * G);
    double* kh = malloc(sizeof(double) * (size_t)d);
    double* kr = malloc(sizeof(double) * (size_t)d);
    double* m = malloc(sizeof(double) * (size_t)G);
    double* l = malloc(sizeof(double) * (size_t)G);
    long total = J->bg ? J->nbg : (long)J->B * Hkv;
    for (;;) {
        long it = atomic_fetch_add(&J->next, 1);
        if (it >= total) break;
        long item = J->bg ? J->bg[it] : it;
        int b = (int)(item / Hkv), g = (int)(item % Hkv);
        int64_t i = (int64_t)J->L - 1;   /* the new token sits at the last cache slot */
        int64_t lo = 0;
        if (cfg->window > 0 && i - cfg->window + 1 > 0) lo = i - cfg->window + 1;
        for (int hl = 0; hl < G; ++hl) {
            size_t qoff = ((size_t)b * Hq + g * G + hl) * (size_t)d;
            for (int c = 0; c < d; ++c) qd[(size_t)hl * d + c] = bf16_to_double(J->q[qoff + c]);
            m[hl] = -INFINITY;
            l[hl] = 0.0;
            double* o = J->out + qoff;
            for (int c = 0; c < d; ++c) o[c] = 0.0;
        }
        /* pass 1: all scores */
        for (int64_t j = lo; j <= i; ++j) {
            decode_key(J, b, g, j, kh, kr);
            for (int hl = 0; hl < G; ++hl) {
                double acc = 0.0;
                const double* qh = qd + (size_t)hl * d;
                for (int c = 0; c < d; ++c) acc += qh[c] * kr[c];
                double sv = cfg->scale * acc;
                s[(size_t)hl * nk + (size_t)(j - lo)] = sv;
                if (sv > m[hl]) m[hl] = sv;
            }
        }
        /* pass 2: softmax weights and the weighted sum of values */
        for (int hl = 0; hl < G; ++hl)
            for (int64_t j = lo; j <= i; ++j)
                l[hl] += exp(s[(size_t)hl * nk + (size_t)(j - lo)] - m[hl]);
        for (int64_t j = lo; j <= i; ++j) {
            decode_key(J, b, g, j, kh, kr);
            const double* vj = kh;
            if (cfg->kv_is_k == 2) vj = kr;
            if (cfg->kv_is_k == 0) {
                cache_row(J, 1, b, g, j, kr);
                vj = kr;
            }
            for (int hl = 0; hl < G; ++hl) {
                double w = exp(s[(size_t)hl * nk + (size_t)(j - lo)] - m[hl]) / l[hl];
                double* o = J->out + ((size_t)b * Hq + g * G + hl) * (size_t)d;
                for (int c = 0; c < d; ++c) o[c] += w * vj[c];
            }
        }
        if (J->lse)
            for (int hl = 0; hl < G; ++hl)
                J->lse[(size_t)b * Hq + g * G + hl] = i >= lo ? m[hl] + log(l[hl]) : -INFINITY;
    }
    free(s); free(qd); free(kh); free(kr); free(m); free(l);
    return NULL;
}

static int decode_run(decode_job* J, int nthreads) {
    int nt = online_cores(nthreads);
    int work = J->bg ? J->nbg : J->B * J->cfg->n_kv_heads;
    if (work == 0) return 0;
    if (nt > work) nt = work;
    pthread_t* th = malloc(sizeof(pthread_t) * (size_t)nt);
    for (int t = 0; t < nt; ++t) pthread_create(&th[t], NULL, decode_worker, J);
    for (int t = 0; t < nt; ++t) pthread_join(th[t], NULL);
    free(th);
    return 0;
}

static int check_items(const int32_t* bg, int nbg, int B, const g4o_cfg* cfg) {
    if (bg)
        for (int i = 0; i < nbg; ++i)
            if (bg[i] < 0 || bg[i] >= B * cfg->n_kv_heads) return -1;
    return 0;
}

int g4o_decode(const uint16_t* q, const uint16_t* kcache, const uint16_t* vcache,
               int B, int L, const g4o_cfg* cfg, const int32_t* bg, int nbg,
               int nthreads, double* out, double* lse) {
    if (!cfg_valid(cfg) || B < 0 || L < 0 || nbg < 0) return -1;
    if (cfg->kv_is_k == 0 && !vcache && L > 0) return -1;
    if (B == 0) return 0;
    if (!q || !out || (L > 0 && !kcache)) return -1;
    if (check_items(bg, nbg, B, cfg)) return -1;
    decode_job J = {q, kcache, vcache, NULL, NULL, NULL, NULL, cfg, bg, nbg, B, L,
                    g4o_rope_pairs(cfg->head_dim, cfg->rope_p), out, lse, 0};
    return decode_run(&J, nthreads);
}

int g4o_decode_int8(const uint16_t* q, const int8_t* kcodes, const float* kscales,
                    const int8_t* vcodes, const float* vscales, int B, int L,
                    const g4o_cfg* cfg, const int32_t* bg, int nbg, int nthreads,
                    double* out, double* lse) {
    if (!cfg_valid(cfg) || B < 0 || L < 0 || nbg < 0) return -1;
    if (cfg->kv_is_k == 0 && (!vcodes || !vscales) && L > 0) return -1;
    if (B == 0) return 0;
    if (!q || !out || (L > 0 && (!kcodes || !kscales))) return -1;
    if (check_items(bg, nbg, B, cfg)) return -1;
    decode_job J = {q, NULL, NULL, kcodes, kscales, vcodes, vscales, cfg, bg, nbg, B, L,
                    g4o_rope_pairs(cfg->head_dim, cfg->rope_p), out, lse, 0};
    return decode_run(&J, nthreads);
}

/*
 * g4attn_oracle.h -- plain fp64 CPU oracle for the Gemma-4-style attention layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference legs may load or call this library.  It shares no code,
 * header, table or constant with the CUDA library under attention_g4attn_b200/.
 *
 * What it computes (Gemma 4 Technical Report, section 2 "Model Architecture", and
 * the explainer pages "K=V" / "p-RoPE" sections that restate it):
 *   1. QKNorm: per-head RMSNorm of q and k over head_dim with a learned gain
 *        RMS(x; g)_c = x_c / sqrt(mean_c(x^2) + eps) * g_c
 *   2. RoPE / p-RoPE: pairs (x_i, x_{i+d/2}) for i < R = floor(p*d/2) rotate by
 *        phi = pos * base^(-2i/d); all other dims are left as they are.
 *   3. scores s_j = scale * rot(qhat, i) . rot(khat_j, j) for keys j visible to row i
 *        (causal: j <= i; sliding window W > 0: i - W < j <= i).
 *   4. values v_j = khat_j (kv_is_k = 1, "keys reused as values", pre-RoPE key),
 *        rot(khat_j, j) (kv_is_k = 2) or the supplied v (kv_is_k = 0).
 *   5. out_i = sum_j softmax(s)_j v_j,  lse_i = log sum_j exp(s_j).
 * Every floating-point step runs in IEEE double.  bf16 inputs are widened exactly.
 */
#ifndef G4ATTN_ORACLE_H
#define G4ATTN_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
    int n_q_heads;      /* Hq */
    int n_kv_heads;     /* Hkv; Hq % Hkv == 0, query head h reads kv head h / (Hq/Hkv) */
    int head_dim;       /* d, even */
    double rope_p;      /* fraction of rotary pairs that rotate; R = floor(p*d/2) */
    double rope_base;   /* RoPE base (theta) */
    int window;         /* 0 = full causal; W > 0 = keys i-W < j <= i */
    double scale;       /* softmax scale applied to q.k */
    int kv_is_k;        /* 0 separate v; 1 v = normed pre-RoPE k; 2 v = normed rotated k */
    int qk_norm;        /* 1 = apply QKNorm to q and k, 0 = use them as given */
    double qk_norm_eps; /* epsilon inside the RMS */
} g4o_cfg;

/* Number of rotated pairs R = floor(p * d / 2). */
int g4o_rope_pairs(int head_dim, double rope_p);

/* RMSNorm of one vector of length d (gamma may be NULL = all ones). */
void g4o_rmsnorm(const double* x, const double* gamma, int d, double eps, double* y);

/* Rotate the first R pairs (i, i + d/2) of x by pos * base^(-2i/d). y may alias x. */
void g4o_rope(const double* x, int d, int R, double base, int64_t pos, double* y);

/* Per-row normalisation + rotation, the standalone prologue.
 *   q_in  [B, T, Hq, d]  bf16 bits;  k_in [B, T, Hkv, d] bf16 bits (either may be NULL)
 *   q_out [B, T, Hq, d]  = rot(RMS(q), pos0 + t)
 *   k_out [B, T, Hkv, d] = RMS(k)               (pre-RoPE, the K(=V) cache)
 *   krot_out [B, T, Hkv, d] = rot(RMS(k), pos0 + t)   (may be NULL)                  */
int g4o_qknorm_rope(const uint16_t* q_in, const uint16_t* k_in,
                    const float* gamma_q, const float* gamma_k,
                    int B, int T, int64_t pos0, const g4o_cfg* cfg,
                    double* q_out, double* k_out, double* krot_out);

/* Prefill attention for a set of query rows.
 *   q [B, T, Hq, d], k [B, T, Hkv, d], v [B, T, Hkv, d] or NULL: bf16 bits, raw (pre-norm)
 *   rows[nrows]: query positions i in [0, T) evaluated for every b and every head
 *   out [B, nrows, Hq, d] doubles; lse [B, Hq, nrows] doubles (may be NULL)
 * Returns 0, or -1 on an invalid argument.  nthreads <= 0 uses every online core. */
int g4o_prefill_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                     const float* gamma_q, const float* gamma_k,
                     int B, int T, const g4o_cfg* cfg,
                     const int32_t* rows, int nrows, int nthreads,
                     double* out, double* lse);

/* Decode: one query per (b, h) at position L-1 against a cache that already holds
 * the normalised keys.
 *   q [B, Hq, d] bf16 bits, already normalised and rotated to position L-1
 *   kcache [B, L, Hkv, d] bf16 bits: normalised pre-RoPE keys (rotation applied here)
 *   vcache [B, L, Hkv, d] or NULL (kv_is_k = 0 requires it)
 *   bg[nbg]: optional list of items b * Hkv + g to evaluate (NULL = every item);
 *            rows of out/lse for other items are left untouched
 *   out [B, Hq, d]; lse [B, Hq] (may be NULL)                                        */
int g4o_decode(const uint16_t* q, const uint16_t* kcache, const uint16_t* vcache,
               int B, int L, const g4o_cfg* cfg, const int32_t* bg, int nbg,
               int nthreads, double* out, double* lse);

/* Decode against an int8 cache (the same operation as g4o_decode): element c of row (b, j, g)
 * is scales[(b * L + j) * Hkv + g] * codes[((b * L + j) * Hkv + g) * d + c], exact in double.
 * vcodes / vscales are the separate values (kv_is_k = 0), else NULL. */
int g4o_decode_int8(const uint16_t* q, const int8_t* kcodes, const float* kscales,
                    const int8_t* vcodes, const float* vscales, int B, int L,
                    const g4o_cfg* cfg, const int32_t* bg, int nbg, int nthreads,
                    double* out, double* lse);

#ifdef __cplusplus
}
#endif
#endif

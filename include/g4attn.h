/*
 * g4attn.h -- C ABI of the g4attn library: the Gemma-4-style attention layer as
 * hand-written sm_100a (B200) CUDA kernels.
 *
 * The operation (Gemma 4 Technical Report, section 2 "Model Architecture"; the
 * yunpan.plus explainer sections "GQA", "K=V", "p-RoPE" and "interleaved layers";
 * the AI Engineer talk notes on GQA 2:1 / 8:1 and head_dim 256 -> 512):
 *   QKNorm   q^ = RMS(q; gamma_q), k^ = RMS(k; gamma_k)  over head_dim, with
 *            RMS(x; g)_c = x_c / sqrt(mean(x^2) + eps) * g_c
 *   p-RoPE   pairs (x_i, x_{i+d/2}), i < R = floor(p*d/2), turn by pos * base^(-2i/d)
 *            ((cos -sin; sin cos)); the other pairs do not turn.  Global layers:
 *            p = 0.25, base 1e6; local layers: p = 1, base 1e4.
 *   GQA      query head h reads kv head h / (Hq/Hkv).
 *   scores   s_ij = scale * rot(q^_i, i) . rot(k^_j, j) for j visible to i: causal
 *            (window = 0: j <= i) or sliding window (window = W: i - W < j <= i).
 *   values   kv_is_k = 1: v_j = k^_j (keys reused as values, the pre-RoPE normed key);
 *            kv_is_k = 2: v_j = rot(k^_j, j); kv_is_k = 0: the supplied v_j.
 *   output   out_i = sum_j softmax_j(s_ij) v_j;   lse_i = log sum_j exp(s_ij).
 *
 * Conventions for every entry point:
 *   - Tensors are row-major, contiguous, [B, T, H, d] with d fastest, in device
 *     memory.  bf16 tensors hold IEEE bfloat16 bit patterns.  Device pointers must be
 *     16-byte aligned (G4ATTN_ERR_MISALIGNED otherwise).
 *   - The caller owns every buffer.  The library never allocates device memory on
 *     these paths; it keeps a small host-side cache only (kernel attributes).
 *   - Calls are asynchronous and ordered on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream).  Arguments are validated before any launch; on an error
 *     nothing is launched.
 *   - The current CUDA device must be an sm_100 part (G4ATTN_ERR_UNSUPPORTED otherwise).
 *   - Return value: G4ATTN_OK or one of the negative codes below.
 */
#ifndef G4ATTN_H
#define G4ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define G4ATTN_API __attribute__((visibility("default")))
#else
#define G4ATTN_API
#endif

typedef uint16_t g4attn_bf16;          /* IEEE bfloat16 bit pattern */
typedef struct CUstream_st* g4attn_stream_t;  /* same type as cudaStream_t */

enum {
    G4ATTN_OK = 0,
    G4ATTN_ERR_INVALID_ARG = -1,   /* null pointer, bad size, inconsistent config */
    G4ATTN_ERR_UNSUPPORTED = -2,   /* head_dim / group / device not handled by the kernels */
    G4ATTN_ERR_MISALIGNED = -3,    /* a pointer is not 16-byte aligned */
    G4ATTN_ERR_WORKSPACE = -4,     /* workspace missing or smaller than *_workspace_size */
    G4ATTN_ERR_CUDA = -5,          /* a CUDA runtime / driver call or launch failed */
    G4ATTN_ERR_TIMEOUT = -6,       /* a device wait gave up (see g4attn_device_status) */
    G4ATTN_ERR_TOO_LARGE = -7      /* g4attn_decode_noalloc: partials exceed its fixed scratch */
};

/* Layer configuration (one attention layer). */
typedef struct g4attn_layer_cfg {
    int n_q_heads;      /* Hq > 0 */
    int n_kv_heads;     /* Hkv > 0, Hq % Hkv == 0; G = Hq / Hkv must divide 128 */
    int head_dim;       /* d: 256 or 512 for the tensor-core kernels */
    float rope_p;       /* fraction of rotary pairs that turn, 0 <= p <= 1 (0.25 global, 1 local) */
    double rope_base;   /* RoPE base > 0 (1e6 global, 1e4 local) */
    int window;         /* 0 = full causal; W > 0 = sliding window i - W < j <= i */
    float scale;        /* softmax scale > 0 (1/sqrt(d) for the pages' layers) */
    int kv_is_k;        /* 0 separate v; 1 v = normed pre-RoPE key; 2 v = normed rotated key */
    int qk_norm;        /* 1 = apply QKNorm (the layers on the pages), 0 = inputs are used as is */
    float qk_norm_eps;  /* eps inside the RMS (1e-6) */
} g4attn_layer_cfg;

/*
 * Standalone prologue: QKNorm and p-RoPE of one block of tokens at positions
 * pos0 .. pos0+T-1 (report section 2: QKNorm, p-RoPE / RoPE; explainer "K=V": the
 * cache of a global layer holds keys only).
 *   q_in       [B, T, Hq, d] bf16, or NULL (then q_out is ignored)
 *   k_in       [B, T, Hkv, d] bf16, or NULL (then kcache_out / krot_out are ignored)
 *   q_out      [B, T, Hq, d] bf16: rot(RMS(q), pos)            (NULL = not written)
 *   kcache_out [B, T, Hkv, d] bf16: RMS(k), not rotated: the K(=V) cache rows
 *   krot_out   [B, T, Hkv, d] bf16: rot(RMS(k), pos)           (NULL = not written)
 *   gamma_q / gamma_k  [d] fp32 device arrays (required when cfg->qk_norm = 1)
 * Writes only.  With qk_norm = 0 the norm step is skipped (pure RoPE).
 */
G4ATTN_API int g4attn_qknorm_rope(const g4attn_bf16* q_in, const g4attn_bf16* k_in,
                       g4attn_bf16* q_out, g4attn_bf16* kcache_out, g4attn_bf16* krot_out,
                       const float* gamma_q, const float* gamma_k,
                       int B, int T, long long pos0,
                       const g4attn_layer_cfg* cfg, g4attn_stream_t stream);

/*
 * Bytes of device workspace g4attn_prefill needs for (B, T, cfg): the normalised key
 * cache and its rotated copy.  Returns 0 when the configuration is invalid.
 */
G4ATTN_API size_t g4attn_prefill_workspace_size(int B, int T, const g4attn_layer_cfg* cfg);

/*
 * Prefill: causal or sliding-window attention of T new tokens at positions 0..T-1
 * over themselves (report section 2; explainer "interleaved layers", "K=V", "p-RoPE").
 *   q      [B, T, Hq, d] bf16, raw (QKNorm and RoPE are applied inside, fused into
 *          the query tile load)
 *   k      [B, T, Hkv, d] bf16, raw
 *   v      [B, T, Hkv, d] bf16 raw values; must be NULL when kv_is_k != 0 and
 *          non-NULL when kv_is_k == 0
 *   gamma_q, gamma_k  [d] fp32
 *   out    [B, T, Hq, d] bf16 (written)
 *   lse    [B, Hq, T] fp32 natural-log sum of exp of the scaled scores, or NULL
 *   workspace / ws_bytes  >= g4attn_prefill_workspace_size(B, T, cfg), 256-byte aligned
 * T = 0 or B = 0 is a no-op.  window >= T behaves as full causal attention.
 */
G4ATTN_API int g4attn_prefill(const g4attn_bf16* q, const g4attn_bf16* k, const g4attn_bf16* v,
                   const float* gamma_q, const float* gamma_k,
                   g4attn_bf16* out, float* lse, void* workspace, size_t ws_bytes,
                   int B, int T, const g4attn_layer_cfg* cfg, g4attn_stream_t stream);

/*
 * Chunked prefill (the serving form of the prefill in report section 2: a long prompt goes
 * through in chunks, each against the cache the earlier chunks left): Tn new tokens at
 * positions P .. P+Tn-1 attend causally, and within the window W = cfg->window on
 * sliding-window layers, to the P earlier positions held in the cache and to the chunk
 * itself.  The chunk's normalised keys (and its raw values) are then in the cache, so the
 * next chunk, or g4attn_decode, continues from position P + Tn.
 *   q, k, v   the chunk's raw queries [B, Tn, Hq, d], keys and values [B, Tn, Hkv, d]
 *             (v as in g4attn_prefill: non-NULL exactly when kv_is_k == 0)
 *   kcache    [B, cache_rows, Hkv, d] bf16: normalised keys, NOT rotated (the layout
 *             g4attn_decode reads) or, with G4ATTN_CACHE_ROTATED, turned to their positions
 *             (the layout g4attn_decode_rotated reads).  Read: positions max(0, P-W+1) ..
 *             P-1 (all P on causal layers).  Written: positions P .. P+Tn-1 (RMS(k) *
 *             gamma_k, turned when ROTATED, rounded to bf16)
 *   vcache    [B, cache_rows, Hkv, d] bf16 separate values (kv_is_k == 0), else NULL;
 *             same rows read and written, the chunk's v copied unchanged
 *   cache_flags  0 or a combination of
 *             G4ATTN_CACHE_RING: position p in row p % cache_rows (window layers with
 *               0 < W <= cache_rows; of a chunk longer than the ring only its last
 *               cache_rows positions are written); without it position p is in row p and
 *               cache_rows >= P + Tn
 *             G4ATTN_CACHE_ROTATED: the keys are stored turned (separate-value layers only,
 *               kv_is_k == 0: a keys-as-values cache must hold the unrotated keys, which
 *               are its values)
 *   out       [B, Tn, Hq, d] bf16 (written);  lse [B, Hq, Tn] fp32 or NULL
 *   workspace / ws_bytes  >= g4attn_prefill_chunk_workspace_size(B, P, Tn, cfg),
 *             256-byte aligned (fp16 key rows of the visible positions, their (cos, sin)
 *             table, and a copy of the visible values when kv_is_k == 0)
 * P = 0 is g4attn_prefill plus the cache write.  B = 0 or Tn = 0 is a no-op (nothing is
 * written).  Arguments out of range return G4ATTN_ERR_INVALID_ARG before any launch.
 * The cache must not overlap q, k, v, out or the workspace.
 */
G4ATTN_API size_t g4attn_prefill_chunk_workspace_size(int B, int P, int Tn,
                                                      const g4attn_layer_cfg* cfg);
#define G4ATTN_CACHE_RING 1
#define G4ATTN_CACHE_ROTATED 2
G4ATTN_API int g4attn_prefill_chunk(const g4attn_bf16* q, const g4attn_bf16* k,
                                    const g4attn_bf16* v, const float* gamma_q,
                                    const float* gamma_k, g4attn_bf16* kcache,
                                    g4attn_bf16* vcache, int cache_rows, int cache_flags,
                                    g4attn_bf16* out, float* lse, void* workspace,
                                    size_t ws_bytes, int B, int P, int Tn,
                                    const g4attn_layer_cfg* cfg, g4attn_stream_t stream);

/*
 * Bytes of device workspace g4attn_decode needs for (B, L, cfg): fp32 partial outputs
 * and softmax statistics of the split-KV pass.  Returns 0 for an invalid configuration.
 */
G4ATTN_API size_t g4attn_decode_workspace_size(int B, int L, const g4attn_layer_cfg* cfg);

/*
 * Decode: one new token per sequence, at position L-1, against a cache of L keys that
 * already includes it (explainer "K=V": the global layer keeps a single K cache).
 *   q       [B, 1, Hq, d] bf16: the new queries, already normalised and rotated to
 *           position L-1 (g4attn_qknorm_rope with pos0 = L-1 produces it)
 *   kcache  [B, L, Hkv, d] bf16: normalised, NOT rotated keys; the kernel turns key j
 *           to position j on the fly
 *   vcache  [B, L, Hkv, d] bf16 or NULL: separate values (kv_is_k = 0 only)
 *   out     [B, 1, Hq, d] bf16 (written);  lse [B, Hq] fp32 or NULL
 *   workspace / ws_bytes  >= g4attn_decode_workspace_size(B, L, cfg), 256-byte aligned
 * With window W > 0 only the last W cache rows are read.  L = 0 writes out = 0 and
 * lse = -inf.
 */
G4ATTN_API int g4attn_decode(const g4attn_bf16* q, const g4attn_bf16* kcache, const g4attn_bf16* vcache,
                  int L, g4attn_bf16* out, float* lse, void* workspace, size_t ws_bytes,
                  int B, const g4attn_layer_cfg* cfg, g4attn_stream_t stream);

/*
 * Decode of a sliding-window layer against a ring-buffer cache (report section 2 and the
 * explainer's "interleaved layers": local layers attend to the last W tokens, so their cache
 * only needs the last C >= W positions).  Same operation as g4attn_decode with window W =
 * cfg->window, but the cache holds position p in row p % C:
 *   kring   [B, C, Hkv, d] bf16: normalised, NOT rotated keys; row p % C holds position p
 *           for the last C positions p < L
 *   vring   [B, C, Hkv, d] bf16 or NULL: separate values, same ring (kv_is_k = 0 only)
 *   L       tokens so far; the new query sits at position L-1
 *   C       ring rows: a positive multiple of 64, with 0 < W = cfg->window <= C
 *   workspace / ws_bytes  >= g4attn_decode_ring_workspace_size(B, L, C, cfg)
 * Other arguments and results as in g4attn_decode.  C or W out of range returns
 * G4ATTN_ERR_INVALID_ARG before any launch (and the workspace size function returns 0).
 */
G4ATTN_API size_t g4attn_decode_ring_workspace_size(int B, int L, int C,
                                                    const g4attn_layer_cfg* cfg);
G4ATTN_API int g4attn_decode_ring(const g4attn_bf16* q, const g4attn_bf16* kring,
                                  const g4attn_bf16* vring, int L, int C, g4attn_bf16* out,
                                  float* lse, void* workspace, size_t ws_bytes, int B,
                                  const g4attn_layer_cfg* cfg, g4attn_stream_t stream);

/*
 * Decode against the split cache layout of a keys-as-values layer with R = 64 rotated pairs
 * (the global layers' p-RoPE: head_dim 512, p = 0.25): the keys are stored already rotated
 * to their positions, plus a side copy of the pre-RoPE values of the 2R = 128 rotated dims:
 * 1.25 * d elements per key instead of 2 * d for separate rotated keys and values, 37.5%
 * less (the global-layer cache saving the Gemma 4 report quotes).  No key is turned on the
 * fly; the values are the pre-RoPE keys as in g4attn_decode with kv_is_k = 1.
 *   krot    [B, L, Hkv, d] bf16: normalised keys, rotated to their positions
 *   vside   [B, L, Hkv, 128] bf16: the same keys' pre-RoPE dims [0, 64) then [d/2, d/2 + 64)
 *   workspace / ws_bytes  >= g4attn_decode_workspace_size(B, L, cfg)
 * Other arguments and results as in g4attn_decode.  Needs kv_is_k = 1 and R = 64
 * (G4ATTN_ERR_UNSUPPORTED otherwise).
 */
G4ATTN_API int g4attn_decode_split_cache(const g4attn_bf16* q, const g4attn_bf16* krot,
                                         const g4attn_bf16* vside, int L, g4attn_bf16* out,
                                         float* lse, void* workspace, size_t ws_bytes, int B,
                                         const g4attn_layer_cfg* cfg, g4attn_stream_t stream);

/*
 * Decode of a separate-value layer against a cache of keys stored turned to their positions
 * (the local layers' cache: their values are a tensor of their own, so nothing needs the
 * unrotated key).  Same operation as g4attn_decode (C = 0) or g4attn_decode_ring (C > 0),
 * but no key is turned on the fly:
 *   krot    [B, L or C, Hkv, d] bf16: normalised keys, key of position p turned to angle p
 *           (g4attn_qknorm_rope's krot_out, or g4attn_prefill_chunk with
 *           G4ATTN_CACHE_ROTATED); linear (row p) when C == 0, ring (row p % C) when C > 0
 *   vcache  [B, L or C, Hkv, d] bf16 values, same rows
 *   C       0, or the ring's rows under the rules of g4attn_decode_ring
 *   workspace / ws_bytes  >= g4attn_decode_rotated_workspace_size(B, L, C, cfg)
 * Other arguments and results as in g4attn_decode.  kv_is_k != 0 returns
 * G4ATTN_ERR_UNSUPPORTED.
 */
G4ATTN_API size_t g4attn_decode_rotated_workspace_size(int B, int L, int C,
                                                       const g4attn_layer_cfg* cfg);
G4ATTN_API int g4attn_decode_rotated(const g4attn_bf16* q, const g4attn_bf16* krot,
                                     const g4attn_bf16* vcache, int L, int C, g4attn_bf16* out,
                                     float* lse, void* workspace, size_t ws_bytes, int B,
                                     const g4attn_layer_cfg* cfg, g4attn_stream_t stream);

/*
 * int8 KV cache writer.  The Gemma 4 report's memory table counts the KV cache in int8; the
 * scheme is not on the pages, and the one built here is symmetric with one fp32 scale per row
 * (a position of one kv head):
 *   scale = max_c |x_c| / 127,  code_c = round-half-even(x_c / scale) clamped to [-127, 127],
 * both divisions IEEE fp32 rounded to nearest; a row of zeros has scale 0 and codes 0.  The
 * element the cache stands for is scale * code.  Inputs are expected finite (normalised keys
 * are); a row holding an infinity or a NaN is written with scale NaN and codes 0, so each of
 * its elements reads back as NaN.
 *   x       [rows, d] bf16 (e.g. a [B, L, Hkv, d] cache: rows = B * L * Hkv), 16-byte aligned
 *   codes   [rows, d] int8 (written), 16-byte aligned
 *   scales  [rows] fp32 (written)
 *   d       128, 256 or 512
 * rows = 0 is a no-op; a bad d or null pointer returns G4ATTN_ERR_INVALID_ARG.
 */
G4ATTN_API int g4attn_quantize_int8(const g4attn_bf16* x, int8_t* codes, float* scales,
                                    long long rows, int d, g4attn_stream_t stream);

/*
 * Decode against an int8 KV cache (the Gemma 4 report's memory table counts the KV cache in
 * int8: papers.ananclaw.com explainer, section on long context and memory).  The cache is
 * the one g4attn_quantize_int8 writes: codes [rows, d] int8 and one fp32 scale per row (a
 * position of one kv head), each element standing for scale * code.  Same operation as
 * g4attn_decode (C = 0) or g4attn_decode_ring (C > 0) on that cache:
 *   q        [B, 1, Hq, d] bf16: the new queries, normalised and rotated to position L-1
 *   kcodes   [B, L or C, Hkv, d] int8 and kscales [B, L or C, Hkv] fp32: normalised keys, NOT
 *            rotated (turned on the fly, as in g4attn_decode)
 *   vcodes / vscales  the same layout for separate values (kv_is_k == 0), else both NULL
 *   C        0 (linear cache, row = position) or the ring's rows under g4attn_decode_ring's
 *            rules (row = position % C)
 *   out, lse as in g4attn_decode
 *   workspace / ws_bytes  >= g4attn_decode_int8_workspace_size(B, L, C, cfg), 256-byte aligned
 * The query stays bf16; the codes are widened to bf16 inside the kernel (exact), each key's
 * scale multiplies its score and each value's scale its softmax weight.  kv_is_k 0, 1 and 2
 * are served; at most 8 query heads per kv head (G4ATTN_ERR_UNSUPPORTED otherwise).  codes
 * must be 16-byte aligned, scales 4-byte aligned.  L = 0 writes out = 0 and lse = -inf.
 */
G4ATTN_API size_t g4attn_decode_int8_workspace_size(int B, int L, int C,
                                                    const g4attn_layer_cfg* cfg);
G4ATTN_API int g4attn_decode_int8(const g4attn_bf16* q, const int8_t* kcodes,
                                  const float* kscales, const int8_t* vcodes,
                                  const float* vscales, int L, int C, g4attn_bf16* out,
                                  float* lse, void* workspace, size_t ws_bytes, int B,
                                  const g4attn_layer_cfg* cfg, g4attn_stream_t stream);

/*
 * Decode without a workspace and without allocating (the papers describe no such call;
 * it exists for callers that cannot allocate device memory: plugins whose host framework
 * owns every device allocation and hands them only input and output buffers, and services
 * that reserve the whole device up front).  Same operation, arguments and layouts as
 * g4attn_decode minus the workspace: the split-KV partials live in a fixed 8 MiB device
 * array inside the library, which every device that loads the library holds until the
 * process exits.  The call allocates nothing.
 *   - The call keeps the largest number of CTA pairs (and with it of segments each sequence
 *     is split into) whose partials fit; if even one segment per sequence needs more than
 *     8 MiB (2 * B * Hq * (head_dim + 2) * 4 bytes > 8 MiB: the kernel keeps two partials
 *     per segment), the call returns G4ATTN_ERR_TOO_LARGE and launches nothing.
 *   - The array's device address is looked up at set-up: by the first g4attn call on a
 *     device (any entry point), with that device current, and again if the device's CUDA
 *     context changes (after cudaDeviceReset).  Make that first call before any stream
 *     capture.
 *   - All calls share the one array and it keeps the last call's partials.  Nothing in it
 *     needs to start at zero (every partial is written before it is read), but calls that
 *     overlap on the GPU (different streams, or several host threads) race on it: order
 *     them on one stream or synchronise between them.
 */
G4ATTN_API int g4attn_decode_noalloc(const g4attn_bf16* q, const g4attn_bf16* kcache,
                                     const g4attn_bf16* vcache, int L, g4attn_bf16* out,
                                     float* lse, int B, const g4attn_layer_cfg* cfg,
                                     g4attn_stream_t stream);

/* Human-readable name of a status code (static storage). */
G4ATTN_API const char* g4attn_status_string(int status);

/*
 * Device-side status word.  Every bounded wait inside the kernels (mbarrier spins)
 * gives up after the current wait limit, records G4ATTN_ERR_TIMEOUT here and lets the
 * kernel finish early.  g4attn_device_status synchronises `stream`, returns the word
 * (G4ATTN_OK if no wait gave up since the last reset) and clears it.
 */
G4ATTN_API int g4attn_device_status(g4attn_stream_t stream);

/*
 * Upper bound on the polls of one device wait.  Independently of it, every wait gives
 * up after 2 seconds of wall-clock time (legal waits last microseconds).  The default
 * poll bound is effectively unlimited; tests of the timeout path set a small one.
 * Values < 1 restore the default.  Returns the previous bound.
 */
G4ATTN_API long long g4attn_set_wait_limit(long long polls);

/*
 * Self-test of failure detection.  Launches one CTA on `stream` whose thread waits, with the
 * kernels' bounded wait and at most `polls` polls (polls < 1: the current wait limit), on
 * an mbarrier that nothing arrives on.  The wait gives up and records G4ATTN_ERR_TIMEOUT in
 * the device status word, which g4attn_device_status(stream) then returns (and clears).
 * The CTA holds no copies, MMAs or tensor memory, so the context stays usable.
 * Returns G4ATTN_OK once launched, G4ATTN_ERR_UNSUPPORTED without an sm_100 device,
 * G4ATTN_ERR_CUDA if the launch fails.
 */
G4ATTN_API int g4attn_wait_selftest(long long polls, g4attn_stream_t stream);

/* Library version string. */
G4ATTN_API const char* g4attn_version(void);

#ifdef __cplusplus
}
#endif
#endif /* G4ATTN_H */

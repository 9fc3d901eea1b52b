// kernels.h -- launcher interfaces between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "g4attn.h"

namespace g4 {

// RoPE geometry of a layer: R rotated pairs (i, i + d/2), i < R.
struct Rope {
    int R;
    double log2_base;   // log2(rope_base)
};

struct QkNormRopeArgs {
    const uint16_t* q_in;
    const uint16_t* k_in;
    uint16_t* q_out;
    uint16_t* k_out;      // normalised, not rotated
    uint16_t* krot_out;   // normalised and rotated
    const float* gamma_q;
    const float* gamma_k;
    float2* cs_out;       // optional [T, R] (cos, sin) table of positions pos0 + t
    int k_f16;            // 1: k_out / krot_out are written as fp16 instead of bf16
    int B, T, Hq, Hkv, d;
    long long pos0;
    // Row placement (all default to the dense [B, T, H, d] layout when zero).  Token t of
    // batch b sits at position p = pos0 + t.
    //  inputs  (q_in, k_in, v_in):  row b * in_rows + (in_ring ? p % in_ring : p - in_base)
    //  outputs (q_out, k_out, krot_out, v_out, cs_out): row b * out_rows + p - out_base
    //  cache copies (kc_out, vc_out): row b * kc_rows + (kc_ring ? p % kc_ring : p); with a
    //  ring only the last kc_ring tokens are written (earlier ones would be overwritten)
    int in_rows, in_ring;
    long long in_base;
    int out_rows;
    long long out_base;
    const uint16_t* v_in;  // optional values, copied unchanged to v_out / vc_out
    uint16_t* v_out;
    uint16_t* kc_out;      // optional bf16 copy of the normalised keys: unrotated, or
    uint16_t* vc_out;      // turned to their positions when kc_rot is set
    int kc_rows, kc_ring;
    int kc_rot;
    Rope rope;
    int qk_norm;
    float eps;
};

cudaError_t launch_qknorm_rope(const QkNormRopeArgs& a, cudaStream_t stream);

// Self-test of the bounded waits: a wait that nothing satisfies gives up after `limit` polls
// (or 2 s) and records G4ATTN_ERR_TIMEOUT in *status.
cudaError_t launch_wait_selftest(int* status, long long limit, cudaStream_t stream);

// Split-KV decode (one query per (b, h) at position L-1) and its combine pass.
struct DecodeArgs {
    CUtensorMap tm_k;       // kcache [B, L or C, Hkv, d] as a 4-D map (d, Hkv, rows, B), box (64, 1, 64, 1)
    CUtensorMap tm_v;       // vcache, same geometry (kv_is_k == 0), else a copy of tm_k
    // split cache (split_cache = 1): tm_k holds keys rotated to their positions, tm_vside the
    // pre-RoPE values of the 2R = 128 rotated dims [B, L, Hkv, 128] (the value operand of
    // slot 0; the other slots' dims are the same rotated or not); no key is turned
    CUtensorMap tm_vside;
    int split_cache;
    // int8 cache (int8 = 1): tm_k / tm_v map the int8 codes [B, L or C, Hkv, d] as (d, Hkv,
    // rows, B) with box (64, 1, 64, 1) and 64-byte swizzle; element = scale of its row * code,
    // the scales fp32 [B, L or C, Hkv] (kscale; vscale for separate values)
    int int8;
    const float* kscale;
    const float* vscale;
    const uint16_t* q;      // [B, Hq, d], normalised and rotated
    float* part_o;          // [2S, B, Hq, d]
    float* part_ml;         // [2S, B, Hq, 2]  (running max in log2 units, sum)
    uint16_t* out;          // [B, Hq, d]
    float* lse;             // [B, Hq] or null
    int B, L, Hq, Hkv, d, G;
    int key_lo;             // first visible key position (window), 0 for full attention
    int tile_base;          // position where the pair-tiles start (<= key_lo)
    int ring;               // 0: cache row = position; C > 0: ring of C rows, row = position % C
    // Stream-K split: the B * Hkv sequences' pair-tiles of 128 keys, tiles_per_seq each,
    // are one flat range of total_tiles; CTA pair p takes tiles
    // [p * total_tiles / n_pairs, (p + 1) * total_tiles / n_pairs), so a sequence is cut
    // into segments, one per pair that touches it (at most `splits`).  part_o / part_ml
    // hold two partials per segment (one per CTA of the pair): index 2 * segment + rank.
    int splits;
    int tiles_per_seq, n_pairs;
    long long total_tiles;
    Rope rope;
    float scale_log2;       // scale * log2(e)
    int kv_is_k;
    long long wait_limit;
    int* status;
};

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream);
// Fixed device scratch of g4attn_decode_noalloc (defined in decode.cu).
size_t decode_scratch_bytes();
cudaError_t decode_scratch_ptr(void** out);

// Flash-attention prefill.
struct PrefillArgs {
    // 4-D maps over [B, Tk, Hkv, d] as (d, Hkv, Tk, B), 128-byte swizzle.  The *_s maps load
    // 64 dims x 64 keys (the score operand, half a key tile per CTA of a pair); the *_v
    // maps load 64 dims x 128 keys (the value operand).
    CUtensorMap tm_kn_s;    // normalised pre-RoPE keys (fp16)
    CUtensorMap tm_kr_s;    // normalised rotated keys (fp16)
    CUtensorMap tm_kn_v;
    CUtensorMap tm_kr_v;
    CUtensorMap tm_v;       // separate values (bf16, kv_is_k == 0), else a copy of tm_kn_v
    CUtensorMap tm_q;       // raw queries as (d, Hq, T, B), box (64, G, 128 / G, 1): one row tile
    CUtensorMap tm_cs;      // rope_cs as fp32 (2R, Tk), box (2R, 128 / G); valid when cs_tma
    int cs_tma;             // the (cos, sin) rows of a row tile are loaded by TMA
    const uint16_t* q;      // raw queries [B, T, Hq, d]
    const float* gamma_q;
    const float2* rope_cs;  // [Tk, R] (cos, sin) of the position of key row t, pair i
    uint16_t* out;          // [B, T, Hq, d]
    float* lse;             // [B, Hq, T] or null
    int B, T, Hq, Hkv, d, G;
    int Tk;      // key rows per batch in the key maps and the (cos, sin) table
    int q_off;   // key row of the position of query token 0 (q_off + T <= Tk)
    int window;
    Rope rope;
    int qk_norm;
    float eps;
    float scale_log2;
    int kv_is_k;
    long long wait_limit;
    int* status;
};

cudaError_t launch_prefill(const PrefillArgs& a, cudaStream_t stream);
size_t prefill_smem_bytes(int d);
size_t prefill_cs_stage_bytes(int d);   // room for the (cos, sin) rows staged in the prologue

}  // namespace g4

// prefill.cu -- flash-attention prefill for the Gemma-4-style layer on tcgen05 / TMEM.
//
// One CTA computes one 128-row tile of packed query rows: row r is token m0 + r / G of
// query head g*G + r % G, i.e. the G query heads that share kv head g sit in the MMA M
// dimension (GQA; explainer "GQA": 8:1 in global layers, 2:1 in local layers).
//   prologue  raw q rows -> RMSNorm * gamma -> RoPE / p-RoPE -> fp16, 128-byte-swizzled
//             K-major tile in shared memory (report section 2: QKNorm, p-RoPE)
//   The normalised key copies written by the key pre-pass are fp16 too: QKNorm bounds
//   their range, and fp16 keeps 3 more mantissa bits than bf16 for the values that
//   keys-as-values layers feed straight into the output.
//   per key tile of 128 keys (causal / sliding-window tiles outside the band are skipped):
//     S  = Q K^T        tcgen05.mma M=128 N=128, fp32 in TMEM, K streamed in 64-dim chunks
//                       (rotated chunks from the rotated key copy, the rest from the
//                       normalised pre-RoPE keys)
//     softmax           thread = row: masked row max (lazy: the reference max only moves
//                       when the tile max exceeds it by more than 2^8), P = exp2 rounded to
//                       the format of V into shared memory, running sum of the rounded P
//     O += P V          tcgen05.mma M=128 N=256, V read MN-major from the same 64-dim
//                       chunk layout; V is the pre-RoPE normalised key (keys reused as
//                       values), the rotated key, or the separate values
//   epilogue  O / l -> bf16 rows; lse = m + log2(l) (natural log on output)
// head_dim 512: the 128 x 512 fp32 O accumulator fills all 512 TMEM columns, so the S
// tile borrows columns [128, 256): the softmax warps hold that quarter of O in registers
// while S lives there and put it back before the PV product.
//
// Warp roles (192 threads): warp 0 TMA producer, warp 1 MMA issuer + TMEM owner,
// warps 2..5 prologue / softmax / correction / epilogue.  Every wait is bounded.
#include <cuda_bf16.h>

#include "kernels.h"
#include "sm100.cuh"

namespace g4 {
namespace {

constexpr int kThreads = 192;
constexpr int kBM = 128;               // packed query rows per CTA
constexpr int kBN = 128;               // keys per tile
constexpr int kChunkBytes = 16384;     // 128 keys x 64 dims bf16, 128-byte swizzle
constexpr uint32_t kTmemCols = 512;
constexpr int kBarWG = 1;
constexpr float kLazyMax = 8.0f;       // log2 units

template <int D>
struct PrefillCfg {
    static constexpr int NCH = D / 64;
    static constexpr bool SWAP = (D == 512);
    static constexpr int NSLOT = (D == 512) ? 4 : 8;
    static constexpr uint32_t S_COL = (D == 512) ? 128 : 256;
};

template <int D>
struct __align__(1024) PrefillSmem {
    uint8_t q[PrefillCfg<D>::NCH][kChunkBytes];    // 128 rows x 64 dims per chunk
    uint8_t p[2][kChunkBytes];                     // P: 128 rows x 64 keys per chunk
    uint8_t ring[PrefillCfg<D>::NSLOT][kChunkBytes];
    uint64_t full[PrefillCfg<D>::NSLOT];
    uint64_t empty[PrefillCfg<D>::NSLOT];
    uint64_t s_free, s_full, p_full, o_done, drain;
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ bool chunk_rotated(int c, int d, int R) {
    const int lo = c * 64, hi = lo + 64, h = d / 2;
    return (lo < R) || (lo < h + R && hi > h);
}

struct TileGeom {
    int b, g, m0;      // batch, kv head, first token of the tile
    int tq;            // tokens in the tile (<= 128 / G)
    int j_lo, j_hi;    // key tiles visited (inclusive)
};

__device__ __forceinline__ TileGeom tile_geom(const PrefillArgs& a) {
    TileGeom g;
    const int tpt = kBM / a.G;                         // tokens per tile
    const int mt_count = (a.T + tpt - 1) / tpt;
    // heavy tiles first: the last query tiles of a causal layer see the most keys
    const int idx = blockIdx.x;
    const int mt = mt_count - 1 - idx / (a.B * a.Hkv);
    const int bg = idx % (a.B * a.Hkv);
    g.b = bg / a.Hkv;
    g.g = bg % a.Hkv;
    g.m0 = mt * tpt;
    g.tq = min(tpt, a.T - g.m0);
    const int t_last = g.m0 + g.tq - 1;
    int k_first = 0;
    if (a.window > 0) k_first = max(0, g.m0 - a.window + 1);
    g.j_lo = k_first / kBN;
    g.j_hi = t_last / kBN;
    return g;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ PrefillArgs a) {
    using C = PrefillCfg<D>;
    constexpr int NCH = C::NCH;
    constexpr int NSLOT = C::NSLOT;
    extern __shared__ uint8_t smem_raw[];
    PrefillSmem<D>& sm = *reinterpret_cast<PrefillSmem<D>*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const WaitCtl wc{a.wait_limit, a.status};
    volatile int* abort = &sm.abort;
    const int R = a.rope.R;
    const TileGeom tg = tile_geom(a);
    const int ntiles = tg.j_hi - tg.j_lo + 1;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NSLOT; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], 1);
        }
        mbar_init(&sm.s_free, 1);
        mbar_init(&sm.s_full, 1);
        mbar_init(&sm.p_full, 1);
        mbar_init(&sm.o_done, 1);
        mbar_init(&sm.drain, 1);
        sm.abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(&sm.tmem_base, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t tm_o = tmem;
    const uint32_t tm_s = tmem + C::S_COL;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            prefetch_tmap(&a.tm_kn);
            prefetch_tmap(&a.tm_kr);
            prefetch_tmap(&a.tm_v);
            uint32_t q = 0;
            for (int n = 0; n < ntiles && !*abort; ++n) {
                const int key = (tg.j_lo + n) * kBN;
                if (n + 2 < ntiles)
                    for (int c = 0; c < NCH; ++c) {
                        const bool rot = chunk_rotated(c, D, R);
                        const CUtensorMap* ms = rot ? &a.tm_kr : &a.tm_kn;
                        const CUtensorMap* mv = a.kv_is_k == 0 ? &a.tm_v
                                                : (a.kv_is_k == 2 && rot) ? &a.tm_kr : &a.tm_kn;
                        tma_prefetch_l2_4d(ms, c * 64, tg.g, key + 2 * kBN, tg.b);
                        if (mv != ms) tma_prefetch_l2_4d(mv, c * 64, tg.g, key + 2 * kBN, tg.b);
                    }
                // S chunks then V chunks, in consumption order
                for (int pass = 0; pass < 2 && !*abort; ++pass)
                    for (int c = 0; c < NCH; ++c) {
                        const bool rot = chunk_rotated(c, D, R);
                        const CUtensorMap* map;
                        if (pass == 0) map = rot ? &a.tm_kr : &a.tm_kn;
                        else if (a.kv_is_k == 0) map = &a.tm_v;
                        else map = (a.kv_is_k == 2 && rot) ? &a.tm_kr : &a.tm_kn;
                        const int slot = q % NSLOT;
                        if (!mbar_wait(&sm.empty[slot], ((q / NSLOT) & 1) ^ 1, wc, abort)) break;
                        mbar_arrive_expect_tx(&sm.full[slot], kChunkBytes);
                        tma_load_4d(sm.ring[slot], map, &sm.full[slot], c * 64, tg.g, key, tg.b);
                        ++q;
                    }
            }
            if (*abort) {
                const uint32_t first = q > (uint32_t)NSLOT ? q - NSLOT : 0;
                for (uint32_t k = first; k < q; ++k)
                    mbar_wait_drain(&sm.full[k % NSLOT], (k / NSLOT) & 1, a.wait_limit);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            // S in fp16 (normalised q and k copies); P.V in fp16 when V is the normalised key
            // copy, in bf16 when V is the caller's bf16 values
            const uint32_t idesc_s = idesc_f16kind_f32(128, kBN, false, false, false);
            const uint32_t idesc_o = idesc_f16kind_f32(128, 256, false, true, a.kv_is_k == 0);
            uint32_t q = 0;
            for (int n = 0; n < ntiles; ++n) {
                if (!mbar_wait(&sm.s_free, n & 1, wc, abort)) goto done;
                tc_fence_after();
                for (int c = 0; c < NCH; ++c, ++q) {
                    const uint32_t slot = q % NSLOT;
                    if (!mbar_wait(&sm.full[slot], (q / NSLOT) & 1, wc, abort)) goto done;
                    tc_fence_after();
                    const uint32_t ab = smem_u32(sm.q[c]);
                    const uint32_t bb = smem_u32(sm.ring[slot]);
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16_ss(tm_s, sdesc_sw128(ab + kk * 32, 16, 1024),
                                    sdesc_sw128(bb + kk * 32, 16, 1024), idesc_s,
                                    (c | kk) != 0 ? 1u : 0u);
                    mma_commit(&sm.empty[slot]);
                }
                mma_commit(&sm.s_full);
                if (!mbar_wait(&sm.p_full, n & 1, wc, abort)) goto done;
                tc_fence_after();
                // O[:, 256*grp + 0..255] += P . V[:, 256*grp ...]: four consecutive ring slots
                for (int grp = 0; grp < NCH / 4; ++grp) {
                    const uint32_t q0 = q;
                    for (int u = 0; u < 4; ++u, ++q)
                        if (!mbar_wait(&sm.full[q % NSLOT], (q / NSLOT) & 1, wc, abort)) goto done;
                    tc_fence_after();
                    const uint32_t vb = smem_u32(sm.ring[q0 % NSLOT]);
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t pa = smem_u32(sm.p[kk >> 2]) + (kk & 3) * 32;
                        mma_bf16_ss(tm_o + grp * 256, sdesc_sw128(pa, 16, 1024),
                                    sdesc_sw128(vb + kk * 2048, kChunkBytes, 1024), idesc_o,
                                    (n > 0 || kk > 0) ? 1u : 0u);
                    }
                    for (int u = 0; u < 4; ++u) mma_commit(&sm.empty[(q0 + u) % NSLOT]);
                }
                if (C::SWAP || n == ntiles - 1) mma_commit(&sm.o_done);
            }
        done:
            mma_commit(&sm.drain);
            mbar_wait_drain(&sm.drain, 0, a.wait_limit);
        }
    } else {
        // ------------------------------------ prologue / softmax / correction / epilogue
        const int t128 = threadIdx.x - 64;
        const int wq = warp - 2;                  // 0..3 for the row-parallel prologue
        const int quarter = warp & 3;             // TMEM lane quarter
        const int row = quarter * 32 + lane;      // this thread's TMEM lane = tile row
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const int G = a.G;

        // ---- prologue: QKNorm + RoPE of the 128 packed rows (one warp per row at a time)
        {
            constexpr int E = D / 64;             // elements per lane in each half
            const int half = D / 2;
            for (int r = wq; r < kBM; r += 4) {
                const int tl = r / G, hl = r % G;
                const int tok = tg.m0 + tl;
                float x0[E], x1[E];
                if (tl < tg.tq) {
                    const uint16_t* src =
                        a.q + (((size_t)tg.b * a.T + tok) * a.Hq + (size_t)tg.g * G + hl) * D;
#pragma unroll
                    for (int e = 0; e < E; e += 2) {
                        const float2 f0 = __bfloat1622float2(
                            *reinterpret_cast<const __nv_bfloat162*>(src + lane * E + e));
                        const float2 f1 = __bfloat1622float2(
                            *reinterpret_cast<const __nv_bfloat162*>(src + half + lane * E + e));
                        x0[e] = f0.x; x0[e + 1] = f0.y;
                        x1[e] = f1.x; x1[e + 1] = f1.y;
                    }
                    if (a.qk_norm) {
                        float ss = 0.f;
#pragma unroll
                        for (int e = 0; e < E; ++e) ss += x0[e] * x0[e] + x1[e] * x1[e];
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
                        const float inv = 1.0f / sqrtf(ss / (float)D + a.eps);
#pragma unroll
                        for (int e = 0; e < E; ++e) {
                            x0[e] = x0[e] * inv * a.gamma_q[lane * E + e];
                            x1[e] = x1[e] * inv * a.gamma_q[half + lane * E + e];
                        }
                    }
#pragma unroll
                    for (int e = 0; e < E; ++e) {
                        const int i = lane * E + e;
                        if (i < R) {
                            const float2 cs = a.rope_cs[(size_t)tok * R + i];
                            const float u = x0[e], v = x1[e];
                            x0[e] = u * cs.x - v * cs.y;
                            x1[e] = u * cs.y + v * cs.x;
                        }
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < E; ++e) x0[e] = x1[e] = 0.f;
                }
                // store: element (r, col) of chunk col / 64
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const float* x = hh ? x1 : x0;
                    const int col = hh * half + lane * E;
                    uint32_t w[E / 2];
#pragma unroll
                    for (int e = 0; e < E; e += 2) w[e / 2] = pack_f16x2(x[e], x[e + 1]);
                    uint8_t* base = sm.q[col / 64];
                    const uint32_t off = sw128_offset(r, col % 64);
                    if constexpr (E == 8)
                        *reinterpret_cast<uint4*>(base + off) = make_uint4(w[0], w[1], w[2], w[3]);
                    else if constexpr (E == 4)
                        *reinterpret_cast<uint2*>(base + off) = make_uint2(w[0], w[1]);
                    else
                        *reinterpret_cast<uint32_t*>(base + off) = w[0];
                }
            }
            fence_proxy_async_smem();
            group_sync(kBarWG, 128);
            if (t128 == 0) mbar_arrive(&sm.s_free);   // Q ready, S region free for tile 0
        }

        // ---- main loop
        const bool p_f16 = a.kv_is_k != 0;           // P in the format of V
        const int tok_r = tg.m0 + row / G;          // token of this row
        const bool row_valid = (row / G) < tg.tq;
        float m_ref = -INFINITY, l_sum = 0.f;
        float o1[C::SWAP ? 128 : 1];
        if constexpr (C::SWAP) {
#pragma unroll
            for (int i = 0; i < 128; ++i) o1[i] = 0.f;
        }
        bool ok = true;
        for (int n = 0; n < ntiles && ok; ++n) {
            const int key0 = (tg.j_lo + n) * kBN;
            if constexpr (C::SWAP) {
                if (n > 0) {
                    // O[:, 128..255] leaves TMEM so S(n) can use those columns
                    ok = group_all(mbar_wait(&sm.o_done, (n - 1) & 1, wc, abort), kBarWG, 128);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int c = 0; c < 8; ++c) tmem_ld16(tm_s + c * 16 + lane_off, o1 + c * 16);
                    tmem_ld_wait();
                    tc_fence_before();
                    group_sync(kBarWG, 128);
                    if (t128 == 0) mbar_arrive(&sm.s_free);
                }
            } else {
                if (n > 0 && t128 == 0) mbar_arrive(&sm.s_free);
            }
            ok = group_all(mbar_wait(&sm.s_full, n & 1, wc, abort), kBarWG, 128);
            if (!ok) break;
            tc_fence_after();
            // does any key of this tile need masking for any row of the CTA?
            const int t_first = tg.m0, t_last = tg.m0 + tg.tq - 1;
            const bool need_mask = (key0 + kBN - 1 > t_first) ||
                                   (a.window > 0 && key0 <= t_last - a.window);
            const int lo_r = a.window > 0 ? tok_r - a.window + 1 : 0;
            // pass 1: row max of the scaled, masked scores
            float mx = -INFINITY;
#pragma unroll 1
            for (int c = 0; c < 8; ++c) {
                float s[16];
                tmem_ld16(tm_s + c * 16 + lane_off, s);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int j = key0 + c * 16 + e;
                    const bool vis = !need_mask || (j <= tok_r && j >= lo_r);
                    mx = fmaxf(mx, vis ? s[e] * a.scale_log2 : -INFINITY);
                }
            }
            if (!row_valid) mx = -INFINITY;
            // lazy reference max: move it only when the tile max exceeds it by > 2^8
            float alpha = 1.f;
            if (mx > m_ref + kLazyMax || (m_ref == -INFINITY && mx != -INFINITY)) {
                alpha = (m_ref == -INFINITY) ? 0.f : exp2f(m_ref - mx);
                m_ref = mx;
            }
            // pass 2: P = exp2(s * scale_log2 - m_ref) as bf16 into the A tile of P.V
            float psum = 0.f;
#pragma unroll 1
            for (int c = 0; c < 8; ++c) {
                float s[16];
                tmem_ld16(tm_s + c * 16 + lane_off, s);
                tmem_ld_wait();
                uint32_t w[8];
#pragma unroll
                for (int e = 0; e < 16; e += 2) {
                    float pv[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int j = key0 + c * 16 + e + u;
                        const bool vis = row_valid && (!need_mask || (j <= tok_r && j >= lo_r));
                        pv[u] = vis ? exp2f(fmaf(s[e + u], a.scale_log2, -m_ref)) : 0.f;
                    }
                    // the row sum uses the rounded weights the MMA sees
                    if (p_f16) {
                        const __half2 h = __floats2half2_rn(pv[0], pv[1]);
                        const float2 f = __half22float2(h);
                        psum += f.x + f.y;
                        w[e / 2] = *reinterpret_cast<const uint32_t*>(&h);
                    } else {
                        const __nv_bfloat162 h = __floats2bfloat162_rn(pv[0], pv[1]);
                        const float2 f = __bfloat1622float2(h);
                        psum += f.x + f.y;
                        w[e / 2] = *reinterpret_cast<const uint32_t*>(&h);
                    }
                }
                uint8_t* pb = sm.p[c >> 2];
                const int col = (c & 3) * 16;
                *reinterpret_cast<uint4*>(pb + sw128_offset(row, col)) =
                    make_uint4(w[0], w[1], w[2], w[3]);
                *reinterpret_cast<uint4*>(pb + sw128_offset(row, col + 8)) =
                    make_uint4(w[4], w[5], w[6], w[7]);
            }
            l_sum = l_sum * alpha + psum;
            // correction of the accumulator when the reference max moved (rare)
            const bool warp_rescale = __any_sync(0xffffffffu, alpha != 1.f && n > 0);
            if constexpr (C::SWAP) {
#pragma unroll
                for (int i = 0; i < 128; ++i) o1[i] *= alpha;
            }
            if (warp_rescale) {
                for (int c = 0; c < D / 16; ++c) {
                    if (C::SWAP && c >= 8 && c < 16) continue;   // that quarter is in o1
                    float o[16];
                    tmem_ld16(tm_o + c * 16 + lane_off, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 16; ++e) o[e] *= alpha;
                    tmem_st16(tm_o + c * 16 + lane_off, o);
                }
                tmem_st_wait();
            }
            if constexpr (C::SWAP) {
                // put O[:, 128..255] back for the P.V product
#pragma unroll
                for (int c = 0; c < 8; ++c) tmem_st16(tm_s + c * 16 + lane_off, o1 + c * 16);
                tmem_st_wait();
            }
            fence_proxy_async_smem();
            tc_fence_before();
            group_sync(kBarWG, 128);
            if (t128 == 0) mbar_arrive(&sm.p_full);
        }
        // ---- epilogue
        if (ok) {
            const uint32_t last = C::SWAP ? (uint32_t)(ntiles - 1) : 0u;
            ok = group_all(mbar_wait(&sm.o_done, last & 1, wc, abort), kBarWG, 128);
        }
        if (ok) {
            tc_fence_after();
            const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
            const int h = tg.g * G + row % G;
            uint16_t* dst = a.out + (((size_t)tg.b * a.T + tok_r) * a.Hq + h) * D;
            for (int c = 0; c < D / 16; ++c) {
                float o[16];
                tmem_ld16(tm_o + c * 16 + lane_off, o);
                tmem_ld_wait();
                if (row_valid) {
                    uint32_t w[8];
#pragma unroll
                    for (int e = 0; e < 16; e += 2) w[e / 2] = pack_bf16x2(o[e] * inv, o[e + 1] * inv);
                    *reinterpret_cast<uint4*>(dst + c * 16) = make_uint4(w[0], w[1], w[2], w[3]);
                    *reinterpret_cast<uint4*>(dst + c * 16 + 8) = make_uint4(w[4], w[5], w[6], w[7]);
                }
            }
            if (row_valid && a.lse)
                a.lse[((size_t)tg.b * a.Hq + h) * a.T + tok_r] =
                    l_sum > 0.f ? (m_ref + log2f(l_sum)) * 0.6931471805599453f : -INFINITY;
        }
    }

    // -------------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int D>
cudaError_t run_prefill(const PrefillArgs& a, cudaStream_t stream) {
    const size_t smem = sizeof(PrefillSmem<D>) + 1024;
    cudaError_t e = cudaFuncSetAttribute(prefill_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int tpt = kBM / a.G;
    const int mt_count = (a.T + tpt - 1) / tpt;
    const long long grid = (long long)mt_count * a.B * a.Hkv;
    prefill_kernel<D><<<(unsigned)grid, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

size_t prefill_smem_bytes(int d) {
    return d == 512 ? sizeof(PrefillSmem<512>) + 1024 : sizeof(PrefillSmem<256>) + 1024;
}

cudaError_t launch_prefill(const PrefillArgs& a, cudaStream_t stream) {
    if (a.B == 0 || a.T == 0) return cudaSuccess;
    if (a.d == 512) return run_prefill<512>(a, stream);
    if (a.d == 256) return run_prefill<256>(a, stream);
    return cudaErrorInvalidValue;
}

}  // namespace g4

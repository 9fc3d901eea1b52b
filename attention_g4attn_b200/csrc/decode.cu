// decode.cu -- split-KV flash decoding for one new token per sequence against a bf16
// K(=V) cache, on the 5th-generation tensor core (tcgen05) with TMA-fed shared memory.
//
// Work item = (split s, kv head g, batch b): keys [k0, k1) of one sequence and all G query
// heads that share kv head g (GQA; explainer "GQA": 8 query heads per KV head in global
// layers).  Per tile of 128 keys:
//   S^T[key, head]  = K_tile . Q^T         M = 128 keys, N = 16 (heads, zero padded), K = d
//   O^T[d, head]   += K_tile^T . P^T        M = 128 d-rows per chunk, N = 16, K = 128 keys
// Keys sit on the MMA's M side, so one 128-key tile in shared memory is the K operand of
// the first product and, read MN-major, the V operand of the second (keys reused as
// values, report section 2 / explainer "K=V": one cache read serves both).  The cache
// holds pre-RoPE keys; the rotated pairs (i, i + d/2), i < R, of every key are turned to
// the key's position on the fly (report section 2, p-RoPE) by the softmax warps, in place.
// When the values are the pre-RoPE keys, the value operand is a second TMA pass over the
// same rows (served from L2: the score pass has just read them), so the score copy can be
// turned in place and released as soon as S^T has read it; HBM still reads the cache once.
//
// Warp roles (192 threads): warp 0 TMA producer, warp 1 MMA issuer and TMEM owner,
// warps 2..5 rotation / softmax / epilogue (thread = TMEM lane = key row or d-row).
// The CTA is persistent over work items blockIdx.x, +gridDim.x, ...  Every mbarrier wait
// is bounded (sm100.cuh); on a timeout all roles drain their in-flight work and exit.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <mutex>

#include "kernels.h"
#include "rope.cuh"
#include "sm100.cuh"

namespace g4 {
namespace {

constexpr int kThreads = 192;
constexpr int kTileKeys = 128;
constexpr int kNSlots = 5;           // ring of 32 KB slots: 128 keys x 128 dims (2 chunks)
constexpr int kMaxRotChunks = 2;     // side buffers for the turned chunks (values = pre-RoPE)
constexpr int kSlotBytes = 32768;
constexpr int kChunkBytes = 16384;   // 128 keys x 64 dims, 128-byte swizzled rows
constexpr int kN = 16;               // MMA N: query heads of one KV head, zero padded
constexpr uint32_t kTmemCols = 128;
constexpr int kBarWG = 1;            // named barrier of the softmax warpgroup
constexpr float kLazyMax = 8.0f;     // log2 units: headroom of the lazy reference max
constexpr int kPrefetchTiles = 3;    // L2 prefetch distance, in tiles

struct __align__(1024) DecodeSmem {
    uint8_t ring[kNSlots][kSlotBytes];
    uint8_t rot[kMaxRotChunks][kChunkBytes];
    uint8_t q[8][kN * 128];          // B operand of S^T: per 64-dim chunk, 16 rows x 128 B
    uint8_t p[2][kN * 128];          // B operand of O^T: P^T, K-major, 2 chunks of 64 keys
    float theta[256];                // base^(-2i/d) in fp32, i < R
    float2 base_cs[256];             // cos/sin of tile_start * theta_i
    float2 step_cs[256];             // cos/sin of 128 * theta_i: one tile further
    float red[4][kN];                // cross-warp reductions
    float qb[kN][128];               // rotated dims of q (first and second half, R <= 64)
    uint64_t full[kNSlots];
    uint64_t empty[kNSlots];
    uint64_t s_full, p_full, rot_ready, q_ready, o_done, drain;
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

struct Item {
    int s, g, b, k0, k1;
};

// Splits of one sequence are consecutive items, so concurrent CTAs stream neighbouring
// key ranges of the same (b, g).
__device__ __forceinline__ Item item_of(const DecodeArgs& a, int it) {
    Item r;
    r.s = it % a.splits;
    const int bg = it / a.splits;
    r.g = bg % a.Hkv;
    r.b = bg / a.Hkv;
    r.k0 = a.key_lo + r.s * a.keys_per_split;
    r.k1 = min(a.L, r.k0 + a.keys_per_split);
    if (r.k1 < r.k0) r.k1 = r.k0;
    return r;
}

// Does 64-dim chunk c hold rotated dims?  Rotated dims: [0, R) and [d/2, d/2 + R).
__device__ __forceinline__ bool chunk_rotated(int c, int d, int R) {
    const int lo = c * 64, hi = lo + 64, h = d / 2;
    return (lo < R) || (lo < h + R && hi > h);
}

// D: head dim; NH: query heads per KV head handled by the softmax (8 or 16, >= G);
// REL: relative rotation (values are not the rotated key and R <= 64).
// Chunk (64 dims) held by half h of the k-th slot of a tile.  Score slots of the two-pass
// mode pair each chunk with its rotation partner (chunks k and k + NCH/2), so turning a
// key needs one slot; value slots, and the slots of the one-pass mode (values = rotated
// keys), hold consecutive chunks (2k, 2k+1), the 128 value rows of one O^T block.
// One-pass slots hold chunk pairs (2m, 2m+1) in the order m = 0, npair/2, 1, npair/2+1, ...
// so the two rotation partners (chunks 0 and nch/2) arrive in the first two slots.
__device__ __forceinline__ int slot_pair(int k, int npair) {
    return (k & 1) ? (npair / 2 + k / 2) : (k / 2);
}
__device__ __forceinline__ int slot_chunk(int k, int h, bool partner_pairs, int nch) {
    return partner_pairs ? k + h * (nch / 2) : 2 * slot_pair(k, nch / 2) + h;
}
// Slot index and half of chunk c within a tile.
__device__ __forceinline__ void chunk_slot(int c, bool partner_pairs, int nch, int& k, int& h) {
    if (partner_pairs) {
        k = c % (nch / 2);
        h = c / (nch / 2);
    } else {
        const int m = c / 2, np = nch / 2;
        h = c & 1;
        k = (m < np / 2) ? 2 * m : 2 * (m - np / 2) + 1;
    }
}

template <int D, int NH, bool REL>
__global__ void __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ DecodeArgs a) {
    constexpr int NCH = D / 64;     // 64-dim chunks per key row
    constexpr int NPAIR = D / 128;  // 32 KB ring slots per tile and tensor
    extern __shared__ uint8_t smem_raw[];
    DecodeSmem& sm = *reinterpret_cast<DecodeSmem*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const WaitCtl wc{a.wait_limit, a.status};
    volatile int* abort = &sm.abort;
    const int R = a.rope.R;
    // One pass over the cache: a tile in shared memory is the K operand of S^T and the V
    // operand of O^T.  Turned chunks go to side buffers when the values are the pre-RoPE
    // keys, in place when they are the rotated keys.  Separate values take a second pass.
    const bool sep_v = a.kv_is_k == 0;
    const bool side_rot = a.kv_is_k == 1;
    const int n_items = a.splits * a.Hkv * a.B;
    const int slots_per_tile = sep_v ? 2 * NPAIR : NPAIR;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kNSlots; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], 1);
        }
        mbar_init(&sm.s_full, 1);
        mbar_init(&sm.p_full, 1);
        mbar_init(&sm.rot_ready, 1);
        mbar_init(&sm.q_ready, 1);
        mbar_init(&sm.o_done, 1);
        mbar_init(&sm.drain, 1);
        sm.abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(&sm.tmem_base, kTmemCols);
    if (warp >= 2) {
        for (int i = threadIdx.x - 64; i < R; i += 128) {
            sm.theta[i] = (float)exp2(-(2.0 * (double)i / (double)D) * a.rope.log2_base);
            sm.step_cs[i] = rope_cos_sin((long long)kTileKeys, i, D, a.rope.log2_base);
        }
        for (int i = threadIdx.x - 64; i < (int)(sizeof(sm.p) / 16); i += 128)
            reinterpret_cast<uint4*>(&sm.p[0][0])[i] = make_uint4(0, 0, 0, 0);
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t tm_s = tmem;          // S^T: 16 columns
    const uint32_t tm_o = tmem + 16;     // O^T: NPAIR blocks of 16 columns

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            prefetch_tmap(&a.tm_k);
            if (sep_v) prefetch_tmap(&a.tm_v);
            // L2 prefetch cursor: runs kPrefetchTiles tiles ahead of the loads, across the
            // items of this CTA, so HBM keeps streaming while the ring slots are busy
            int pf_it = blockIdx.x, pf_t = 0;
            long long pf_count = 0, load_count = 0;
            uint32_t q = 0;   // ring slots filled so far
            for (int it = blockIdx.x; it < n_items && !*abort; it += gridDim.x) {
                const Item w = item_of(a, it);
                const int nt = ceil_div(w.k1 - w.k0, kTileKeys);
                for (int t = 0; t < nt && !*abort; ++t, ++load_count) {
                    const int key = w.k0 + t * kTileKeys;
                    while (pf_count <= load_count + kPrefetchTiles && pf_it < n_items) {
                        const Item pw = item_of(a, pf_it);
                        const int pnt = ceil_div(pw.k1 - pw.k0, kTileKeys);
                        if (pf_t < pnt) {
                            const int pk = pw.k0 + pf_t * kTileKeys;
                            for (int c = 0; c < NCH; ++c) {
                                tma_prefetch_l2_4d(&a.tm_k, c * 64, pw.g, pk, pw.b);
                                if (a.kv_is_k == 0)   // a separate value cache
                                    tma_prefetch_l2_4d(&a.tm_v, c * 64, pw.g, pk, pw.b);
                            }
                            ++pf_count;
                        }
                        if (++pf_t >= pnt) {
                            pf_t = 0;
                            pf_it += gridDim.x;
                        }
                    }
                    for (int pass = 0; pass < (sep_v ? 2 : 1) && !*abort; ++pass) {
                        const CUtensorMap* map = pass ? &a.tm_v : &a.tm_k;
                        const bool partner = sep_v && pass == 0;
                        for (int k = 0; k < NPAIR; ++k) {
                            const int slot = q % kNSlots;
                            if (!mbar_wait(&sm.empty[slot], ((q / kNSlots) & 1) ^ 1, wc, abort))
                                break;
                            mbar_arrive_expect_tx(&sm.full[slot], kSlotBytes);
                            for (int h = 0; h < 2; ++h) {
                                const int c = pass ? 2 * k + h : slot_chunk(k, h, partner, NCH);
                                tma_load_4d(sm.ring[slot] + h * kChunkBytes, map, &sm.full[slot],
                                            c * 64, w.g, key, w.b);
                            }
                            ++q;
                        }
                    }
                }
            }
            // before the CTA exits, every copy it started must have landed
            if (*abort) {
                const uint32_t first = q > (uint32_t)kNSlots ? q - kNSlots : 0;
                for (uint32_t k = first; k < q; ++k)
                    mbar_wait_drain(&sm.full[k % kNSlots], (k / kNSlots) & 1, a.wait_limit);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc_s = idesc_bf16_f32(128, kN, false, false);
            const uint32_t idesc_o = idesc_bf16_f32(128, kN, true, false);  // A = V^T, MN-major
            uint32_t q = 0, tile = 0, item_n = 0;
            for (int it = blockIdx.x; it < n_items; it += gridDim.x, ++item_n) {
                const Item w = item_of(a, it);
                const int nt = ceil_div(w.k1 - w.k0, kTileKeys);
                if (!mbar_wait(&sm.q_ready, item_n & 1, wc, abort)) goto done;
                for (int t = 0; t < nt; ++t, ++tile) {
                    const uint32_t qk = q;
                    const uint32_t qv = sep_v ? q + NPAIR : q;
                    bool first = true;
                    // S^T over the chunks that need no rotation, as soon as they land; in the
                    // two-pass mode each score slot is released right after its last MMA
                    for (int k = 0; k < NPAIR; ++k) {
                        const uint32_t qq = qk + k, slot = qq % kNSlots;
                        if (!mbar_wait(&sm.full[slot], (qq / kNSlots) & 1, wc, abort)) goto done;
                        tc_fence_after();
                        bool has_rot = false;
                        for (int h = 0; h < 2; ++h) {
                            const int c = slot_chunk(k, h, sep_v, NCH);
                            if (chunk_rotated(c, D, R)) { has_rot = true; continue; }
                            const uint32_t ab = smem_u32(sm.ring[slot] + h * kChunkBytes);
                            const uint32_t bb = smem_u32(sm.q[c]);
                            for (int kk = 0; kk < 4; ++kk) {
                                mma_bf16_ss(tm_s, sdesc_sw128(ab + kk * 32, 16, 1024),
                                            sdesc_sw128(bb + kk * 32, 16, 1024), idesc_s,
                                            first ? 0u : 1u);
                                first = false;
                            }
                        }
                        if (sep_v && !has_rot) mma_commit(&sm.empty[slot]);
                    }
                    // then the rotated chunks, once the softmax warps have turned them
                    if (R > 0) {
                        if (!mbar_wait(&sm.rot_ready, tile & 1, wc, abort)) goto done;
                        tc_fence_after();
                        for (int k = 0; k < NPAIR; ++k) {
                            const uint32_t slot = (qk + k) % kNSlots;
                            bool has_rot = false;
                            for (int h = 0; h < 2; ++h) {
                                const int c = slot_chunk(k, h, sep_v, NCH);
                                if (!chunk_rotated(c, D, R)) continue;
                                has_rot = true;
                                const uint32_t ab =
                                    side_rot ? smem_u32(sm.rot[c == 0 ? 0 : 1])
                                             : smem_u32(sm.ring[slot] + h * kChunkBytes);
                                const uint32_t bb = smem_u32(sm.q[c]);
                                for (int kk = 0; kk < 4; ++kk) {
                                    mma_bf16_ss(tm_s, sdesc_sw128(ab + kk * 32, 16, 1024),
                                                sdesc_sw128(bb + kk * 32, 16, 1024), idesc_s,
                                                first ? 0u : 1u);
                                    first = false;
                                }
                            }
                            if (sep_v && has_rot) mma_commit(&sm.empty[slot]);
                        }
                    }
                    mma_commit(&sm.s_full);
                    // O^T += V^T . P^T once the softmax warps have written P
                    if (!mbar_wait(&sm.p_full, tile & 1, wc, abort)) goto done;
                    tc_fence_after();
                    for (int pr = 0; pr < NPAIR; ++pr) {
                        const uint32_t k = qv + pr, slot = k % kNSlots;
                        if (sep_v && !mbar_wait(&sm.full[slot], (k / kNSlots) & 1, wc, abort))
                            goto done;
                        tc_fence_after();
                        const int blk = sep_v ? pr : slot_pair(pr, NPAIR);   // O^T block
                        const uint32_t ab = smem_u32(sm.ring[slot]);
                        for (int kk = 0; kk < 8; ++kk) {
                            // 16 keys per step = two 8-row groups of 1024 B; the slot's second
                            // 64-dim chunk is the next 64-element MN block (LBO)
                            const uint64_t ad = sdesc_sw128(ab + kk * 2048, kChunkBytes, 1024);
                            const uint32_t pb = smem_u32(sm.p[kk >> 2]) + (kk & 3) * 32;
                            mma_bf16_ss(tm_o + blk * 16, ad, sdesc_sw128(pb, 16, 1024), idesc_o,
                                        (t > 0 || kk > 0) ? 1u : 0u);
                        }
                        mma_commit(&sm.empty[slot]);   // each slot as soon as its MMAs finish
                    }
                    q += slots_per_tile;
                }
                mma_commit(&sm.o_done);
            }
        done:
            // all issued MMAs must finish before the tensor memory is released
            mma_commit(&sm.drain);
            mbar_wait_drain(&sm.drain, 0, a.wait_limit);
        }
    } else {
        // ---------------------------------------------- rotation / softmax / epilogue
        const int t128 = threadIdx.x - 64;            // 0..127
        const int quarter = warp & 3;                 // TMEM lane quarter of this warp
        const int row = quarter * 32 + lane;          // TMEM lane: key row or d-row
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const int G = a.G;
        const float c2 = a.scale_log2;
        // Relative rotation (REL): key row `row` of every tile sits at angle row*theta_i from
        // the tile start, so its (cos, sin) are fixed per thread; the tile start angle goes
        // onto the query instead: q' = R(-key0 theta) q, and q' . R(row theta) k equals
        // q . R((key0 + row) theta) k.
        __half2 rcs[REL ? 64 : 1];
        if constexpr (REL) {
#pragma unroll
            for (int i = 0; i < 64; ++i) {
                float sn = 0.f, cn = 1.f;
                if (i < R) sincosf((float)row * sm.theta[i], &sn, &cn);
                rcs[i] = __floats2half2_rn(cn, sn);
            }
        }
        uint32_t q = 0, tile = 0, item_n = 0;
        bool ok = true;
        for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++item_n) {
            const Item w = item_of(a, it);
            const int nt = ceil_div(w.k1 - w.k0, kTileKeys);
            // stage the G queries of (b, g) as the B operand of S^T (K-major, swizzled)
            for (int e = t128; e < kN * (D / 8); e += 128) {
                const int h = e / (D / 8), c8 = e % (D / 8);
                uint4 v = make_uint4(0, 0, 0, 0);
                if (h < G)
                    v = *reinterpret_cast<const uint4*>(
                        a.q + ((size_t)w.b * a.Hq + (size_t)w.g * G + h) * D + c8 * 8);
                *reinterpret_cast<uint4*>(sm.q[c8 / 8] + sw128_offset(h, (c8 % 8) * 8)) = v;
            }
            if constexpr (REL) {   // the rotated dims of q, to be turned per tile
                for (int e = t128; e < NH * 2 * R; e += 128) {
                    const int h = e / (2 * R), k = e % (2 * R);
                    const int dim = k < R ? k : D / 2 + (k - R);
                    float v = 0.f;
                    if (h < G)
                        v = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
                            a.q + ((size_t)w.b * a.Hq + (size_t)w.g * G + h) * D + dim));
                    sm.qb[h][k < R ? k : 64 + (k - R)] = v;
                }
            }
            fence_proxy_async_smem();
            group_sync(kBarWG, 128);
            if (t128 == 0) mbar_arrive(&sm.q_ready);

            float m_run[NH], l_part[NH];
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                m_run[h] = -INFINITY;
                l_part[h] = 0.f;
            }
            for (int t = 0; t < nt; ++t, ++tile) {
                const int key0 = w.k0 + t * kTileKeys;
                const uint32_t qk = q;
                q += slots_per_tile;
                // ---- turn the rotated pairs of this tile's keys (and, REL, the queries)
                if (R > 0) {
                    // start angle of the tile: exact (fp64-reduced) at the first tile of an
                    // item, then advanced by one tile (128 keys) per step
                    for (int i = t128; i < R; i += 128) {
                        if (t == 0) {
                            sm.base_cs[i] = rope_cos_sin((long long)key0, i, D, a.rope.log2_base);
                        } else {
                            const float2 b0 = sm.base_cs[i], st = sm.step_cs[i];
                            sm.base_cs[i] = make_float2(b0.x * st.x - b0.y * st.y,
                                                        b0.x * st.y + b0.y * st.x);
                        }
                    }
                    bool got = true;
                    for (int k = 0; k < NPAIR && got; ++k)
                        if (chunk_rotated(slot_chunk(k, 0, sep_v, NCH), D, R) ||
                            chunk_rotated(slot_chunk(k, 1, sep_v, NCH), D, R))
                            got = mbar_wait(&sm.full[(qk + k) % kNSlots],
                                            ((qk + k) / kNSlots) & 1, wc, abort);
                    ok = group_all(got, kBarWG, 128);   // also orders base_cs writes
                    if (!ok) break;
                    if constexpr (REL) {
                        // q' = R(-key0 theta) q on the rotated dims (chunks 0 and NCH/2)
                        for (int e = t128; e < G * R; e += 128) {
                            const int h = e / R, i = e % R;
                            const float2 cs = sm.base_cs[i];
                            const float x = sm.qb[h][i], y = sm.qb[h][64 + i];
                            *reinterpret_cast<__nv_bfloat16*>(sm.q[0] + sw128_offset(h, i)) =
                                __float2bfloat16_rn(x * cs.x + y * cs.y);
                            *reinterpret_cast<__nv_bfloat16*>(sm.q[NCH / 2] + sw128_offset(h, i)) =
                                __float2bfloat16_rn(y * cs.x - x * cs.y);
                        }
                        // keys: R(row theta) on the rotated pairs of this thread's row
                        int k1, h1s, k2, h2s;
                        chunk_slot(0, sep_v, NCH, k1, h1s);
                        chunk_slot(NCH / 2, sep_v, NCH, k2, h2s);
                        uint8_t* src1 = sm.ring[(qk + k1) % kNSlots] + h1s * kChunkBytes;
                        uint8_t* src2 = sm.ring[(qk + k2) % kNSlots] + h2s * kChunkBytes;
                        uint8_t* dst1 = side_rot ? sm.rot[0] : src1;
                        uint8_t* dst2 = side_rot ? sm.rot[1] : src2;
#pragma unroll
                        for (int g8 = 0; g8 < 8; ++g8) {
                            const bool rotg = g8 * 8 < R;
                            if (!side_rot && !rotg) continue;   // in place: nothing to copy
                            const uint32_t off = sw128_offset(row, g8 * 8);
                            uint4 x1 = *reinterpret_cast<const uint4*>(src1 + off);
                            uint4 x2 = *reinterpret_cast<const uint4*>(src2 + off);
                            if (rotg) {
                                __nv_bfloat162* h1 = reinterpret_cast<__nv_bfloat162*>(&x1);
                                __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&x2);
#pragma unroll
                                for (int e2 = 0; e2 < 4; ++e2) {
                                    const float2 u = __bfloat1622float2(h1[e2]);
                                    const float2 v = __bfloat1622float2(h2[e2]);
                                    const int i0 = g8 * 8 + 2 * e2;
                                    const float2 ca = __half22float2(rcs[i0]);
                                    const float2 cb = __half22float2(rcs[i0 + 1]);
                                    const bool r0 = i0 < R, r1 = i0 + 1 < R;
                                    const float u0 = r0 ? u.x * ca.x - v.x * ca.y : u.x;
                                    const float v0 = r0 ? u.x * ca.y + v.x * ca.x : v.x;
                                    const float u1 = r1 ? u.y * cb.x - v.y * cb.y : u.y;
                                    const float v1 = r1 ? u.y * cb.y + v.y * cb.x : v.y;
                                    h1[e2] = __floats2bfloat162_rn(u0, u1);
                                    h2[e2] = __floats2bfloat162_rn(v0, v1);
                                }
                            }
                            *reinterpret_cast<uint4*>(dst1 + off) = x1;
                            *reinterpret_cast<uint4*>(dst2 + off) = x2;
                        }
                    } else {
                        // absolute angles: angle(key0 + row) = angle(key0) + row * theta_i
                        const float fr = (float)row;
                        for (int c = 0; c < NCH / 2; ++c) {
                            if (!chunk_rotated(c, D, R)) continue;
                            const int c2i = c + NCH / 2;   // partner chunk: dims + d/2
                            uint8_t* src1;
                            uint8_t* src2;
                            int k1, h1s, k2, h2s;
                            chunk_slot(c, sep_v, NCH, k1, h1s);
                            chunk_slot(c2i, sep_v, NCH, k2, h2s);
                            src1 = sm.ring[(qk + k1) % kNSlots] + h1s * kChunkBytes;
                            src2 = sm.ring[(qk + k2) % kNSlots] + h2s * kChunkBytes;
                            uint8_t* dst1 = side_rot ? sm.rot[0] : src1;
                            uint8_t* dst2 = side_rot ? sm.rot[1] : src2;
                            for (int g8 = 0; g8 < 8; ++g8) {
                                const uint32_t off = sw128_offset(row, g8 * 8);
                                uint4 x1 = *reinterpret_cast<const uint4*>(src1 + off);
                                uint4 x2 = *reinterpret_cast<const uint4*>(src2 + off);
                                __nv_bfloat162* h1 = reinterpret_cast<__nv_bfloat162*>(&x1);
                                __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&x2);
#pragma unroll
                                for (int e2 = 0; e2 < 4; ++e2) {
                                    const float2 u = __bfloat1622float2(h1[e2]);
                                    const float2 v = __bfloat1622float2(h2[e2]);
                                    float uo[2] = {u.x, u.y}, vo[2] = {v.x, v.y};
#pragma unroll
                                    for (int e = 0; e < 2; ++e) {
                                        const int i = c * 64 + g8 * 8 + e2 * 2 + e;
                                        if (i < R) {
                                            float x = fr * sm.theta[i];
                                            x = fmaf(-6.2831853f, rintf(x * 0.15915494f), x);
                                            float so, co;
                                            __sincosf(x, &so, &co);
                                            const float2 b = sm.base_cs[i];
                                            const float cc = b.x * co - b.y * so;
                                            const float ss = b.y * co + b.x * so;
                                            const float p0 = uo[e], p1 = vo[e];
                                            uo[e] = p0 * cc - p1 * ss;
                                            vo[e] = p0 * ss + p1 * cc;
                                        }
                                    }
                                    h1[e2] = __floats2bfloat162_rn(uo[0], uo[1]);
                                    h2[e2] = __floats2bfloat162_rn(vo[0], vo[1]);
                                }
                                *reinterpret_cast<uint4*>(dst1 + off) = x1;
                                *reinterpret_cast<uint4*>(dst2 + off) = x2;
                            }
                        }
                    }
                    fence_proxy_async_smem();
                    group_sync(kBarWG, 128);
                    if (t128 == 0) mbar_arrive(&sm.rot_ready);
                }
                // ---- softmax over the 128 keys of the tile (thread = key)
                ok = group_all(mbar_wait(&sm.s_full, tile & 1, wc, abort), kBarWG, 128);
                if (!ok) break;
                tc_fence_after();
                float s[kN];
                tmem_ld16(tm_s + lane_off, s);
                tmem_ld_wait();
                const bool valid = key0 + row < w.k1;
                float x[NH];
                bool big = false;
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    x[h] = (valid && h < G) ? s[h] * c2 : -INFINITY;
                    big |= x[h] > m_run[h] + kLazyMax;
                }
                // lazy reference max: only when some score of the tile exceeds the running
                // reference by more than 2^8 (and on the first tile) do the warps reduce
                const bool fast = (t > 0) && group_all(!big, kBarWG, 128);
                float alpha[NH];
#pragma unroll
                for (int h = 0; h < NH; ++h) alpha[h] = 1.f;
                if (!fast) {
                    float mt[NH];
#pragma unroll
                    for (int h = 0; h < NH; ++h) {
                        mt[h] = x[h];
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1)
                            mt[h] = fmaxf(mt[h], __shfl_xor_sync(0xffffffffu, mt[h], o));
                    }
                    if (lane == 0)
#pragma unroll
                        for (int h = 0; h < NH; ++h) sm.red[quarter][h] = mt[h];
                    group_sync(kBarWG, 128);
                    bool rescale = false;
#pragma unroll
                    for (int h = 0; h < NH; ++h) {
                        const float tmax = fmaxf(fmaxf(sm.red[0][h], sm.red[1][h]),
                                                 fmaxf(sm.red[2][h], sm.red[3][h]));
                        if (tmax > m_run[h] + kLazyMax ||
                            (m_run[h] == -INFINITY && tmax != -INFINITY)) {
                            alpha[h] = (m_run[h] == -INFINITY) ? 0.f : exp2f(m_run[h] - tmax);
                            m_run[h] = tmax;
                            rescale |= t > 0;
                        }
                    }
                    group_sync(kBarWG, 128);   // red[] is rewritten below
                    // rescale O^T (thread = d-row, column = head).  O is idle: the MMA that
                    // wrote S for this tile ran after the previous O update.
                    if (rescale) {
                        for (int pr = 0; pr < NPAIR; ++pr) {
                            float o[kN];
                            tmem_ld16(tm_o + pr * 16 + lane_off, o);
                            tmem_ld_wait();
#pragma unroll
                            for (int h = 0; h < NH; ++h) o[h] *= alpha[h];
                            tmem_st16(tm_o + pr * 16 + lane_off, o);
                        }
                        tmem_st_wait();
                    }
                }
                // P^T: row = head, K-major, 64 keys per 128-byte row, two chunks
                {
                    uint8_t* pb = sm.p[row >> 6];
                    const int kc = row & 63;
#pragma unroll
                    for (int h = 0; h < NH; ++h) {
                        const float p = (x[h] == -INFINITY) ? 0.f : ex2_approx(x[h] - m_run[h]);
                        const __nv_bfloat16 pr = __float2bfloat16_rn(p);
                        // the running sum uses the rounded weight the MMA sees
                        l_part[h] = l_part[h] * alpha[h] + __bfloat162float(pr);
                        *reinterpret_cast<__nv_bfloat16*>(pb + sw128_offset(h, kc)) = pr;
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                group_sync(kBarWG, 128);
                if (t128 == 0) mbar_arrive(&sm.p_full);
            }
            if (!ok) break;
            // ---- item epilogue: partial O^T, running max and sum
            ok = group_all(mbar_wait(&sm.o_done, item_n & 1, wc, abort), kBarWG, 128);
            if (!ok) break;
            tc_fence_after();
            const size_t obase = ((size_t)w.s * a.B + w.b) * a.Hq + (size_t)w.g * G;
            for (int pr = 0; pr < NPAIR; ++pr) {
                float o[kN];
                tmem_ld16(tm_o + pr * 16 + lane_off, o);
                tmem_ld_wait();
#pragma unroll
                for (int h = 0; h < NH; ++h)
                    if (h < G) a.part_o[(obase + h) * D + pr * 128 + row] = nt > 0 ? o[h] : 0.f;
            }
#pragma unroll
            for (int h = 0; h < NH; ++h)
#pragma unroll
                for (int o = 16; o > 0; o >>= 1)
                    l_part[h] += __shfl_xor_sync(0xffffffffu, l_part[h], o);
            if (lane == 0)
#pragma unroll
                for (int h = 0; h < NH; ++h) sm.red[quarter][h] = l_part[h];
            group_sync(kBarWG, 128);
            if (t128 < G) {
                const float l = sm.red[0][t128] + sm.red[1][t128] + sm.red[2][t128] +
                                sm.red[3][t128];
                float mv = m_run[0];
#pragma unroll
                for (int h = 1; h < NH; ++h) mv = (t128 == h) ? m_run[h] : mv;
                a.part_ml[(obase + t128) * 2 + 0] = mv;
                a.part_ml[(obase + t128) * 2 + 1] = l;
            }
            tc_fence_before();
            group_sync(kBarWG, 128);   // red[] and O^T are reused by the next item
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

// Merge the split partials of one (b, h):
//   out = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s,   M = max_s m_s (log2 units).
__global__ void decode_combine_kernel(const __grid_constant__ DecodeArgs a) {
    const int bh = blockIdx.x;   // b * Hq + h
    const size_t stride = (size_t)a.B * a.Hq;
    float M = -INFINITY;
    for (int s = 0; s < a.splits; ++s) M = fmaxf(M, a.part_ml[(s * stride + bh) * 2]);
    float den = 0.f;
    for (int s = 0; s < a.splits; ++s) {
        const float m = a.part_ml[(s * stride + bh) * 2];
        if (m != -INFINITY) den += exp2f(m - M) * a.part_ml[(s * stride + bh) * 2 + 1];
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    for (int c = threadIdx.x; c < a.d; c += blockDim.x) {
        float acc = 0.f;
        for (int s = 0; s < a.splits; ++s) {
            const float m = a.part_ml[(s * stride + bh) * 2];
            if (m != -INFINITY) acc += exp2f(m - M) * a.part_o[(s * stride + bh) * a.d + c];
        }
        a.out[(size_t)bh * a.d + c] = __bfloat16_as_ushort(__float2bfloat16_rn(acc * inv));
    }
    if (threadIdx.x == 0 && a.lse)
        a.lse[bh] = den > 0.f ? (M + log2f(den)) * 0.6931471805599453f : -INFINITY;
}

template <int D, int NH, bool REL>
cudaError_t run_decode(const DecodeArgs& a, int grid, size_t smem, cudaStream_t stream) {
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, NH, REL>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    decode_kernel<D, NH, REL><<<grid, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

template <int D>
cudaError_t dispatch_decode(const DecodeArgs& a, int grid, size_t smem, cudaStream_t stream) {
    const bool rel = a.kv_is_k != 2 && a.rope.R <= 64;
    if (a.G <= 8)
        return rel ? run_decode<D, 8, true>(a, grid, smem, stream)
                   : run_decode<D, 8, false>(a, grid, smem, stream);
    return rel ? run_decode<D, 16, true>(a, grid, smem, stream)
               : run_decode<D, 16, false>(a, grid, smem, stream);
}

}  // namespace

size_t decode_smem_bytes() { return sizeof(DecodeSmem) + 1024; }

// ------------------------------------------------------------------------------------
// Fixed scratch for g4attn_decode_noalloc: the split partials live in this file-scope
// device array instead of a caller workspace.  Every device that loads the library holds
// it until the process exits.  In host code the array's name is only a stand-in, so its
// device address is fetched with cudaGetSymbolAddress, once per device, with that device
// current, and passed to the kernels.
// ------------------------------------------------------------------------------------
constexpr size_t kDecodeScratchBytes = size_t(8) << 20;   // 8 MiB
static __device__ __align__(256) unsigned char g_decode_scratch[kDecodeScratchBytes];

size_t decode_scratch_bytes() { return kDecodeScratchBytes; }

cudaError_t decode_scratch_ptr(void** out) {
    constexpr int kMaxDev = 64;
    static void* ptr[kMaxDev] = {};
    static bool ready[kMaxDev] = {};
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(mu);
    if (!ready[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess) return e;
        ptr[dev] = p;
        ready[dev] = true;
    }
    *out = ptr[dev];
    return cudaSuccess;
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
    const size_t smem = decode_smem_bytes();
    const int n_items = a.splits * a.Hkv * a.B;
    if (n_items > 0) {
        int dev = 0, sms = 148;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const int grid = n_items < sms ? n_items : sms;
        cudaError_t e = a.d == 512 ? dispatch_decode<512>(a, grid, smem, stream)
                        : a.d == 256 ? dispatch_decode<256>(a, grid, smem, stream)
                                     : cudaErrorInvalidValue;
        if (e != cudaSuccess) return e;
    }
    if (a.B * a.Hq > 0) decode_combine_kernel<<<a.B * a.Hq, 128, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace g4

// decode.cu -- split-KV flash decoding for one new token per sequence against a bf16
// K(=V) cache, on the 5th-generation tensor core (tcgen05) with TMA-fed shared memory.
//
// Work item = a run of consecutive pair-tiles of one sequence (batch b, kv head g): keys
// [k0, k1) and all G query heads that share kv head g (GQA; explainer "GQA": 8 query heads
// per KV head in global layers).  The sequences' tiles form one flat range split evenly
// over the CTA pairs (stream-K), so a pair meets one to three items and every pair the same
// number of tiles; each item's results are one segment's partials of the combine.  Two CTAs of a cluster share an item and stream it in pair-tiles of 128 keys:
// CTA r takes keys [64 r, 64 r + 64) of each pair-tile and keeps its own running softmax,
// so each CTA's result is one partial of the split-KV combine.  A CTA's 64 keys sit in
// shared memory as D/128 slots of 128 rows x 64 dims: in slot j, row k < 64 holds dims
// [64j, 64j + 64) of key k and row 64 + k holds dims [d/2 + 64j, d/2 + 64j + 64) of the
// same key, so the two halves of every key row are stacked on the MMA's M side.  One
// 2-CTA MMA (cta_group::2, M = 256: 128 rows from each CTA) serves the pair:
//   S^T[half*64 + key, n] = K . Q^T over the slot's 64 dims        N = 2 NH
// where B rows n < NH (queries over the first-half dims) come from CTA 0 and rows n >= NH
// (second-half dims) from CTA 1; the two useful quarters of each CTA's S^T (rows < 64 with
// n < NH, rows >= 64 with n >= NH) are the two halves of its scores and are added by its
// softmax threads.  The same slot, read MN-major, is the value operand of
//   O^T[dim, n] += V^T . P^T                                        M = 128 dims per CTA
// with B rows n < NH holding CTA 0's P and rows n >= NH CTA 1's P: columns [r NH, r NH + NH)
// of CTA r's O^T are its own partial (keys reused as values, report section 2 / explainer
// "K=V": one cache read serves both).  RoPE pairs dims (i, i + d/2), i < R (report
// section 2, p-RoPE): both members of a pair sit in the same slot, rows k and 64 + k, so
// the rotation warps turn a key's rotated pairs inside one slot.  With pre-RoPE values the
// turned slot goes to a side buffer and the original stays as the value operand.
//
// Pipeline: per CTA, a rotation warpgroup waits for a pair-tile's slots, stages the queries
// of a new item and turns the rotated pairs, while a softmax warpgroup works on the tile
// before; one thread of the first CTA issues every MMA of the pair (a single issuing thread
// keeps the tensor pipe fed best), the value product of a tile as soon as both CTAs' P are
// ready and the score product of the next tile once both CTAs have it turned.
//
// Warp roles (320 threads per CTA): warp 0 TMA producer, warp 1 TMEM owner and (first CTA)
// MMA issuer, warps 2..5 softmax / epilogue (thread = TMEM lane), warps 6..9 query staging
// and key rotation.  Every mbarrier wait is bounded (sm100.cuh); on a timeout all roles
// drain their in-flight work and exit.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kernels.h"
#include "rope.cuh"
#include "sm100.cuh"

namespace g4 {
namespace {

constexpr int kThreads = 320;
constexpr int kTileKeys = 64;        // keys per CTA per pair-tile
constexpr int kPairKeys = 128;       // keys per pair-tile
constexpr int kSlotBytes = 16384;    // 128 rows x 128 B: 64 keys x 64 dims of each half
constexpr int kBoxBytes = 8192;      // one TMA box: 64 keys x 64 dims
constexpr int kBarSM = 1;            // named barrier of the softmax warpgroup
constexpr int kBarRot = 2;           // named barrier of the rotation warpgroup
constexpr float kLazyMax = 8.0f;     // log2 units: headroom of the lazy reference max

// I8: the cache holds int8 codes with one fp32 scale per row.  A slot's codes (8 KB: 64-byte
// rows, 64-byte swizzle) land by TMA in the upper half of its 16 KB ring slot, and the
// rotation warps widen them in place into the bf16 layout the MMAs read (exact: |code| <=
// 127 needs 8 bits), so the ring keeps its depth.
constexpr int kCodeOff = kSlotBytes / 2;   // byte offset of a slot's int8 codes

template <int NH>
struct DecodeCfg {
    static constexpr int NS = 2 * NH;                // N of both MMAs (the pair's B rows)
    static constexpr int HH = NH / 2;                // heads finished by each half of the rows
    static constexpr int NSLOT = NH == 8 ? 11 : 10;  // ring slots of 16 KB
    static constexpr uint32_t TMEM_COLS = NH == 8 ? 128 : 256;   // 2 S^T + D/128 O^T blocks
};

// The MMA operands (ring, side buffers, q, P) start on 1024-byte boundaries: the hardware's
// 128-byte swizzle is a function of the shared-memory address, and the offsets computed
// here (sw128_offset) assume each tile starts on such a boundary.
template <int NH>
struct __align__(1024) DecodeSmem {
    using C = DecodeCfg<NH>;
    alignas(1024) uint8_t ring[C::NSLOT][kSlotBytes];
    uint8_t side[2][kSlotBytes];       // turned slot 0 of tiles j & 1 (values = pre-RoPE keys)
    // this CTA's half of the B operand of S^T per slot (NH rows: queries over the first
    // half of d in CTA 0, the second half in CTA 1), K-major, swizzled; q[4] (and, head_dim
    // 256, q[3]) are second copies of slot 0's (slot 1's) operand, which the relative
    // rotation rewrites per tile (tile j uses copy j & 1)
    uint8_t q[5][NH * 128];
    uint8_t p[2][NH * 128];            // this CTA's half of the B operand of O^T: its P^T
    float xs[2][64][C::HH];            // score halves handed to the other half's threads
    float theta[256];                  // base^(-2i/d) in fp32
    float2 base_cs[256];               // cos/sin of tile_start * theta_i
    float2 step_cs[256];               // cos/sin of 128 * theta_i: one pair-tile further
    float red[4][C::HH];               // cross-warp reductions
    float alpha[NH];                   // rescale factors of O^T
    float mfin[NH];                    // running max per head at the end of an item
    uint64_t full[C::NSLOT];           // this CTA's loads landed
    uint64_t empty[C::NSLOT];          // the pair's MMAs are done with the slot
    // per-tile barriers come in pairs (tile j uses [j & 1], phase (j >> 1) & 1): a waiter is
    // never more than one phase of a barrier behind (the rotation warps wait for S(j - 2)
    // before they arrive on rot_ready for tile j).  rot_ready and p_full live in the first
    // CTA and count one arrival from each CTA.
    uint64_t s_full[2], p_full[2], pv_done[2], rot_ready[2];
    uint64_t q_free, drain;            // once per item: all its scores done / teardown
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

struct Item {
    int s, g, b, k0, k1;   // segment, kv head, batch; positions [k0, k1) of the item's tiles
    int lo;                // first visible position in the item (>= k0)
};

// The pair that owns flat tile t: the largest p with p * total / n_pairs <= t.
__device__ __forceinline__ int pair_of_tile(const DecodeArgs& a, long long t) {
    return (int)(((t + 1) * a.n_pairs - 1) / a.total_tiles);
}

// This pair's flat tile range and the sequences it touches.
struct PairRange {
    long long t0, t1;
    int bg0, n_items;
};

__device__ __forceinline__ PairRange pair_range(const DecodeArgs& a, int pair) {
    PairRange r;
    r.t0 = (long long)pair * a.total_tiles / a.n_pairs;
    r.t1 = (long long)(pair + 1) * a.total_tiles / a.n_pairs;
    r.bg0 = (int)(r.t0 / a.tiles_per_seq);
    r.n_items = r.t1 > r.t0 ? (int)((r.t1 - 1) / a.tiles_per_seq) - r.bg0 + 1 : 0;
    return r;
}

// Item k of the pair: its part of sequence bg0 + k, and which segment of that sequence it is.
__device__ __forceinline__ Item item_of(const DecodeArgs& a, int pair, const PairRange& pr, int k) {
    Item r;
    const int bg = pr.bg0 + k;
    const long long s0 = (long long)bg * a.tiles_per_seq;
    const long long lo = pr.t0 > s0 ? pr.t0 : s0;
    const long long hi = pr.t1 < s0 + a.tiles_per_seq ? pr.t1 : s0 + a.tiles_per_seq;
    r.g = bg % a.Hkv;
    r.b = bg / a.Hkv;
    r.s = pair - pair_of_tile(a, s0);
    r.k0 = a.tile_base + (int)(lo - s0) * kPairKeys;
    r.k1 = min(a.L, a.tile_base + (int)(hi - s0) * kPairKeys);
    r.lo = max(r.k0, a.key_lo);
    return r;
}

// Four K-steps of one slot (64 dims of S^T, or 64 keys of O^T) as pair MMAs: the matrix
// descriptors advance by a fixed amount of their start-address field (16-byte units).
__device__ __forceinline__ void mma4_pair(uint32_t d, uint64_t a, uint32_t a_step, uint64_t b,
                                          uint32_t b_step, uint32_t idesc, uint32_t acc0) {
    mma_pair_f16(d, a, b, idesc, acc0);
    mma_pair_f16(d, a + a_step, b + b_step, idesc, 1u);
    mma_pair_f16(d, a + 2 * a_step, b + 2 * b_step, idesc, 1u);
    mma_pair_f16(d, a + 3 * a_step, b + 3 * b_step, idesc, 1u);
}

constexpr uint32_t kSlotDesc = kSlotBytes >> 4;   // one ring slot, in descriptor units


// The q operand copy that tile parity `odd` of rotated slot sb reads.
__host__ __device__ constexpr int q_copy(int sb, bool odd) { return odd ? (sb == 0 ? 4 : 3) : sb; }

// Sixteen int8 codes (one 16-byte piece of a code row) as sixteen bf16, exactly: each
// code c is biased to the byte u = c + 128, placed in the low mantissa bits of the fp32
// 2^23 (0x4B0000uu = 2^23 + u), and 2^23 + 128 is subtracted, which leaves c exact in fp32;
// its upper half is then c as a bf16 (c needs at most 8 significant bits).
__device__ __forceinline__ void widen_i8x16(uint4 in, uint4& lo, uint4& hi) {
    const uint32_t w[4] = {in.x ^ 0x80808080u, in.y ^ 0x80808080u, in.z ^ 0x80808080u,
                           in.w ^ 0x80808080u};
    uint32_t o[8];
    const float2 bias = make_float2(8388736.0f, 8388736.0f);   // 2^23 + 128
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f01 = sub_f2(make_float2(__uint_as_float(__byte_perm(w[i], 0x4B000000u, 0x7540)),
                                              __uint_as_float(__byte_perm(w[i], 0x4B000000u, 0x7541))),
                                  bias);
        const float2 f23 = sub_f2(make_float2(__uint_as_float(__byte_perm(w[i], 0x4B000000u, 0x7542)),
                                              __uint_as_float(__byte_perm(w[i], 0x4B000000u, 0x7543))),
                                  bias);
        o[2 * i] = __byte_perm(__float_as_uint(f01.x), __float_as_uint(f01.y), 0x7632);
        o[2 * i + 1] = __byte_perm(__float_as_uint(f23.x), __float_as_uint(f23.y), 0x7632);
    }
    lo = make_uint4(o[0], o[1], o[2], o[3]);
    hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// D: head dim; NH: query heads per KV head handled by the softmax (8 or 16, >= G);
// RS: slots turned by the relative rotation (0: absolute angles).  One slot (R <= 64, values
// not the rotated key) is the p-RoPE of the global layers; two (R <= 128, head_dim 256,
// separate values, at most 4 query heads per kv head) the full RoPE of the local layers.
// I8: an int8 cache (codes and per-row scales), widened to bf16 in shared memory.
template <int D, int NH, int RS, bool I8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ DecodeArgs a) {
    using C = DecodeCfg<NH>;
    constexpr bool REL = RS > 0;
    static_assert(RS < 2 || (D == 256 && NH == 8), "two relative slots: head_dim 256, NH 8");
    // (the host takes RS = 2 only for G <= 4)
    constexpr int NSB = D / 128;    // slots per tile and tensor
    constexpr int NS = C::NS, HH = C::HH, NSLOT = C::NSLOT;
    extern __shared__ uint8_t smem_raw[];
    DecodeSmem<NH>& sm = *reinterpret_cast<DecodeSmem<NH>*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const WaitCtl wc{a.wait_limit, a.status};
    volatile int* abort = &sm.abort;
    const int R = a.rope.R;
    const int nrot = (R + 63) / 64;   // slots holding rotated pairs: 0 .. nrot-1
    // K and V share the ring slots unless the values are a separate tensor (second pass).
    // Turned slots go to the side buffer when the values are the pre-RoPE keys.
    const bool sep_v = a.kv_is_k == 0;
    const bool side_rot = a.kv_is_k == 1;
    const uint32_t rank = cluster_rank();
    const int pair = blockIdx.x >> 1;
    const PairRange pr = pair_range(a, pair);
    const int n_items = pr.n_items;   // this pair's items
    // split cache: the key slots (already rotated) and one value slot for the rotated dims
    const bool split = a.split_cache != 0;
    const int slots_per_tile = sep_v ? 2 * NSB : (split ? NSB + 1 : NSB);

    if (threadIdx.x == 0) {
        for (int i = 0; i < NSLOT; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.s_full[i], 1);
            mbar_init(&sm.p_full[i], 2);
            mbar_init(&sm.pv_done[i], 1);
            mbar_init(&sm.rot_ready[i], 2);
        }
        mbar_init(&sm.q_free, 1);
        mbar_init(&sm.drain, 1);
        sm.abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc_pair(&sm.tmem_base, C::TMEM_COLS);
    if (warp >= 2 && warp < 6) {
        for (int i = threadIdx.x - 64; i < R; i += 128) {
            sm.theta[i] = (float)exp2(-(2.0 * (double)i / (double)D) * a.rope.log2_base);
            sm.step_cs[i] = rope_cos_sin((long long)kPairKeys, i, D, a.rope.log2_base);
        }
        for (int i = threadIdx.x - 64; i < (int)(sizeof(sm.p) / 16); i += 128)
            reinterpret_cast<uint4*>(&sm.p[0][0])[i] = make_uint4(0, 0, 0, 0);
        fence_proxy_async_smem();
    }
    tc_fence_before();
    cluster_sync();   // barriers of both CTAs initialised before any remote arrival
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t tm_o = tmem + 64;     // O^T: NSB blocks of NS columns

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            prefetch_tmap(&a.tm_k);
            if (sep_v) prefetch_tmap(&a.tm_v);
            if (split) prefetch_tmap(&a.tm_vside);
            uint32_t q = 0;   // ring slots filled so far
            for (int it = 0; it < n_items && !*abort; ++it) {
                const Item w = item_of(a, pair, pr, it);
                const int nt = ceil_div(w.k1 - w.k0, kPairKeys);
                for (int t = 0; t < nt && !*abort; ++t) {
                    const int kpos = w.k0 + t * kPairKeys + (int)rank * kTileKeys;
                    // cache row of this CTA's 64 keys (a ring holds position p at p % C; the
                    // tiles are 64-aligned and C a multiple of 64, so a box never wraps)
                    const int key = a.ring > 0 ? kpos % a.ring : kpos;
                    for (int pass = 0; pass < (sep_v ? 2 : 1) && !*abort; ++pass) {
                        const CUtensorMap* map = pass ? &a.tm_v : &a.tm_k;
                        for (int sb = 0; sb < NSB; ++sb) {
                            const int slot = q % NSLOT;
                            if (!mbar_wait(&sm.empty[slot], ((q / NSLOT) & 1) ^ 1, wc, abort))
                                break;
                            if constexpr (I8) {
                                // int8 codes: rows k (first half) then 64 + k (second half),
                                // 64 bytes each, in the slot's upper 8 KB
                                mbar_arrive_expect_tx(&sm.full[slot], kSlotBytes / 2);
                                tma_load_4d(sm.ring[slot] + kCodeOff, map, &sm.full[slot], sb * 64,
                                            w.g, key, w.b);
                                tma_load_4d(sm.ring[slot] + kCodeOff + kBoxBytes / 2, map,
                                            &sm.full[slot], D / 2 + sb * 64, w.g, key, w.b);
                            } else {
                                mbar_arrive_expect_tx(&sm.full[slot], kSlotBytes);
                                tma_load_4d(sm.ring[slot], map, &sm.full[slot], sb * 64, w.g, key,
                                            w.b);
                                tma_load_4d(sm.ring[slot] + kBoxBytes, map, &sm.full[slot],
                                            D / 2 + sb * 64, w.g, key, w.b);
                            }
                            ++q;
                        }
                    }
                    if (split && !*abort) {
                        // pre-RoPE values of the rotated dims: first-half dims in rows k,
                        // their partners (d/2 + ...) in rows 64 + k, like slot 0
                        const int slot = q % NSLOT;
                        if (mbar_wait(&sm.empty[slot], ((q / NSLOT) & 1) ^ 1, wc, abort)) {
                            mbar_arrive_expect_tx(&sm.full[slot], kSlotBytes);
                            tma_load_4d(sm.ring[slot], &a.tm_vside, &sm.full[slot], 0, w.g, key, w.b);
                            tma_load_4d(sm.ring[slot] + kBoxBytes, &a.tm_vside, &sm.full[slot], 64,
                                        w.g, key, w.b);
                            ++q;
                        }
                    }
                }
            }
            // before the CTA exits, every copy it started must have landed
            if (*abort) {
                const uint32_t first = q > (uint32_t)NSLOT ? q - NSLOT : 0;
                for (uint32_t k = first; k < q; ++k)
                    mbar_wait_drain(&sm.full[k % NSLOT], (k / NSLOT) & 1);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer (first CTA only)
        if (lane == 0 && rank == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(256, NS, false, false);
            constexpr uint32_t idesc_o = idesc_bf16_f32(256, NS, true, false);  // A = V^T
            constexpr uint32_t kQDesc = (NH * 128) >> 4;
            constexpr uint32_t kPDesc = (NH * 128) >> 4;
            const uint64_t d_ring_k = sdesc_sw128(smem_u32(sm.ring[0]), 16, 1024);
            const uint64_t d_ring_mn = sdesc_sw128(smem_u32(sm.ring[0]), kBoxBytes, 1024);
            const uint64_t d_side = sdesc_sw128(smem_u32(sm.side[0]), 16, 1024);
            const uint64_t d_q = sdesc_sw128(smem_u32(sm.q[0]), 16, 1024);
            const uint64_t d_p = sdesc_sw128(smem_u32(sm.p[0]), 16, 1024);
            // cursors of the score product (sc) and the value product (pc): item, tile
            // within it, global tile index and ring position
            struct Cursor {
                int it, t, nt;
                uint32_t g, q;
            };
            auto tiles_of = [&](int it) {
                if (it >= n_items) return 0;
                const Item w = item_of(a, pair, pr, it);
                return ceil_div(w.k1 - w.k0, kPairKeys);
            };
            auto advance = [&](Cursor& c) {
                c.q += slots_per_tile;
                ++c.g;
                if (++c.t >= c.nt) {
                    c.t = 0;
                    c.it += 1;
                    c.nt = tiles_of(c.it);
                }
            };
            Cursor sc{0, 0, tiles_of(0), 0u, 0u};
            Cursor pc = sc;
            unsigned long long t_idle = 0;
            long long polls = 0;
            while (pc.it < n_items) {
                bool did = false;
                if (pc.g < sc.g && mbar_test_wait(&sm.p_full[pc.g & 1], (pc.g >> 1) & 1)) {
                    // O^T += V^T . P^T for tile pc.g: both CTAs' P are ready
                    tc_fence_after();
                    const uint64_t pb = d_p + (pc.g & 1) * kPDesc;
                    const uint32_t qv = sep_v ? pc.q + NSB : pc.q;
#pragma unroll
                    for (int sb = 0; sb < NSB; ++sb) {
                        // split cache: slot 0's values come from the tile's extra slot
                        const uint32_t slot = (split && sb == 0 ? pc.q + NSB : qv + sb) % NSLOT;
                        // 16 keys per step = two 8-row groups of 1024 B
                        mma4_pair(tm_o + sb * NS, d_ring_mn + slot * kSlotDesc, 2048 >> 4, pb,
                                  32 >> 4, idesc_o, pc.t == 0 ? 0u : 1u);
                        mma_commit_pair(&sm.empty[slot]);
                    }
                    mma_commit_pair(&sm.pv_done[pc.g & 1]);
                    advance(pc);
                    did = true;
                } else if (sc.it < n_items && sc.g < pc.g + 2 &&
                           mbar_test_wait(&sm.rot_ready[sc.g & 1], (sc.g >> 1) & 1)) {
                    // S^T for tile sc.g: both CTAs have its slots (turned) and, at the
                    // start of an item, its queries; its S^T buffer was read by the softmax
                    // of tile sc.g - 2, whose value product has been issued
                    tc_fence_after();
                    const uint32_t tm_s = tmem + (sc.g & 1) * 32;
                    uint32_t acc = 0;
#pragma unroll
                    for (int sb = 0; sb < NSB; ++sb) {
                        const uint32_t slot = (sc.q + sb) % NSLOT;
                        const bool rot = sb < nrot;
                        const uint64_t ad = (rot && side_rot) ? d_side + (sc.g & 1) * kSlotDesc
                                                              : d_ring_k + slot * kSlotDesc;
                        const uint64_t bd =
                            d_q + (REL && sb < nrot ? q_copy(sb, sc.g & 1) : sb) * kQDesc;
                        mma4_pair(tm_s, ad, 32 >> 4, bd, 32 >> 4, idesc_s, acc);
                        acc = 1;
                        // score slots of a separate-value layer (and the rotated key slot of a
                        // split cache) go back right away
                        if (sep_v || (split && sb == 0)) mma_commit_pair(&sm.empty[slot]);
                    }
                    mma_commit_pair(&sm.s_full[sc.g & 1]);
                    if (sc.t == sc.nt - 1) mma_commit_pair(&sm.q_free);   // q may be restaged
                    advance(sc);
                    did = true;
                }
                if (did) {
                    polls = 0;
                    continue;
                }
                // nothing ready: bounded polling, like every other wait
                if (*abort) break;
                if ((++polls & 63) == 0) {
                    const unsigned long long now = global_ns();
                    if (polls == 64) t_idle = now;
                    if (polls >= a.wait_limit || now - t_idle > kWaitTimeoutNs) {
                        atomicExch(a.status, (int)G4ATTN_ERR_TIMEOUT);
                        *abort = 1;
                        break;
                    }
                }
            }
            // all issued MMAs must finish before either CTA frees its tensor memory
            mma_commit_pair(&sm.drain);
            mbar_wait_drain(&sm.drain, 0);
        }
    } else if (warp < 6) {
        // ------------------------------------------------- softmax / epilogue (warps 2..5)
        const int t128 = threadIdx.x - 64;            // 0..127
        const int quarter = warp & 3;                 // TMEM lane quarter of this warp
        const int row = quarter * 32 + lane;          // TMEM lane: (half, key) or O^T dim row
        const int hf = row >> 6;                      // half of d whose score rows this is
        const int key = row & 63;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const int G = a.G;
        const float c2 = a.scale_log2;
        const uint32_t ocol = rank * NH;              // this CTA's columns of O^T
        uint32_t gt = 0;
        bool ok = true;
        // the value product of tile j is complete (a no-op for j < 0)
        auto wait_pv = [&](int j) -> bool {
            const bool good = j < 0 || mbar_wait(&sm.pv_done[j & 1], (j >> 1) & 1, wc, abort);
            return group_all(good, kBarSM, 128);
        };
        // I8: the fp32 scales of this thread's key in tile t of item w (key, then value
        // scale; the value scale is the key's when the values are the keys).  They are
        // fetched one tile ahead of their use.
        auto scale_of = [&](const Item& w, int t) -> float2 {
            float2 r = make_float2(0.f, 0.f);
            if constexpr (I8) {
                const int pos = w.k0 + t * kPairKeys + (int)rank * kTileKeys + key;
                if (pos < w.k1) {
                    const int rows = a.ring > 0 ? a.ring : a.L;
                    const size_t idx =
                        ((size_t)w.b * rows + (a.ring > 0 ? pos % a.ring : pos)) * a.Hkv + w.g;
                    r.x = __ldg(a.kscale + idx);
                    r.y = sep_v ? __ldg(a.vscale + idx) : r.x;
                }
            }
            return r;
        };
        float2 scl_next = make_float2(0.f, 0.f);
        if (I8 && n_items > 0) scl_next = scale_of(item_of(a, pair, pr, 0), 0);
        for (int it = 0; it < n_items && ok; ++it) {
            const Item w = item_of(a, pair, pr, it);
            const int nt = ceil_div(w.k1 - w.k0, kPairKeys);
            float m_run[HH], l_part[HH];
#pragma unroll
            for (int j = 0; j < HH; ++j) {
                m_run[j] = -INFINITY;
                l_part[j] = 0.f;
            }
            for (int t = 0; t < nt; ++t, ++gt) {
                const float2 scl = scl_next;
                if constexpr (I8) {
                    if (t + 1 < nt) scl_next = scale_of(w, t + 1);
                    else if (it + 1 < n_items) scl_next = scale_of(item_of(a, pair, pr, it + 1), 0);
                }
                ok = group_all(mbar_wait(&sm.s_full[gt & 1], (gt >> 1) & 1, wc, abort), kBarSM,
                               128);
                if (!ok) break;
                tc_fence_after();
                const int key0 = w.k0 + t * kPairKeys + (int)rank * kTileKeys;
                float sp[NH];
                if constexpr (NH == 8) tmem_ld8(tmem + (gt & 1) * 32 + hf * NH + lane_off, sp);
                else tmem_ld16(tmem + (gt & 1) * 32 + hf * NH + lane_off, sp);
                tmem_ld_wait();
                // hand the heads the other half finishes to it, take ours from it
#pragma unroll
                for (int j = 0; j < HH; ++j) sm.xs[hf ^ 1][key][j] = hf ? sp[j] : sp[HH + j];
                group_sync(kBarSM, 128);
                const bool valid = key0 + key < w.k1 && key0 + key >= w.lo;
                // int8 cache: the key's score is its scale times the product with its codes
                const float c2k = I8 ? c2 * scl.x : c2;
                float x[HH];
                bool big = false;
#pragma unroll
                for (int j = 0; j < HH; ++j) {
                    const int h = hf * HH + j;
                    const float sc = (hf ? sp[HH + j] : sp[j]) + sm.xs[hf][key][j];
                    x[j] = (valid && h < G) ? sc * c2k : -INFINITY;
                    big |= x[j] > m_run[j] + kLazyMax;
                }
                // lazy reference max: only when some score of the tile exceeds the running
                // reference by more than 2^8 (and on the first tile) do the warps reduce
                const bool fast = (t > 0) && group_all(!big, kBarSM, 128);
                float alpha[HH];
#pragma unroll
                for (int j = 0; j < HH; ++j) alpha[j] = 1.f;
                if (!fast) {
#pragma unroll
                    for (int j = 0; j < HH; ++j) {
                        float mt = x[j];
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1)
                            mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
                        if (lane == 0) sm.red[quarter][j] = mt;
                    }
                    group_sync(kBarSM, 128);
                    bool resc = false;
#pragma unroll
                    for (int j = 0; j < HH; ++j) {
                        const float tmax = fmaxf(sm.red[2 * hf][j], sm.red[2 * hf + 1][j]);
                        if (tmax > m_run[j] + kLazyMax ||
                            (m_run[j] == -INFINITY && tmax != -INFINITY)) {
                            alpha[j] = (m_run[j] == -INFINITY) ? 0.f : exp2f(m_run[j] - tmax);
                            m_run[j] = tmax;
                            resc |= t > 0;
                        }
                    }
                    if (lane == 0 && (quarter & 1) == 0)
#pragma unroll
                        for (int j = 0; j < HH; ++j) sm.alpha[hf * HH + j] = alpha[j];
                    const bool rescale = !group_all(!resc, kBarSM, 128);  // also orders alpha
                    // rescale this CTA's O^T columns (thread = dim row, column = head) once
                    // the value product of the tile before is complete; the next one waits
                    // for this tile's P
                    if (rescale) {
                        ok = wait_pv((int)gt - 1);
                        if (!ok) break;
                        tc_fence_after();
                        for (int sb = 0; sb < NSB; ++sb) {
                            float o[NH];
                            if constexpr (NH == 8) tmem_ld8(tm_o + sb * NS + ocol + lane_off, o);
                            else tmem_ld16(tm_o + sb * NS + ocol + lane_off, o);
                            tmem_ld_wait();
#pragma unroll
                            for (int h = 0; h < NH; ++h) o[h] *= sm.alpha[h];
                            if constexpr (NH == 8) tmem_st8(tm_o + sb * NS + ocol + lane_off, o);
                            else tmem_st16(tm_o + sb * NS + ocol + lane_off, o);
                        }
                        tmem_st_wait();
                    }
                }
                // P^T into p[gt & 1] once the value product that last read it is complete
                ok = wait_pv((int)gt - 2);
                if (!ok) break;
                {
                    uint8_t* pb = sm.p[gt & 1];
#pragma unroll
                    for (int j = 0; j < HH; ++j) {
                        const float p = (x[j] == -INFINITY) ? 0.f : ex2_approx(x[j] - m_run[j]);
                        // int8 cache: the value operand holds the codes, so the weight carries
                        // the value's scale (bf16 keeps fp32's exponent range)
                        const __nv_bfloat16 pr = __float2bfloat16_rn(I8 ? p * scl.y : p);
                        // the running sum uses the rounded weight the MMA sees (int8: the
                        // unrounded weight, the scale being folded into the rounded one)
                        l_part[j] = l_part[j] * alpha[j] + (I8 ? p : __bfloat162float(pr));
                        *reinterpret_cast<__nv_bfloat16*>(pb + sw128_offset(hf * HH + j, key)) = pr;
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                group_sync(kBarSM, 128);
                if (t128 == 0) {
                    if (rank == 0) mbar_arrive(&sm.p_full[gt & 1]);
                    else mbar_arrive_remote(&sm.p_full[gt & 1], 0);
                }
            }
            if (!ok) break;
            // ---- item epilogue: this CTA's partial O^T, running max and sum
            ok = wait_pv((int)gt - 1);
            if (!ok) break;
            tc_fence_after();
            const size_t obase =
                ((size_t)(2 * w.s + (int)rank) * a.B + w.b) * a.Hq + (size_t)w.g * G;
            const int dim0 = (row < 64) ? row : D / 2 + (row - 64);
            for (int sb = 0; sb < NSB; ++sb) {
                float o[NH];
                if constexpr (NH == 8) tmem_ld8(tm_o + sb * NS + ocol + lane_off, o);
                else tmem_ld16(tm_o + sb * NS + ocol + lane_off, o);
                tmem_ld_wait();
#pragma unroll
                for (int h = 0; h < NH; ++h)
                    if (h < G) a.part_o[(obase + h) * D + sb * 64 + dim0] = o[h];
            }
#pragma unroll
            for (int j = 0; j < HH; ++j) {
                float l = l_part[j];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
                if (lane == 0) sm.red[quarter][j] = l;
                if (lane == 0 && (quarter & 1) == 0) sm.mfin[hf * HH + j] = m_run[j];
            }
            group_sync(kBarSM, 128);
            if (t128 < G) {
                const int h = t128, hh = h / HH, j = h % HH;
                a.part_ml[(obase + h) * 2 + 0] = sm.mfin[h];
                a.part_ml[(obase + h) * 2 + 1] = sm.red[2 * hh][j] + sm.red[2 * hh + 1][j];
            }
            tc_fence_before();
            group_sync(kBarSM, 128);   // red[] and O^T are reused by the next item
        }
    } else {
        // ---------------------------------------- query staging / key rotation (warps 6..9)
        const int t128 = threadIdx.x - 192;           // 0..127
        const int rk = t128 & 63;                     // key row of this thread
        const int cp = t128 >> 6;                     // columns [32 cp, 32 cp + 32)
        const int G = a.G;
        constexpr int QV = NH * NSB * 8 / 128;        // 16-byte pieces of q staged per thread
        // REL: heads cp, cp + 2, ... of pair rk (two turned slots: at most 4 query heads per
        // kv head, which keeps the per-thread state within the register budget)
        constexpr int QH = RS == 2 ? 2 : NH / 2;
        constexpr int NRS = REL ? RS : 1;             // REL: rotated slots served
        // Relative rotation (REL): key row rk of this CTA sits at angle (64 rank + rk) theta_i
        // from the start of the pair-tile, so its (cos, sin) are fixed per thread; the start
        // angle goes onto the query, which both CTAs' keys share in the pair MMA:
        // q' = R(-key0 theta) q, and q' . R((64 rank + rk) theta) k equals
        // q . R((key0 + 64 rank + rk) theta) k.  rc / rs hold cos / sin of the column pairs
        // (2m, 2m + 1) of this thread (rotated slot r: pairs 64 r + 32 cp + 2m) as packed bf16
        // pairs: the turn runs on bf16x2 multiply-adds, 4 per pair of columns (fp32 math with
        // its unpacking and repacking took 11 and sat on the per-tile chain, 6% of the decode
        // rate).  With 10 warps a thread gets at most 168 registers: with two slots -sin is
        // formed per use (5 operations) rather than held, and the query pairs stay packed.
        __nv_bfloat162 rc[REL ? 16 * NRS : 1], rs[REL ? 16 * NRS : 1];
        __nv_bfloat162 rn[NRS == 1 && REL ? 16 : 1];  // -sin (one slot)
        __nv_bfloat162 qxy[NRS][REL ? QH : 1];       // REL: pair 64 r + rk of q (x, y)
        float2 bcs[NRS], stp[NRS];                   // REL: cos/sin of pair start * theta and
                                                     // of 128 * theta, pair 64 r + rk
        // the next item's queries and start angles, fetched one tile ahead of their use
        uint4 qpre[QV];
        __nv_bfloat162 qxyp[NRS][REL ? QH : 1];
        float2 bpre[2];
        auto prefetch = [&](int it2) {
            const Item w2 = item_of(a, pair, pr, it2);
            const long long k0r = (long long)w2.k0 + (long long)rank * kTileKeys;
            const uint16_t* qg = a.q + ((size_t)w2.b * a.Hq + (size_t)w2.g * G) * D;
#pragma unroll
            for (int j = 0; j < QV; ++j) {
                // this CTA's B rows: head h over dims (rank * d/2 + 64 sb + [0, 64))
                const int e = t128 + 128 * j;
                const int h = e / (NSB * 8), sb = (e / 8) % NSB, c8 = e % 8;
                qpre[j] = make_uint4(0, 0, 0, 0);
                if (h < G)
                    qpre[j] = *reinterpret_cast<const uint4*>(
                        qg + (size_t)h * D + rank * (D / 2) + sb * 64 + c8 * 8);
            }
            if constexpr (REL) {
#pragma unroll
                for (int r = 0; r < NRS; ++r) {
                    const int i = 64 * r + rk;   // this thread's pair in rotated slot r
#pragma unroll
                    for (int j = 0; j < QH; ++j) {
                        const int h = cp + 2 * j;
                        const bool on = h < G && i < R;
                        const __nv_bfloat16 z = __float2bfloat16_rn(0.f);
                        qxyp[r][j] = __halves2bfloat162(
                            on ? *reinterpret_cast<const __nv_bfloat16*>(qg + (size_t)h * D + i) : z,
                            on ? *reinterpret_cast<const __nv_bfloat16*>(qg + (size_t)h * D + D / 2 + i)
                               : z);
                    }
                    // q' turns by the start of the pair-tile (shared by both CTAs)
                    bpre[r] = i < R ? rope_cos_sin((long long)w2.k0, i, D, a.rope.log2_base)
                                    : make_float2(1.f, 0.f);
                }
            } else {
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int i = t128 + 128 * j;
                    bpre[j] = i < R ? rope_cos_sin(k0r, i, D, a.rope.log2_base)
                                    : make_float2(1.f, 0.f);
                }
            }
        };
        if (n_items > 0) prefetch(0);   // the loads fly while the constants below are computed
        if constexpr (REL) {
            // angles (64 rank + rk) theta_i <= 127 rad: reduced by the nearest multiple of 2 pi,
            // then the fast intrinsic on [-pi, pi] (the accurate sincosf took 10 us per CTA here)
            const float pos = (float)((int)rank * kTileKeys + rk);
            auto turn = [&](int i, float& sn, float& cs) {
                float x = pos * sm.theta[i];
                x = fmaf(-6.2831853f, rintf(x * 0.15915494f), x);
                __sincosf(x, &sn, &cs);
            };
#pragma unroll
            for (int m = 0; m < 16 * NRS; ++m) {
                const int i0 = 64 * (m / 16) + 32 * cp + 2 * (m % 16);
                float s0 = 0.f, c0 = 1.f, s1 = 0.f, c1 = 1.f;
                if (i0 < R) turn(i0, s0, c0);
                if (i0 + 1 < R) turn(i0 + 1, s1, c1);
                rc[m] = __floats2bfloat162_rn(c0, c1);
                rs[m] = __floats2bfloat162_rn(s0, s1);
                if constexpr (NRS == 1) rn[m] = __floats2bfloat162_rn(-s0, -s1);
            }
        }
#pragma unroll
        for (int r = 0; r < NRS; ++r) {
            bcs[r] = make_float2(1.f, 0.f);
            stp[r] = (REL && 64 * r + rk < R) ? sm.step_cs[64 * r + rk] : make_float2(1.f, 0.f);
        }
        uint32_t q = 0, gt = 0, item_n = 0;
        bool ok = true;
        for (int it = 0; it < n_items && ok; ++it, ++item_n) {
            const Item w = item_of(a, pair, pr, it);
            const int nt = ceil_div(w.k1 - w.k0, kPairKeys);
            for (int t = 0; t < nt; ++t, ++gt) {
                const uint32_t qk = q;
                q += slots_per_tile;
                // before rewriting the B operands: the first tile of an item needs every
                // score product of the previous item complete (it restages all of q), a
                // later tile only the one that last read its side buffer and q copy (gt - 2).
                // The wait on S(gt - 2) also keeps this role less than two tiles ahead of
                // the issuer on the paired rot_ready barriers, whatever the ring depth (a
                // head_dim 256 keys-as-values layer has 2 slots per tile, 5.5 tiles of ring)
                if (t == 0 && item_n > 0) {
                    ok = group_all(mbar_wait(&sm.q_free, (item_n - 1) & 1, wc, abort), kBarRot,
                                   128);
                } else if (t > 0 && gt > 1) {
                    ok = group_all(mbar_wait(&sm.s_full[gt & 1], ((gt - 2) >> 1) & 1, wc, abort),
                                   kBarRot, 128);
                }
                if (!ok) break;
                if (t == 0) {
                    // stage this CTA's half of the queries' B operand; the operands of the
                    // relatively rotated slots go to both of their copies
#pragma unroll
                    for (int j = 0; j < QV; ++j) {
                        const int e = t128 + 128 * j;
                        const int h = e / (NSB * 8), sb = (e / 8) % NSB, c8 = e % 8;
                        *reinterpret_cast<uint4*>(sm.q[sb] + sw128_offset(h, c8 * 8)) = qpre[j];
                        if (REL && sb < NRS)
                            *reinterpret_cast<uint4*>(sm.q[q_copy(sb, true)] +
                                                      sw128_offset(h, c8 * 8)) = qpre[j];
                    }
                    if constexpr (REL) {
#pragma unroll
                        for (int r = 0; r < NRS; ++r) {
#pragma unroll
                            for (int j = 0; j < QH; ++j) qxy[r][j] = qxyp[r][j];
                            bcs[r] = bpre[r];
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 2; ++j)
                            if (t128 + 128 * j < R) sm.base_cs[t128 + 128 * j] = bpre[j];
                    }
                }
                // fetch the next item's queries now: the loads fly during this tile's work
                if (t == nt - 1 && it + 1 < n_items) prefetch(it + 1);
                bool got = true;
                if constexpr (I8) {
                    // widen the tile's slots in place: thread (rk, cp) takes rows rk and 64 + rk
                    // (the two halves of key rk), dims [32 cp, 32 cp + 32) of the slot.  Code row
                    // r sits at kCodeOff + 64 r with the 64-byte swizzle (16-byte piece c at
                    // piece c ^ ((r >> 1) & 3)), conflict-free for 8 consecutive rows.  The bf16
                    // rows 64..127 overwrite the codes, so every thread reads its codes of the
                    // slot before any thread writes.
                    for (int k = 0; k < slots_per_tile && got; ++k) {
                        const uint32_t sq = qk + k;
                        got = mbar_wait(&sm.full[sq % NSLOT], (sq / NSLOT) & 1, wc, abort);
                        uint8_t* slotp = sm.ring[sq % NSLOT];
                        uint4 w8[2][2];
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int row = 64 * h + rk;
#pragma unroll
                            for (int c = 0; c < 2; ++c) {
                                const int piece = 2 * cp + c;   // dims [16 piece, 16 piece + 16)
                                w8[h][c] = got ? *reinterpret_cast<const uint4*>(
                                                     slotp + kCodeOff + row * 64 +
                                                     ((piece ^ ((row >> 1) & 3)) << 4))
                                               : make_uint4(0, 0, 0, 0);
                            }
                        }
                        if (!group_all(got, kBarRot, 128)) {
                            got = false;
                            break;
                        }
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int row = 64 * h + rk;
#pragma unroll
                            for (int c = 0; c < 2; ++c) {
                                const int piece = 2 * cp + c;
                                uint4 lo, hi;
                                widen_i8x16(w8[h][c], lo, hi);
                                *reinterpret_cast<uint4*>(slotp + sw128_offset(row, 16 * piece)) = lo;
                                *reinterpret_cast<uint4*>(slotp + sw128_offset(row, 16 * piece + 8)) = hi;
                            }
                        }
                    }
                    // every widened row is in place before the turns below read them
                    got = group_all(got, kBarRot, 128);
                } else {
                    // the slots with rotated pairs first: they are turned while the rest land
                    // (the relative rotation turns its first slot while its second one lands)
                    const int nfirst = REL ? (nrot > 0 ? 1 : 0) : nrot;
                    for (int k = 0; k < nfirst && got; ++k)
                        got = mbar_wait(&sm.full[(qk + k) % NSLOT], ((qk + k) / NSLOT) & 1, wc,
                                        abort);
                }
                if (R > 0) {
                    // start angle of this CTA's tile: exact (fp64-reduced) at the first tile
                    // of an item, then advanced by one pair-tile (128 keys) per step
                    if constexpr (REL) {
                        if (t > 0) {
#pragma unroll
                            for (int r = 0; r < NRS; ++r)
                                bcs[r] = make_float2(bcs[r].x * stp[r].x - bcs[r].y * stp[r].y,
                                                     bcs[r].x * stp[r].y + bcs[r].y * stp[r].x);
                        }
                    } else if (t > 0) {
                        for (int i = t128; i < R; i += 128) {
                            const float2 b0 = sm.base_cs[i], st = sm.step_cs[i];
                            sm.base_cs[i] = make_float2(b0.x * st.x - b0.y * st.y,
                                                        b0.x * st.y + b0.y * st.x);
                        }
                    }
                }
                ok = group_all(got, kBarRot, 128);   // also orders base_cs writes
                if (!ok) break;
                if (R > 0) {
                    if constexpr (REL) {
#pragma unroll
                        for (int r = 0; r < NRS; ++r) {
                            if (r >= nrot) break;
                            if (!I8 && r > 0) {   // the next rotated slot, landed while slot r-1 turned
                                const uint32_t k = qk + r;
                                got = group_all(mbar_wait(&sm.full[k % NSLOT], (k / NSLOT) & 1,
                                                          wc, abort),
                                                kBarRot, 128);
                                if (!got) break;
                            }
                            // this CTA's half of q' = R(-key0 theta) q on pair 64 r + rk, key0
                            // the start of the pair-tile (first-half dim in CTA 0, second-half
                            // dim in CTA 1), into copy gt & 1 of rotated slot r's operand
                            uint8_t* qd = sm.q[q_copy(r, gt & 1)];
                            if (64 * r + rk < R) {
#pragma unroll
                                for (int j = 0; j < QH; ++j) {
                                    const int h = cp + 2 * j;
                                    if (h < G) {
                                        const float2 b = bcs[r];
                                        const float2 xy = __bfloat1622float2(qxy[r][j]);
                                        const float v = rank == 0 ? xy.x * b.x + xy.y * b.y
                                                                  : xy.y * b.x - xy.x * b.y;
                                        *reinterpret_cast<__nv_bfloat16*>(qd + sw128_offset(h, rk)) =
                                            __float2bfloat16_rn(v);
                                    }
                                }
                            }
                            // keys: R(rk theta) on the rotated pairs of row rk (dims in row rk,
                            // their partners in row 64 + rk of slot r)
                            uint8_t* src = sm.ring[(qk + r) % NSLOT];
                            uint8_t* dst = side_rot ? sm.side[gt & 1] : src;
#pragma unroll
                            for (int g8 = 0; g8 < 4; ++g8) {
                                const int col = 32 * cp + 8 * g8;
                                const bool rotg = 64 * r + col < R;
                                if (!side_rot && !rotg) continue;   // in place: nothing to copy
                                const uint32_t o1 = sw128_offset(rk, col);
                                const uint32_t o2 = sw128_offset(64 + rk, col);
                                uint4 x1 = *reinterpret_cast<const uint4*>(src + o1);
                                uint4 x2 = *reinterpret_cast<const uint4*>(src + o2);
                                if (rotg) {
                                    // pairs whose cos/sin are (1, 0) turn into themselves, so
                                    // the columns at or past R need no special case
                                    uint32_t* w1 = &x1.x;
                                    uint32_t* w2 = &x2.x;
#pragma unroll
                                    for (int m = 0; m < 4; ++m) {
                                        const __nv_bfloat162 u = *reinterpret_cast<const __nv_bfloat162*>(&w1[m]);
                                        const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&w2[m]);
                                        const int i = 16 * r + 4 * g8 + m;
                                        __nv_bfloat162 u2;
                                        if constexpr (NRS == 1) u2 = __hfma2(u, rc[i], __hmul2(v, rn[i]));
                                        else u2 = __hfma2(u, rc[i], __hneg2(__hmul2(v, rs[i])));
                                        const __nv_bfloat162 v2 = __hfma2(u, rs[i], __hmul2(v, rc[i]));
                                        w1[m] = *reinterpret_cast<const uint32_t*>(&u2);
                                        w2[m] = *reinterpret_cast<const uint32_t*>(&v2);
                                    }
                                }
                                *reinterpret_cast<uint4*>(dst + o1) = x1;
                                *reinterpret_cast<uint4*>(dst + o2) = x2;
                            }
                        }
                    } else {
                        // absolute angles: angle(key0 + rk) = angle(key0) + rk * theta_i
                        const float fr = (float)rk;
                        for (int sb = 0; sb < nrot; ++sb) {
                            uint8_t* src = sm.ring[(qk + sb) % NSLOT];
                            uint8_t* dst = side_rot ? sm.side[gt & 1] : src;
                            for (int g8 = 0; g8 < 4; ++g8) {
                                const int col = 32 * cp + 8 * g8;
                                const uint32_t o1 = sw128_offset(rk, col);
                                const uint32_t o2 = sw128_offset(64 + rk, col);
                                uint4 x1 = *reinterpret_cast<const uint4*>(src + o1);
                                uint4 x2 = *reinterpret_cast<const uint4*>(src + o2);
                                __nv_bfloat162* h1 = reinterpret_cast<__nv_bfloat162*>(&x1);
                                __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&x2);
#pragma unroll
                                for (int e2 = 0; e2 < 4; ++e2) {
                                    const float2 u = __bfloat1622float2(h1[e2]);
                                    const float2 v = __bfloat1622float2(h2[e2]);
                                    float uo[2] = {u.x, u.y}, vo[2] = {v.x, v.y};
#pragma unroll
                                    for (int e = 0; e < 2; ++e) {
                                        const int i = sb * 64 + col + e2 * 2 + e;
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
                                *reinterpret_cast<uint4*>(dst + o1) = x1;
                                *reinterpret_cast<uint4*>(dst + o2) = x2;
                            }
                        }
                    }
                }
                // every slot of the tile has landed (the MMA issuer relies on this barrier)
                for (int k = nrot; !I8 && k < slots_per_tile && got; ++k)
                    got = mbar_wait(&sm.full[(qk + k) % NSLOT], ((qk + k) / NSLOT) & 1, wc, abort);
                // the tile's operands are in place: one arrival per CTA on the first CTA
                fence_proxy_async_smem();
                ok = group_all(got, kBarRot, 128);
                if (!ok) break;
                if (t128 == 0) {
                    if (rank == 0) mbar_arrive(&sm.rot_ready[gt & 1]);
                    else mbar_arrive_remote(&sm.rot_ready[gt & 1], 0);
                }
            }
        }
    }

    // -------------------------------------------------------------------- teardown
    __syncthreads();
    // the first CTA's MMAs read both CTAs' shared memory: neither leaves before they are
    // done (the issuer waited for its drain commit above)
    tc_fence_before();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, C::TMEM_COLS);
    }
}

// Merge the partials of one (b, h): two per segment, one from each CTA of the pair,
//   out = sum_p 2^(m_p - M) O_p / sum_p 2^(m_p - M) l_p,   M = max_p m_p (log2 units).
// Block (b h, 128-dim chunk), thread = one dim.
constexpr int kCombineThreads = 128;
constexpr int kMaxParts = 1024;   // sanity bound on the partials per sequence

__global__ void __launch_bounds__(kCombineThreads)
    decode_combine_kernel(const __grid_constant__ DecodeArgs a) {
    // launched as a programmatic dependent of the decode kernel: its blocks may start while
    // the decode's last CTAs finish; the partials are read only after the decode grid has
    // completed and its writes are visible
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int bh = blockIdx.x;   // b * Hq + h
    const int tid = threadIdx.x;
    const size_t stride = (size_t)a.B * a.Hq;
    // the segments of this (b, h)'s sequence: one per pair whose tiles it spans
    int nseg = 0;
    if (a.total_tiles > 0) {
        const long long s0 = (long long)(bh / a.Hq * a.Hkv + (bh % a.Hq) / a.G) * a.tiles_per_seq;
        nseg = pair_of_tile(a, s0 + a.tiles_per_seq - 1) - pair_of_tile(a, s0) + 1;
    }
    const int parts = 2 * nseg;
    // a sequence has a few parts: every thread reads their (max, sum) itself (the same
    // addresses across the block) and forms the weights, with no block-wide reduction
    const float2* ml = reinterpret_cast<const float2*>(a.part_ml) + bh;
    float M = -INFINITY;
    for (int s = 0; s < parts; ++s) M = fmaxf(M, ml[s * stride].x);
    const int c = blockIdx.y * kCombineThreads + tid;
    const float* po = a.part_o + (size_t)bh * a.d + c;
    const size_t ps = stride * a.d;
    float dsum = 0.f, acc = 0.f;
    for (int s = 0; s < parts; ++s) {
        const float2 p = ml[s * stride];
        const float w = (p.x == -INFINITY) ? 0.f : exp2f(p.x - M);
        dsum += w * p.y;
        if (c < a.d) acc += w * po[s * ps];
    }
    const float inv = dsum > 0.f ? 1.f / dsum : 0.f;
    if (c < a.d) a.out[(size_t)bh * a.d + c] = __bfloat16_as_ushort(__float2bfloat16_rn(acc * inv));
    if (tid == 0 && blockIdx.y == 0 && a.lse)
        a.lse[bh] = dsum > 0.f ? (M + log2f(dsum)) * 0.6931471805599453f : -INFINITY;
}

template <int D, int NH, int RS, bool I8>
cudaError_t run_decode(const DecodeArgs& a, int grid, cudaStream_t stream) {
    using Smem = DecodeSmem<NH>;
    const size_t smem = sizeof(Smem) + 1024;
    static_assert(sizeof(Smem) + 1024 <= 227 * 1024, "decode shared memory");
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, NH, RS, I8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    decode_kernel<D, NH, RS, I8><<<grid, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

template <int D, bool I8>
cudaError_t dispatch_decode(const DecodeArgs& a, int grid, cudaStream_t stream) {
    // relative rotation: a side buffer holds one turned slot per tile, so the pre-RoPE-value
    // layers (kv_is_k 1) take it for one rotated slot only
    const bool rel1 = a.kv_is_k != 2 && a.rope.R <= 64;
    if (a.G <= 8) {
        if (rel1) return run_decode<D, 8, 1, I8>(a, grid, stream);
        if constexpr (D == 256)
            if (a.kv_is_k == 0 && a.rope.R <= 128 && a.G <= 4)
                return run_decode<D, 8, 2, I8>(a, grid, stream);
        return run_decode<D, 8, 0, I8>(a, grid, stream);
    }
    if constexpr (I8) return cudaErrorInvalidValue;   // int8 caches: at most 8 query heads per kv head
    else return rel1 ? run_decode<D, 16, 1, false>(a, grid, stream)
                     : run_decode<D, 16, 0, false>(a, grid, stream);
}

}  // namespace

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

// The array's device address in the current device's context.  The caller (api.cu) calls
// this at set-up, once per device and context, with that device current, and caches the
// result with the context's id.
cudaError_t decode_scratch_ptr(void** out) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    *out = p;
    return cudaSuccess;
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
    if (2 * a.splits > kMaxParts) return cudaErrorInvalidValue;
    if (a.n_pairs > 0 && a.total_tiles > 0) {
        // one cluster of two CTAs per pair of the stream-K split
        const int grid = 2 * a.n_pairs;
        cudaError_t e;
        if (a.int8) {
            if (a.split_cache || a.G > 8) return cudaErrorInvalidValue;
            e = a.d == 512 ? dispatch_decode<512, true>(a, grid, stream)
                : a.d == 256 ? dispatch_decode<256, true>(a, grid, stream)
                             : cudaErrorInvalidValue;
        } else {
            e = a.d == 512 ? dispatch_decode<512, false>(a, grid, stream)
                : a.d == 256 ? dispatch_decode<256, false>(a, grid, stream)
                             : cudaErrorInvalidValue;
        }
        if (e != cudaSuccess) return e;
    }
    if (a.B * a.Hq > 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(a.B * a.Hq, (a.d + kCombineThreads - 1) / kCombineThreads);
        cfg.blockDim = dim3(kCombineThreads);
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        const cudaError_t e = cudaLaunchKernelEx(&cfg, decode_combine_kernel, a);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

}  // namespace g4

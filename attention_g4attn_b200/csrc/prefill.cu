// prefill.cu -- flash-attention prefill for the Gemma-4-style layer on tcgen05 / TMEM,
// run by pairs of CTAs (a 2-CTA cluster issuing cta_group::2 MMAs).
//
// Each CTA owns one 128-row tile of packed query rows: row r is token m0 + r / G of query
// head g*G + r % G, so the G query heads that share kv head g sit in the MMA M dimension
// (GQA; explainer "GQA": 8:1 in global layers, 2:1 in local layers).  The two CTAs of a
// pair hold consecutive row tiles of the same (batch, kv head) and share every key tile:
// one MMA of M = 256 covers both row tiles while each CTA stages only half of the key
// tile (S: 64 of the 128 keys; P.V: 128 of the 256 value dims of an N=256 block), which
// halves the shared-memory and L2 traffic per CTA.
//   prologue  raw q rows -> RMSNorm * gamma -> RoPE / p-RoPE -> fp16, 128-byte-swizzled
//             K-major tile in shared memory (report section 2: QKNorm, p-RoPE).  The key
//             pre-pass writes the normalised keys (pre-RoPE and rotated) as fp16 too:
//             QKNorm bounds their range and fp16 keeps 3 more mantissa bits than bf16 for
//             the values that keys-as-values layers feed straight into the output.
//   per key tile of 128 keys (causal / sliding-window tiles outside the band are skipped):
//     S  = Q K^T        M=256 N=128, fp32 in TMEM; rotated 64-dim chunks come from the
//                       rotated key copy, the others from the pre-RoPE copy
//     softmax           two threads per row: masked row max with a lazy reference (it only
//                       moves when the tile max exceeds it by more than 2^8), P = exp2
//                       rounded to the format of V (head_dim 512: into shared memory;
//                       head_dim 256: into tensor memory over its scores), running sum of the
//                       rounded P
//     O += P V          M=256 N=256 per 256-dim block, V read MN-major; V is the pre-RoPE
//                       key (keys reused as values), the rotated key, or the caller's values
//   epilogue  O / l -> bf16 rows; lse = (m + log2 l) ln 2
// head_dim 512: a 128 x 512 fp32 O fills all 512 TMEM columns, so S borrows columns
// [128, 256): the softmax warps hold that quarter of O in registers while S lives there.
// head_dim 256 (the model's local layers, whose window spans only 9-10 key tiles per pair;
// causal head_dim-256 launches take the same path): the launch holds as many pairs as fit
// at once, each looping over row-tile items, so a pair pays its set-up once, loads the next
// item's queries while the current item's last scores are used, and turns them before
// writing the current output, while the tensor core starts the next item's scores.
//
// Warp roles (320 threads per CTA): warp 0 TMA producer (both CTAs), warp 1 TMEM owner and,
// in the leader CTA, the MMA issuer; warps 2..9 prologue / softmax / epilogue, two threads
// per tile row (each half of the row's score and output columns).  Every wait is bounded; a
// CTA that gives up raises the abort flag of both CTAs of its pair.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "kernels.h"
#include "sm100.cuh"

namespace g4 {
namespace {

constexpr int kThreads = 320;
constexpr int kBM = 128;               // packed query rows per CTA
constexpr int kBN = 128;               // keys per tile (shared by the pair)
constexpr int kSlot = 16384;           // ring slot: 64 keys x 128 dims (S) or 128 keys x 64 dims (V)
constexpr uint32_t kTmemCols = 512;
constexpr int kBarWG = 1;               // the eight row warps
constexpr int kBarPair0 = 2;            // + lane quarter: the two warps of one quarter
constexpr float kLazyMax = 8.0f;       // log2 units

template <int D>
struct PrefillCfg {
    static constexpr int NCH = D / 64;
    static constexpr bool SWAP = (D == 512);
    // head_dim 256: P lives in tensor memory over the scores it came from, so the shared
    // memory of P buffers goes to the ring (10 slots, 2.5 tiles)
    static constexpr int NSLOT = (D == 512) ? 4 : 10;
    static constexpr uint32_t S_COL = (D == 512) ? 128 : 256;
    // head_dim 256: two S buffers (NBUF; columns 256 and 384), so the scores of tile n + 1
    // are computed while the softmax works on tile n; P(n) overwrites the first 64 columns
    // of S(n) as packed bf16 / fp16 and is the tensor-memory A operand of P.V
    static constexpr int NBUF = (D == 512) ? 1 : 2;
    // head_dim 256: the CTA pair loops over row-tile items (persistent), the ring running on
    // from one item to the next; head_dim 512 takes one item per pair
    static constexpr bool PERSIST = (D == 256);
    static constexpr int NS = D / 128;     // S stages per tile (128 dims each)
    static constexpr int NV = D / 256;     // P.V blocks per tile (2 slots each)
};

// head_dim 512 keeps P in shared memory (128 rows x 64 keys per chunk): its S borrows O
// columns, and P.V writes all of them
template <int D>
struct PrefillPArea {
    uint8_t p[1][2][16384];
};
template <>
struct PrefillPArea<256> {};

template <int D>
struct __align__(1024) PrefillSmem : PrefillPArea<D> {
    uint8_t q[PrefillCfg<D>::NCH][16384];  // 128 rows x 64 dims per chunk
    uint8_t ring[PrefillCfg<D>::NSLOT][kSlot];
    uint64_t full[PrefillCfg<D>::NSLOT];   // used in the leader: both CTAs' bytes land here
    uint64_t empty[PrefillCfg<D>::NSLOT];  // per CTA, released by the leader's MMA commits
    // per buffer (tile n uses [n % NBUF]); s_free / p_full / q_ready / o_free count one
    // arrival per CTA; the once-per-item barriers (q_full, q_ready, q_free, o_done, o_free)
    // complete one phase per item
    uint64_t s_free[2], s_full[2], p_full[2], pv_done[2];
    uint64_t q_full, q_ready, o_done, o1_done, drain;
    uint64_t q_free;                       // the item's score products are done with q
    uint64_t o_free;                       // the item's output is read out of O
    float xchg[2][128];                    // a value of each row from each of its two threads
    uint32_t issued;                       // ring positions this CTA's producer filled
    uint32_t q_loads;                      // query tiles this CTA's producer loaded
    uint32_t peer_issued;                  // leader only: the same count of the other CTA
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ bool chunk_rotated(int c, int d, int R) {
    const int lo = c * 64, hi = lo + 64, h = d / 2;
    return (lo < R) || (lo < h + R && hi > h);
}

struct PairGeom {
    int b, g;
    int m0, tq;        // this CTA: first token, valid tokens (<= 0: no valid row)
    int j_lo, j_hi;    // key tiles visited by the pair (inclusive)
};

// Row-tile pairs per (batch, kv head) and the launch's items: one per (pair, batch, kv head).
__device__ __forceinline__ int row_pairs(const PrefillArgs& a) {
    const int tpt = kBM / a.G;
    return ((a.T + tpt - 1) / tpt + 1) / 2;
}

// Geometry of item c for CTA `rank` of the pair.
__device__ __forceinline__ PairGeom pair_geom(const PrefillArgs& a, uint32_t rank, int c) {
    PairGeom g;
    const int tpt = kBM / a.G;                          // tokens per row tile
    const int pairs = row_pairs(a);
    const int bgn = a.B * a.Hkv;
    // Causal layers: all row tiles of one (batch, kv head) in a row, heavy (late) tiles first,
    // so the pairs in flight stream the keys of one head (about 80 MB at T = 65536, inside
    // L2) instead of all heads at staggered positions: DRAM reads of a T = 65536 launch fell
    // from 269 GB to 6.3 GB and its time from 164 to 141 ms.  Sliding-window layers read a
    // short band per pair; there interleaving the heads measured faster.  A persistent pair
    // takes items c, c + P, c + 2P, ... (P pairs launched), so the pairs in flight work on
    // neighbouring items in the same order.
    const bool head_major = a.window <= 0;
    const int pr = head_major ? pairs - 1 - c % pairs : pairs - 1 - c / bgn;
    const int bg = head_major ? c / pairs : c % bgn;
    g.b = bg / a.Hkv;
    g.g = bg % a.Hkv;
    const int mt = 2 * pr + (int)rank;
    g.m0 = mt * tpt;
    g.tq = min(tpt, a.T - g.m0);
    // key rows of the pair's first and last query tokens
    const int first_tok = a.q_off + 2 * pr * tpt;
    const int last_tok = a.q_off + min(a.T, (2 * pr + 2) * tpt) - 1;
    int k_first = 0;
    if (a.window > 0) k_first = max(0, first_tok - a.window + 1);
    g.j_lo = k_first / kBN;
    g.j_hi = last_tok / kBN;
    return g;
}

template <int D, bool PF16>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ PrefillArgs a) {
    using C = PrefillCfg<D>;
    constexpr int NCH = C::NCH;
    constexpr int NSLOT = C::NSLOT;
    extern __shared__ uint8_t smem_raw[];
    PrefillSmem<D>& sm = *reinterpret_cast<PrefillSmem<D>*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const WaitCtl wc{a.wait_limit, a.status};
    volatile int* abort = &sm.abort;
    const int R = a.rope.R;
    // this pair's items: pair, pair + n_pairs, ... below the launch's item count
    const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
    const int n_items = row_pairs(a) * a.B * a.Hkv;
    const int my_items = pair < n_items ? (n_items - 1 - pair) / n_pairs + 1 : 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NSLOT; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.s_free[i], 2);   // one arrival per CTA of the pair
            mbar_init(&sm.s_full[i], 1);
            mbar_init(&sm.p_full[i], 2);
            mbar_init(&sm.pv_done[i], 1);
        }
        mbar_init(&sm.q_full, 1);   // this CTA's raw query tile (and cos/sin rows) landed
        mbar_init(&sm.q_ready, 2);
        mbar_init(&sm.o_done, 1);
        mbar_init(&sm.o1_done, 1);   // head_dim 512: the first 256-dim block of P.V is done
        mbar_init(&sm.drain, 1);
        mbar_init(&sm.q_free, 1);
        mbar_init(&sm.o_free, 2);
        sm.abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc_pair(&sm.tmem_base, kTmemCols);
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t tm_o = tmem;
    const uint32_t tm_s = tmem + C::S_COL;   // S buffer b at tm_s + 128 b
    // head_dim 512: the (cos, sin) rows of the query tile are staged by TMA in the P buffer
    // during the prologue; head_dim 256 reads them from the table
    uint8_t* cs_stage = nullptr;
    if constexpr (C::SWAP) cs_stage = &sm.p[0][0][0];

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&a.tm_kn_s);
            prefetch_tmap(&a.tm_kr_s);
            prefetch_tmap(&a.tm_kn_v);
            prefetch_tmap(&a.tm_kr_v);
            prefetch_tmap(&a.tm_v);
            uint32_t q = 0, nq = 0;   // ring positions filled, query tiles loaded
            for (int k = 0; k < my_items && !*abort; ++k) {
                const PairGeom pg = pair_geom(a, rank, pair + k * n_pairs);
                const int ntiles = pg.j_hi - pg.j_lo + 1;
                // the query buffer takes the next item once the previous item's score
                // products are done with it
                if (k > 0 && !mbar_wait(&sm.q_free, (k - 1) & 1, wc, abort)) break;
                {
                    // the raw query tile (one box per 64-dim chunk, rows = token * G + head)
                    // and, head_dim 512, the (cos, sin) rows of its tokens
                    const int tpt = kBM / a.G;
                    const bool cs = C::SWAP && a.cs_tma;
                    const uint32_t cs_bytes = cs ? (uint32_t)(tpt * R * 8) : 0u;
                    mbar_arrive_expect_tx(&sm.q_full, (uint32_t)(NCH * 16384) + cs_bytes);
                    for (int c = 0; c < NCH; ++c)
                        tma_load_4d(sm.q[c], &a.tm_q, &sm.q_full, c * 64, pg.g * a.G, pg.m0,
                                    pg.b);
                    if (cs) tma_load_2d(cs_stage, &a.tm_cs, &sm.q_full, 0, a.q_off + pg.m0);
                    ++nq;
                }
                for (int n = 0; n < ntiles && !*abort; ++n) {
                    const int key0 = (pg.j_lo + n) * kBN;
                    if (n + 2 < ntiles) {   // pull this CTA's share of a later tile into L2
                        const int kp = key0 + 2 * kBN;
                        for (int c = 0; c < NCH; ++c)
                            tma_prefetch_l2_4d(chunk_rotated(c, D, R) ? &a.tm_kr_s : &a.tm_kn_s,
                                               c * 64, pg.g, kp + 64 * (int)rank, pg.b);
                    }
                    for (int s = 0; s < C::NS && !*abort; ++s, ++q) {
                        const int slot = q % NSLOT;
                        if (!mbar_wait(&sm.empty[slot], ((q / NSLOT) & 1) ^ 1, wc, abort)) break;
                        if (leader) mbar_arrive_expect_tx(&sm.full[slot], 2 * kSlot);
                        for (int h = 0; h < 2; ++h) {
                            const int c = 2 * s + h;
                            const CUtensorMap* map =
                                chunk_rotated(c, D, R) ? &a.tm_kr_s : &a.tm_kn_s;
                            tma_load_4d_pair(sm.ring[slot] + h * (kSlot / 2), map, &sm.full[slot],
                                             c * 64, pg.g, key0 + 64 * (int)rank, pg.b);
                        }
                    }
                    for (int v = 0; v < C::NV && !*abort; ++v)
                        for (int u = 0; u < 2 && !*abort; ++u, ++q) {
                            const int slot = q % NSLOT;
                            if (!mbar_wait(&sm.empty[slot], ((q / NSLOT) & 1) ^ 1, wc, abort))
                                break;
                            if (leader) mbar_arrive_expect_tx(&sm.full[slot], 2 * kSlot);
                            const int c = 4 * v + 2 * (int)rank + u;   // this CTA's half of the block
                            const bool rot = chunk_rotated(c, D, R);
                            const CUtensorMap* map = a.kv_is_k == 0 ? &a.tm_v
                                                     : (a.kv_is_k == 2 && rot) ? &a.tm_kr_v
                                                                               : &a.tm_kn_v;
                            tma_load_4d_pair(sm.ring[slot], map, &sm.full[slot], c * 64, pg.g,
                                             key0, pg.b);
                        }
                }
            }
            sm.q_loads = nq;
            sm.issued = q;   // read at teardown, after __syncthreads
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (leader CTA only)
        if (lane == 0 && leader) {
            const uint32_t idesc_s = idesc_f16kind_f32(256, kBN, false, false, false);
            const uint32_t idesc_o = idesc_f16kind_f32(256, 256, false, true, !PF16);
            // shared-memory descriptors of the first buffer of each kind; an operand's start
            // address field (16-byte units) is advanced by adding to the descriptor
            const uint64_t dq0 = sdesc_sw128(smem_u32(sm.q[0]), 16, 1024);
            const uint64_t dr0 = sdesc_sw128(smem_u32(sm.ring[0]), 16, 1024);
            const uint64_t dv0 = sdesc_sw128(smem_u32(sm.ring[0]), kSlot, 1024);   // V: MN-major
            constexpr uint32_t kChunkD = 16384 >> 4, kSlotD = kSlot >> 4, kHalfD = (kSlot / 2) >> 4;
            if constexpr (C::SWAP) {
                // one item per pair (the host launches one cluster per item)
                const PairGeom pg = pair_geom(a, rank, pair);
                const int ntiles = my_items > 0 ? pg.j_hi - pg.j_lo + 1 : 0;
                const uint64_t dp0 = sdesc_sw128(smem_u32(sm.p[0][0]), 16, 1024);
                uint32_t q = 0;
                for (int n = 0; n < ntiles; ++n) {
                    if (!mbar_wait(&sm.s_free[0], n & 1, wc, abort)) goto done;
                    tc_fence_after();
                    for (int s = 0; s < C::NS; ++s, ++q) {
                        const uint32_t slot = q % NSLOT;
                        if (!mbar_wait(&sm.full[slot], (q / NSLOT) & 1, wc, abort)) goto done;
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            mma_pair_f16(tm_s, dq0 + (2 * s + (kk >> 2)) * kChunkD + (kk & 3) * 2,
                                         dr0 + slot * kSlotD + (kk >> 2) * kHalfD + (kk & 3) * 2,
                                         idesc_s, (s | kk) != 0 ? 1u : 0u);
                        mma_commit_pair(&sm.empty[slot]);
                    }
                    mma_commit_pair(&sm.s_full[0]);
                    if (!mbar_wait(&sm.p_full[0], n & 1, wc, abort)) goto done;
                    tc_fence_after();
                    for (int v = 0; v < C::NV; ++v, q += 2) {
                        const uint32_t s0 = q % NSLOT, s1 = (q + 1) % NSLOT;
                        if (!mbar_wait(&sm.full[s0], (q / NSLOT) & 1, wc, abort)) goto done;
                        if (!mbar_wait(&sm.full[s1], ((q + 1) / NSLOT) & 1, wc, abort))
                            goto done;
                        tc_fence_after();
                        // V: 16 keys per step (two 8-row groups of 1024 B); the CTA's second
                        // 64-dim chunk sits in the next slot (LBO)
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            mma_pair_f16(tm_o + v * 256, dp0 + (kk >> 2) * kChunkD + (kk & 3) * 2,
                                         dv0 + s0 * kSlotD + kk * (2048 >> 4), idesc_o,
                                         (n > 0 || kk > 0) ? 1u : 0u);
                        mma_commit_pair(&sm.empty[s0]);
                        mma_commit_pair(&sm.empty[s1]);
                        // the O quarter that S borrows lies in block 0: the softmax warps can
                        // move it out while block 1 runs
                        if (v == 0) mma_commit_pair(&sm.o1_done);
                    }
                    if (n == ntiles - 1) mma_commit_pair(&sm.o_done);
                }
            } else {
                // tile g's slots sit at ring positions 4g .. 4g + 3 (S stages, then V), g
                // counting the tiles of all of this pair's items.  The thread issues whichever
                // product is ready, the scores of the next tile first: a value product never
                // waits behind the key loads of a later score product, and its slots go back
                // to the producer as early as possible.  S(g) and then P(g) occupy TMEM buffer
                // g & 1 until the value product of tile g is done.  An item's scores start once
                // both CTAs have turned its queries (the previous item's output may still be
                // read out then); its first value product waits until that output is read.
                constexpr int SPT = C::NS + 2 * C::NV;   // slots per tile
                auto slots_full = [&](uint32_t q0, int cnt) {
                    for (int k = 0; k < cnt; ++k) {
                        const uint32_t q = q0 + (uint32_t)k;
                        if (!mbar_test_wait(&sm.full[q % NSLOT], (q / NSLOT) & 1)) return false;
                    }
                    return true;
                };
                int gb = 0;   // tiles of the earlier items
                for (int k = 0; k < my_items; ++k) {
                    const PairGeom pg = pair_geom(a, rank, pair + k * n_pairs);
                    const int ntiles = pg.j_hi - pg.j_lo + 1;
                    if (!mbar_wait(&sm.q_ready, k & 1, wc, abort)) goto done;
                    int sc = 0, pc = 0;   // next tile of the score product / of the value product
                    long long polls = 0;
                    unsigned long long t_idle = 0;
                    while (pc < ntiles) {
                        // S(g) into buffer g & 1, whose P(g - 2) the value product of tile g - 2
                        // has read
                        const int gs = gb + sc;
                        if (sc < ntiles &&
                            (gs < 2 || mbar_test_wait(&sm.pv_done[gs & 1], ((gs - 2) >> 1) & 1)) &&
                            slots_full((uint32_t)(gs * SPT), C::NS)) {
                            const uint32_t b = gs & 1;
                            tc_fence_after();
                            for (int s = 0; s < C::NS; ++s) {
                                const uint32_t slot = (uint32_t)(gs * SPT + s) % NSLOT;
#pragma unroll
                                for (int kk = 0; kk < 8; ++kk)
                                    mma_pair_f16(tm_s + 128 * b,
                                                 dq0 + (2 * s + (kk >> 2)) * kChunkD + (kk & 3) * 2,
                                                 dr0 + slot * kSlotD + (kk >> 2) * kHalfD + (kk & 3) * 2,
                                                 idesc_s, (s | kk) != 0 ? 1u : 0u);
                                mma_commit_pair(&sm.empty[slot]);
                            }
                            mma_commit_pair(&sm.s_full[b]);
                            // the item's last scores: its queries may give way to the next item's
                            if (sc == ntiles - 1) mma_commit_pair(&sm.q_free);
                            ++sc;
                            polls = 0;
                            continue;
                        }
                        // O += P(g) V(g) once both CTAs wrote P(g) (tensor memory, over S(g)),
                        // its value slots landed and, for an item's first tile, the previous
                        // item's output is read out of O
                        const int gp = gb + pc;
                        if (pc < sc && mbar_test_wait(&sm.p_full[gp & 1], (gp >> 1) & 1) &&
                            slots_full((uint32_t)(gp * SPT + C::NS), 2 * C::NV) &&
                            (pc > 0 || k == 0 || mbar_test_wait(&sm.o_free, (k - 1) & 1))) {
                            const uint32_t pb = gp & 1;
                            tc_fence_after();
                            for (int v = 0; v < C::NV; ++v) {
                                const uint32_t q = (uint32_t)(gp * SPT + C::NS + 2 * v);
                                const uint32_t s0 = q % NSLOT, s1 = (q + 1) % NSLOT;
#pragma unroll
                                for (int kk = 0; kk < 8; ++kk)   // 16 keys = 8 packed P columns
                                    mma_pair_f16_ts(tm_o + v * 256, tm_s + 128 * pb + 8 * kk,
                                                    dv0 + s0 * kSlotD + kk * (2048 >> 4), idesc_o,
                                                    (pc > 0 || kk > 0) ? 1u : 0u);
                                mma_commit_pair(&sm.empty[s0]);
                                mma_commit_pair(&sm.empty[s1]);
                            }
                            mma_commit_pair(&sm.pv_done[pb]);
                            if (pc == ntiles - 1) mma_commit_pair(&sm.o_done);
                            ++pc;
                            polls = 0;
                            continue;
                        }
                        // nothing ready: bounded polling, like every other wait
                        if (*abort) goto done;
                        if ((++polls & 63) == 0) {
                            const unsigned long long now = global_ns();
                            if (polls == 64) t_idle = now;
                            if (polls >= a.wait_limit || now - t_idle > kWaitTimeoutNs) {
                                atomicExch(a.status, (int)G4ATTN_ERR_TIMEOUT);
                                *abort = 1;
                                goto done;
                            }
                        }
                    }
                    gb += ntiles;
                }
            }
        done:;
        }
    } else {
        // ------------------------------------ prologue / softmax / correction / epilogue
        // Eight warps.  Warps w and w + 4 share TMEM lane quarter w & 3, so the two threads of
        // tile row r = 32 (w & 3) + lane sit in a pair of warps: thread (row, ch) takes the
        // row's score columns [64 ch, 64 ch + 64) and output columns [D/2 ch, D/2 ch + D/2).
        // Both keep the row's reference max (they update it from the same values), and they
        // agree on it through a shared-memory exchange behind a 64-thread barrier of the pair.
        const int t256 = threadIdx.x - 64;         // 0..255
        const int wq = warp - 2;                   // 0..7
        const int quarter = warp & 3;              // TMEM lane quarter
        const int ch = wq >> 2;                    // column half of the row
        const int row = quarter * 32 + lane;       // this thread's TMEM lane = tile row
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const int bar_pair = kBarPair0 + quarter;  // the two warps of this lane quarter
        const int G = a.G;
        const int lgG = __ffs(G) - 1;              // G divides 128 (host check): a power of two

        // ---- prologue of item k: QKNorm + RoPE of the 128 packed rows, in place in shared
        // memory.  The raw bf16 tile arrived by TMA (row r = token r / G, head r % G, the layout the
        // MMAs read).  Warp wq turns rows [16 wq, 16 wq + 16) into normalised, rotated fp16
        // rows, one row at a time across the warp: lane l holds dims [H l, H l + H) and their
        // RoPE partners d/2 + [H l, H l + H), so both members of every rotated pair, their
        // gammas (in registers for the whole tile) and a contiguous run of the row's
        // (cos, sin) entries are the lane's own; the row's sum of squares is a warp sum.
        constexpr int H = D / 64;                  // dims per lane in each half of the row
        auto prologue = [&](int k) -> bool {
            const PairGeom pq = pair_geom(a, rank, pair + k * n_pairs);
            constexpr int half = D / 2;
            const int i0 = lane * H;               // first pair index of this lane
            const int col = i0 % 64;               // column within the 64-dim chunk
            uint8_t* const qu = sm.q[i0 / 64];
            uint8_t* const qv = sm.q[(half + i0) / 64];
            const float2* const cs_smem = reinterpret_cast<const float2*>(cs_stage);
            const float2* const cs_glob = a.rope_cs + (size_t)(a.q_off + pq.m0) * R;
            const bool rot_lane = i0 < R;
            float gu[H], gv[H];   // (read again per item: not held across the main loop)
#pragma unroll
            for (int kk = 0; kk < H; ++kk) {
                gu[kk] = a.qk_norm ? __ldg(a.gamma_q + i0 + kk) : 1.f;
                gv[kk] = a.qk_norm ? __ldg(a.gamma_q + half + i0 + kk) : 1.f;
            }
            // NB rows per step, each stage over all of them, so the rows' load, warp-sum and
            // square-root latencies overlap (8 rows at head_dim 256 spill registers beside the
            // state the next item's epilogue keeps)
            constexpr int NB = 4;
            // head_dim 256: the (cos, sin) of the lane's pairs at the warp's first token come
            // from the table (L2, read before the query wait); from one token to the next they
            // turn by theta_i <= 1 rad (its cos and sin in fp32; angle addition, at most 15
            // steps: ~1e-6 rad)
            const bool turn4 = H == 4 && rot_lane && i0 + 4 <= R;
            float2 cr[H == 4 ? 4 : 1], stp[H == 4 ? 4 : 1];
            if constexpr (H == 4) {
                const int tok0 = (wq * 16) >> lgG;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    cr[kk] = make_float2(1.f, 0.f);
                    stp[kk] = make_float2(1.f, 0.f);
                    if (turn4) {
                        const float th =
                            exp2f(-(2.f * (float)(i0 + kk) / (float)D) * (float)a.rope.log2_base);
                        __sincosf(th, &stp[kk].y, &stp[kk].x);
                    }
                }
                if (turn4 && tok0 < pq.tq) {
                    const float4* g = reinterpret_cast<const float4*>(cs_glob + (size_t)tok0 * R + i0);
                    const float4 lo = __ldg(g), hi = __ldg(g + 1);
                    cr[0] = make_float2(lo.x, lo.y);
                    cr[1] = make_float2(lo.z, lo.w);
                    cr[2] = make_float2(hi.x, hi.y);
                    cr[3] = make_float2(hi.z, hi.w);
                }
            }
            const bool good = group_all(mbar_wait(&sm.q_full, k & 1, wc, abort), kBarWG, 256);
            if (good) {
#pragma unroll 1
                for (int r0 = wq * 16; r0 < wq * 16 + 16; r0 += NB) {
                    float u[NB][H], v[NB][H];
#pragma unroll
                    for (int j = 0; j < NB; ++j) {
                        const uint32_t off = sw128_offset(r0 + j, col);
                        if constexpr (H == 4) {
                            const uint2 wu = *reinterpret_cast<const uint2*>(qu + off);
                            const uint2 wv = *reinterpret_cast<const uint2*>(qv + off);
                            const float2 u0 = bf16x2_to_f2(wu.x), u1 = bf16x2_to_f2(wu.y);
                            const float2 v0 = bf16x2_to_f2(wv.x), v1 = bf16x2_to_f2(wv.y);
                            u[j][0] = u0.x; u[j][1] = u0.y; u[j][2] = u1.x; u[j][3] = u1.y;
                            v[j][0] = v0.x; v[j][1] = v0.y; v[j][2] = v1.x; v[j][3] = v1.y;
                        } else {
                            const uint4 wu = *reinterpret_cast<const uint4*>(qu + off);
                            const uint4 wv = *reinterpret_cast<const uint4*>(qv + off);
                            const uint32_t au[4] = {wu.x, wu.y, wu.z, wu.w};
                            const uint32_t av[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                            for (int m = 0; m < 4; ++m) {
                                const float2 fu = bf16x2_to_f2(au[m]), fv = bf16x2_to_f2(av[m]);
                                u[j][2 * m] = fu.x; u[j][2 * m + 1] = fu.y;
                                v[j][2 * m] = fv.x; v[j][2 * m + 1] = fv.y;
                            }
                        }
                    }
                    if (a.qk_norm) {
                        float ss[NB];
#pragma unroll
                        for (int j = 0; j < NB; ++j) {
                            ss[j] = 0.f;
#pragma unroll
                            for (int k = 0; k < H; ++k)
                                ss[j] = fmaf(u[j][k], u[j][k], fmaf(v[j][k], v[j][k], ss[j]));
                        }
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
                            for (int j = 0; j < NB; ++j) ss[j] += __shfl_xor_sync(0xffffffffu, ss[j], o);
#pragma unroll
                        for (int j = 0; j < NB; ++j) {
                            const float inv = rsqrtf(ss[j] / (float)D + a.eps);
#pragma unroll
                            for (int k = 0; k < H; ++k) {
                                u[j][k] = u[j][k] * inv * gu[k];
                                v[j][k] = v[j][k] * inv * gv[k];
                            }
                        }
                    }
#pragma unroll
                    for (int j = 0; j < NB; ++j) {
                        const int r = r0 + j;
                        // rows past the end of the sequence hold zeros (TMA fill) and have no
                        // (cos, sin) row in the table: they skip the rotation
                        if (rot_lane && (r >> lgG) < pq.tq) {
                            const size_t cso = (size_t)(r >> lgG) * R + i0;
                            float2 c[H];
                            bool have = false;
                            if constexpr (H == 4) {
                                if (turn4) {
#pragma unroll
                                    for (int kk = 0; kk < 4; ++kk) c[kk] = cr[kk];
                                    have = true;
                                }
                            }
                            if (!have) {
#pragma unroll
                                for (int k = 0; k < H; ++k)   // shared-memory rows or the table
                                    c[k] = i0 + k >= R ? make_float2(1.f, 0.f)
                                           : a.cs_tma ? cs_smem[cso + k] : cs_glob[cso + k];
                            }
#pragma unroll
                            for (int k = 0; k < H; ++k) {
                                const float x = u[j][k] * c[k].x - v[j][k] * c[k].y;
                                v[j][k] = u[j][k] * c[k].y + v[j][k] * c[k].x;
                                u[j][k] = x;
                            }
                        }
                        const uint32_t off = sw128_offset(r, col);
                        if constexpr (H == 4) {
                            *reinterpret_cast<uint2*>(qu + off) =
                                make_uint2(pack_f16x2(u[j][0], u[j][1]), pack_f16x2(u[j][2], u[j][3]));
                            *reinterpret_cast<uint2*>(qv + off) =
                                make_uint2(pack_f16x2(v[j][0], v[j][1]), pack_f16x2(v[j][2], v[j][3]));
                        } else {
                            *reinterpret_cast<uint4*>(qu + off) =
                                make_uint4(pack_f16x2(u[j][0], u[j][1]), pack_f16x2(u[j][2], u[j][3]),
                                           pack_f16x2(u[j][4], u[j][5]), pack_f16x2(u[j][6], u[j][7]));
                            *reinterpret_cast<uint4*>(qv + off) =
                                make_uint4(pack_f16x2(v[j][0], v[j][1]), pack_f16x2(v[j][2], v[j][3]),
                                           pack_f16x2(v[j][4], v[j][5]), pack_f16x2(v[j][6], v[j][7]));
                        }
                        if constexpr (H == 4) {
                            // the next row's token: one theta_i further
                            if (((r + 1) >> lgG) != (r >> lgG)) {
#pragma unroll
                                for (int kk = 0; kk < 4; ++kk)
                                    cr[kk] = make_float2(cr[kk].x * stp[kk].x - cr[kk].y * stp[kk].y,
                                                         cr[kk].x * stp[kk].y + cr[kk].y * stp[kk].x);
                            }
                        }
                    }
                }
            }
            fence_proxy_async_smem();
            group_sync(kBarWG, 256);
            // Q ready (and, head_dim 512, S free for tile 0)
            if (t256 == 0) mbar_arrive_remote(C::SWAP ? &sm.s_free[0] : &sm.q_ready, 0);
            return good;
        };

        // ---- items: main loop, the next item's prologue, then this item's epilogue
        const float c2 = a.scale_log2;              // > 0 (checked on the host)
        // head_dim 512: this thread's 64 columns of the O quarter that S borrows
        uint32_t o1[C::SWAP ? 64 : 1];
        // the row's value of v over both threads of the pair (both read the same two values)
        auto pair_max = [&](float v) -> float {
            sm.xchg[ch][row] = v;
            group_sync(bar_pair, 64);
            return fmaxf(sm.xchg[0][row], sm.xchg[1][row]);
        };
        bool ok = my_items > 0 && prologue(0);
        int gb = 0;   // tiles of the earlier items
        // (head_dim 512: one item per pair)
        const int loop_items = C::PERSIST ? my_items : min(my_items, 1);
        for (int k = 0; k < loop_items && ok; ++k) {
            // (the geometry is recomputed where needed rather than held across the tiles)
            int ntiles, j_lo, tok_r, t_first, t_last;
            bool row_valid;
            {
                const PairGeom pg = pair_geom(a, rank, pair + k * n_pairs);
                ntiles = pg.j_hi - pg.j_lo + 1;
                j_lo = pg.j_lo;
                tok_r = pg.m0 + row / G;                // token of this row
                row_valid = (row / G) < pg.tq;
                t_first = a.q_off + pg.m0;
                t_last = t_first + pg.tq - 1;
            }
            const int kr_r = a.q_off + tok_r;           // key row of its position (mask bound)
            const int lo_r = a.window > 0 ? kr_r - a.window + 1 : 0;
            // rows past the end of the sequence hold zero queries; a finite reference keeps
            // their (never stored) P finite on the unmasked path
            float m_ref = row_valid ? -INFINITY : 0.f, l_own = 0.f;
            if constexpr (C::SWAP) {
#pragma unroll
                for (int i = 0; i < 64; ++i) o1[i] = 0u;
            }
            for (int n = 0; n < ntiles && ok; ++n) {
                const int gt = C::PERSIST ? gb + n : n;   // tile index over the pair's items
                const int key0 = (j_lo + n) * kBN;
                const int keyc = key0 + 64 * ch;        // key of this thread's first column
                if constexpr (C::SWAP) {
                    if (n > 0) {
                        // this thread's half of O[:, 128..255] leaves TMEM so S(n) can use those
                        // columns (block 0 of the previous P.V is done; block 1 may still run, it
                        // does not touch them)
                        ok = group_all(mbar_wait(&sm.o1_done, (n - 1) & 1, wc, abort), kBarWG, 256);
                        if (!ok) break;
                        tc_fence_after();
                        tmem_ld32_nowait(tm_s + 64 * ch + lane_off, o1);
                        tmem_ld32_nowait(tm_s + 64 * ch + 32 + lane_off, o1 + 32);
                        tmem_ld_wait();
                        tc_fence_before();
                        group_sync(kBarWG, 256);
                        if (t256 == 0) mbar_arrive_remote(&sm.s_free[0], 0);
                    }
                }
                const uint32_t sbuf = C::SWAP ? 0u : (uint32_t)(gt & 1);
                const uint32_t tm_sn = tm_s + 128 * sbuf;   // this tile's S
                ok = group_all(C::SWAP ? mbar_wait(&sm.s_full[0], gt & 1, wc, abort)
                                       : mbar_wait(&sm.s_full[sbuf], (gt >> 1) & 1, wc, abort),
                               kBarWG, 256);
                if (!ok) break;
                tc_fence_after();
                const bool need_mask = (key0 + kBN - 1 > t_first) ||
                                       (a.window > 0 && key0 <= t_last - a.window);
                float psum = 0.f, alpha = 1.f;
                // head_dim 256: P(n) waits in registers (packed pairs) until the pass stands, then
                // overwrites the first 64 columns of S(n) in tensor memory
                uint32_t pw[C::SWAP ? 1 : 32];
                // one pass over this thread's 64 scores with reference -negm (log2 units): P
                // (rounded to the format of V) to the P buffer (head_dim 512) or pw (head_dim 256),
                // its sum to ps, the largest visible raw score to mxr; MASK drops keys outside the
                // causal band or the window (a separate copy of the loop, so unmasked tiles test
                // nothing)
                auto pass = [&](auto mask_tag, float negm, float& ps, float& mxr) {
                    constexpr bool MASK = decltype(mask_tag)::value;
                    uint32_t sa[32], sb[32];
                    tmem_ld32_nowait(tm_sn + 64 * ch + lane_off, sa);
                    tmem_ld32_nowait(tm_sn + 64 * ch + 32 + lane_off, sb);
                    tmem_ld_wait();
#pragma unroll
                    for (int bb = 0; bb < 2; ++bb) {
                        const uint32_t* cur = bb ? sb : sa;
                        uint32_t w[16];
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            float s0 = __uint_as_float(cur[e]), s1 = __uint_as_float(cur[e + 1]);
                            if constexpr (MASK) {
                                const int j = keyc + bb * 32 + e;
                                if (!(row_valid && j <= kr_r && j >= lo_r)) s0 = -INFINITY;
                                if (!(row_valid && j + 1 <= kr_r && j + 1 >= lo_r)) s1 = -INFINITY;
                            }
                            mxr = fmaxf(mxr, fmaxf(s0, s1));
                            const float p0 = ex2_approx(fmaf(s0, c2, negm));
                            const float p1 = ex2_approx(fmaf(s1, c2, negm));
                            if constexpr (PF16) {
                                w[e / 2] = pack_f16x2(p0, p1);
                                ps += p0 + p1;
                            } else {
                                const __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
                                const float2 f = __bfloat1622float2(h);
                                ps += f.x + f.y;
                                w[e / 2] = *reinterpret_cast<const uint32_t*>(&h);
                            }
                        }
                        if constexpr (C::SWAP) {
                            // keys 64 ch .. 64 ch + 63 are P chunk ch
                            uint8_t* pb = sm.p[0][ch];
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                *reinterpret_cast<uint4*>(pb + sw128_offset(row, bb * 32 + 8 * k)) =
                                    make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
                        } else {
#pragma unroll
                            for (int k = 0; k < 16; ++k) pw[16 * bb + k] = w[k];
                        }
                    }
                };
                auto run = [&](float negm, float& ps, float& mxr) {
                    if (need_mask) pass(std::true_type{}, negm, ps, mxr);
                    else pass(std::false_type{}, negm, ps, mxr);
                };
                // the largest visible raw score of this thread's 64 columns, no exponentials
                auto scan = [&](auto mask_tag, float& mxr) {
                    constexpr bool MASK = decltype(mask_tag)::value;
                    uint32_t sa[32], sb[32];
                    tmem_ld32_nowait(tm_sn + 64 * ch + lane_off, sa);
                    tmem_ld32_nowait(tm_sn + 64 * ch + 32 + lane_off, sb);
                    tmem_ld_wait();
#pragma unroll
                    for (int bb = 0; bb < 2; ++bb) {
                        const uint32_t* cur = bb ? sb : sa;
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            float s0 = __uint_as_float(cur[e]);
                            if constexpr (MASK) {
                                const int j = keyc + bb * 32 + e;
                                if (!(row_valid && j <= kr_r && j >= lo_r)) s0 = -INFINITY;
                            }
                            mxr = fmaxf(mxr, s0);
                        }
                    }
                };
                float mxr = -INFINITY;
                if (C::PERSIST && __any_sync(0xffffffffu, m_ref == -INFINITY)) {
                    // rows without a reference yet (their first visible keys): the row's largest
                    // score over both threads first, then one pass with it.  head_dim 256 only:
                    // there one tile in ten is an item's first; the head_dim-512 loop measured
                    // slower with the branch
                    if (need_mask) scan(std::true_type{}, mxr);
                    else scan(std::false_type{}, mxr);
                    const float mx = pair_max(mxr * c2);
                    if (mx > m_ref + kLazyMax || (m_ref == -INFINITY && mx != -INFINITY)) {
                        alpha = (m_ref == -INFINITY) ? 0.f : exp2f(m_ref - mx);
                        m_ref = mx;
                    }
                    run(m_ref == -INFINITY ? 0.f : -m_ref, psum, mxr);
                    // head_dim 256: P overwrites S columns the partner thread reads
                    if constexpr (!C::SWAP) group_sync(bar_pair, 64);
                } else {
                    // one pass with the current reference; the row's largest score over both
                    // threads decides whether the reference moves (it moves only when a score
                    // exceeds it by more than the lazy headroom, or while it is -inf), and then
                    // the pass runs again with the new one
                    run(m_ref == -INFINITY ? 0.f : -m_ref, psum, mxr);
                    const float mx = pair_max(mxr * c2);
                    const bool jump = mx > m_ref + kLazyMax || (m_ref == -INFINITY && mx != -INFINITY);
                    // the warps of the pair hold the same rows: the same decision in both
                    if (__any_sync(0xffffffffu, jump)) {
                        if (jump) {
                            alpha = (m_ref == -INFINITY) ? 0.f : exp2f(m_ref - mx);
                            m_ref = mx;
                        }
                        psum = 0.f;
                        run(m_ref == -INFINITY ? 0.f : -m_ref, psum, mxr);
                        // head_dim 256: P overwrites S columns the partner thread reads
                        if constexpr (!C::SWAP) group_sync(bar_pair, 64);
                    }
                }
                if constexpr (!C::SWAP) {
                    // P(n) as packed pairs over the first 64 columns of S(n): this thread's 64 keys
                    // are columns [32 ch, 32 ch + 32), the A operand of the value product
                    tmem_st16_u32(tm_sn + 32 * ch + lane_off, pw);
                    tmem_st16_u32(tm_sn + 32 * ch + 16 + lane_off, pw + 16);
                }
                l_own = l_own * alpha + psum;
                // correction of the accumulator when a finite reference max moved (rare: a row
                // whose reference was still -inf has an all-zero accumulator); with two S
                // buffers the value product of the tile before may still be running
                if (__any_sync(0xffffffffu, alpha != 1.f && alpha != 0.f && n > 0)) {
                    if (!C::SWAP &&
                        !mbar_wait(&sm.pv_done[(gt - 1) & 1], ((gt - 1) >> 1) & 1, wc, abort))
                        *abort = 1;
                    if constexpr (C::SWAP) {
#pragma unroll
                        for (int i = 0; i < 64; ++i) o1[i] = __float_as_uint(__uint_as_float(o1[i]) * alpha);
                    }
                    // this thread's output columns [D/2 ch, D/2 ch + D/2) (head_dim 512: less the
                    // quarter in o1)
                    for (int c = (D / 64) * ch; c < (D / 64) * (ch + 1); ++c) {
                        if (C::SWAP && c >= 4 && c < 8) continue;
                        uint32_t o[32];
                        tmem_ld32_nowait(tm_o + c * 32 + lane_off, o);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st32_nowait(tm_o + c * 32 + lane_off, o);
                    }
                }
                if constexpr (C::SWAP) {
                    // this thread's half of O[:, 128..255] back for the P.V product
                    tmem_st32_nowait(tm_s + 64 * ch + lane_off, o1);
                    tmem_st32_nowait(tm_s + 64 * ch + 32 + lane_off, o1 + 32);
                }
                tmem_st_wait();   // P, O quarter and any rescaled O in TMEM
                fence_proxy_async_smem();
                tc_fence_before();
                group_sync(kBarWG, 256);
                if (t256 == 0) mbar_arrive_remote(&sm.p_full[sbuf], 0);
            }
            if (!ok) break;
            // the next item's queries are normalised and turned before this item's output is
            // written, so the next item's first score products run during this epilogue
            if constexpr (C::PERSIST) {
                if (k + 1 < my_items) {
                    ok = prologue(k + 1);
                    if (!ok) break;
                }
            }
            // ---- epilogue
            ok = group_all(mbar_wait(&sm.o_done, C::PERSIST ? k & 1 : 0, wc, abort), kBarWG, 256);
            if (!ok) break;
            {
                tc_fence_after();
                // the row's sum over both threads (the end-of-tile barrier above ordered the last
                // exchange's reads before this write)
                sm.xchg[ch][row] = l_own;
                group_sync(bar_pair, 64);
                const float l_sum = sm.xchg[0][row] + sm.xchg[1][row];
                const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
                const PairGeom pg = pair_geom(a, rank, pair + k * n_pairs);
                const int h = pg.g * G + row % G;
                uint16_t* dst = a.out + (((size_t)pg.b * a.T + tok_r) * a.Hq + h) * D + (D / 2) * ch;
                const uint32_t tcol = tm_o + (D / 2) * ch + lane_off;
                const bool out32 = (reinterpret_cast<uintptr_t>(a.out) & 31) == 0;
                // the next block of O loads while the current one is converted and stored
                uint32_t oa[32], ob[32];
                tmem_ld32_nowait(tcol, oa);
#pragma unroll 1
                for (int c = 0; c < D / 64; c += 2) {
                    tmem_ld_wait();
                    tmem_ld32_nowait(tcol + (c + 1) * 32, ob);
                    auto store = [&](const uint32_t* o, int cc) {
                        if (!row_valid) return;
                        uint32_t w[16];
#pragma unroll
                        for (int e = 0; e < 32; e += 2)
                            w[e / 2] = pack_bf16x2(__uint_as_float(o[e]) * inv,
                                                   __uint_as_float(o[e + 1]) * inv);
                        if (out32) {
                            // whole 32-byte sectors per lane: a row's pieces are 64 B apart
                            // from the warp's other rows, so 16-byte stores wrote half sectors
                            st_global_v8(dst + cc * 32, w);
                            st_global_v8(dst + cc * 32 + 16, w + 8);
                        } else {
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                *reinterpret_cast<uint4*>(dst + cc * 32 + 8 * k) =
                                    make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
                        }
                    };
                    store(oa, c);
                    tmem_ld_wait();
                    if (c + 2 < D / 64) tmem_ld32_nowait(tcol + (c + 2) * 32, oa);
                    store(ob, c + 1);
                }
                if (row_valid && a.lse && ch == 0)
                    a.lse[((size_t)pg.b * a.Hq + h) * a.T + tok_r] =
                        l_sum > 0.f ? (m_ref + log2f(l_sum)) * 0.6931471805599453f : -INFINITY;
            }
            if constexpr (C::PERSIST) {
                // O is read out: the next item's value product may overwrite it
                tc_fence_before();
                group_sync(kBarWG, 256);
                if (t256 == 0) mbar_arrive_remote(&sm.o_free, 0);
                gb += ntiles;
            }
        }
    }

    // -------------------------------------------------------------------- teardown
    // A CTA that gave up tells its peer, so the peer's waits end promptly too, and the
    // other CTA tells the leader how many ring positions it filled.
    __syncthreads();   // every role is done: neither producer issues another copy
    if (threadIdx.x == 0) {
        if (*abort) st_shared_remote_u32((const void*)&sm.abort, rank ^ 1u, 1u);
        if (!leader) st_shared_remote_u32((const void*)&sm.peer_issued, 0u, sm.issued);
    }
    tc_fence_before();
    cluster_sync();
    if (*abort && threadIdx.x == 0) {
        // Every copy either CTA started must land before either frees its shared memory.
        // The query tile completes on this CTA's own barrier.  The key / value halves of
        // both CTAs complete on the leader's ring barriers, which the leader settles: a
        // position filled by one CTA only gets the other half's bytes counted as arrived
        // (and, if the leader never armed it, is armed first), so every phase completes
        // exactly when the copies that were issued have landed.  A slot is refilled only
        // after both halves of its previous position were consumed, so positions below
        // the last NSLOT have landed already.  A query tile is loaded only after both CTAs'
        // prologues used the one before, so only the last one can be in flight.
        if (sm.q_loads > 0) mbar_wait_drain(&sm.q_full, (sm.q_loads - 1) & 1);
        if (leader) {
            const uint32_t mine = sm.issued, peer = sm.peer_issued;
            const uint32_t hi = mine > peer ? mine : peer;
            const uint32_t lo = hi > (uint32_t)NSLOT ? hi - (uint32_t)NSLOT : 0u;
            for (uint32_t k = lo; k < hi; ++k) {
                uint64_t* bar = &sm.full[k % NSLOT];
                if (k >= mine) {            // only the other CTA filled it
                    mbar_arrive_expect_tx(bar, 2 * kSlot);
                    mbar_complete_tx(bar, kSlot);
                } else if (k >= peer) {     // only the leader filled it
                    mbar_complete_tx(bar, kSlot);
                }
                mbar_wait_drain(bar, (k / NSLOT) & 1);
            }
        }
    }
    tc_fence_before();
    cluster_sync();   // the leader's settled copies have landed in both CTAs
    if (leader && warp == 1 && lane == 0) {
        // every MMA of the pair must be complete before either CTA frees its columns
        mma_commit_pair(&sm.drain);
        mbar_wait_drain(&sm.drain, 0);
    }
    tc_fence_before();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

template <int D, bool PF16>
cudaError_t run_prefill(const PrefillArgs& a, cudaStream_t stream) {
    const size_t smem = sizeof(PrefillSmem<D>) + 1024;
    static_assert(sizeof(PrefillSmem<D>) + 1024 <= 227 * 1024, "prefill shared memory");
    cudaError_t e = cudaFuncSetAttribute(prefill_kernel<D, PF16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int tpt = kBM / a.G;
    const int mt_count = (a.T + tpt - 1) / tpt;
    const long long items = (long long)((mt_count + 1) / 2) * a.B * a.Hkv;
    if (items > (1LL << 30)) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * items), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if constexpr (PrefillCfg<D>::PERSIST) {
        // persistent pairs: as many clusters as fit on the device at once (looked up once per
        // device), each looping over its share of the items
        static int max_clusters[64] = {};
        int dev = 0;
        if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
        if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
        if (max_clusters[dev] <= 0) {
            int n = 0;
            if ((e = cudaOccupancyMaxActiveClusters(&n, prefill_kernel<D, PF16>, &cfg)) !=
                cudaSuccess)
                return e;
            if (n <= 0) return cudaErrorInvalidConfiguration;
            max_clusters[dev] = n;
        }
        if (items > max_clusters[dev]) cfg.gridDim = dim3((unsigned)(2 * max_clusters[dev]), 1, 1);
    }
    e = cudaLaunchKernelEx(&cfg, prefill_kernel<D, PF16>, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

size_t prefill_cs_stage_bytes(int d) {
    // head_dim 256 stages none: its ring runs on across a pair's items
    return d == 512 ? sizeof(PrefillPArea<512>::p) : 0;
}

size_t prefill_smem_bytes(int d) {
    return d == 512 ? sizeof(PrefillSmem<512>) + 1024 : sizeof(PrefillSmem<256>) + 1024;
}

cudaError_t launch_prefill(const PrefillArgs& a, cudaStream_t stream) {
    if (a.B == 0 || a.T == 0) return cudaSuccess;
    // P takes the 16-bit format of V: fp16 when V is the normalised key copy, bf16 when V
    // is the caller's values
    const bool pf16 = a.kv_is_k != 0;
    if (a.d == 512) return pf16 ? run_prefill<512, true>(a, stream) : run_prefill<512, false>(a, stream);
    if (a.d == 256) return pf16 ? run_prefill<256, true>(a, stream) : run_prefill<256, false>(a, stream);
    return cudaErrorInvalidValue;
}

}  // namespace g4

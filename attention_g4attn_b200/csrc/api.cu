// api.cu -- the C ABI of g4attn: argument validation, workspace layout, TMA tensor-map
// encoding and stream-ordered launches.  No device memory is allocated here.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "g4attn.h"
#include "kernels.h"

namespace g4 {
// int8 KV cache writer (quant.cu): rows of d bf16 elements -> d int8 codes + one fp32 scale
cudaError_t launch_quantize_int8(const uint16_t* x, int8_t* codes, float* scales, long long rows,
                                 int d, cudaStream_t stream);
}  // namespace g4

namespace {

__device__ int g_device_status = 0;   // written by bounded waits that give up

constexpr long long kDefaultWaitLimit = 1LL << 62;   // polls; the 2 s time bound rules
std::atomic<long long> g_wait_limit{kDefaultWaitLimit};

constexpr int kMaxDevices = 64;
struct DeviceInfo {
    bool probed = false;
    bool supported = false;
    int sms = 0;
    unsigned long long ctx_id = 0;   // id of the context the addresses below belong to
    int* status = nullptr;           // device address of g_device_status
    void* scratch = nullptr;         // device address of the no-alloc decode's scratch
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);
EncodeTiledFn g_encode = nullptr;
CtxGetCurrentFn g_ctx_current = nullptr;
CtxGetIdFn g_ctx_id = nullptr;

template <typename F>
F driver_fn(const char* name) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        return reinterpret_cast<F>(fn);
    cudaGetLastError();
    return nullptr;
}

// Unique id of the current CUDA context (0 if it cannot be read).  Device addresses of the
// library's __device__ variables belong to a context: after cudaDeviceReset the runtime
// creates a new primary context and the module's variables move, so addresses are cached
// together with this id and looked up again when it changes.
unsigned long long current_ctx_id() {
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!g_ctx_current || !g_ctx_id || g_ctx_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
    if (g_ctx_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Probe the current device: compute capability 10.0, SM count, and the device addresses of
// the status word and the no-alloc scratch (once per device and context).
int current_device(DeviceInfo** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return G4ATTN_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_encode) {
        g_encode = driver_fn<EncodeTiledFn>("cuTensorMapEncodeTiled");
        g_ctx_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
        g_ctx_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
    }
    DeviceInfo& d = g_dev[dev];
    if (!d.probed) {
        d.probed = true;
        int major = 0, minor = 0;
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
        d.supported = (major == 10 && minor == 0) && g_encode != nullptr;
        cudaGetLastError();
    }
    if (!d.supported) return G4ATTN_ERR_UNSUPPORTED;
    const unsigned long long ctx = current_ctx_id();
    if (!d.status || ctx == 0 || ctx != d.ctx_id) {
        void* p = nullptr;
        void* s = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess ||
            g4::decode_scratch_ptr(&s) != cudaSuccess) {
            cudaGetLastError();
            return G4ATTN_ERR_CUDA;
        }
        d.status = static_cast<int*>(p);
        d.scratch = s;
        d.ctx_id = ctx;
    }
    *out = &d;
    return G4ATTN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int rope_pairs(const g4attn_layer_cfg* c) {
    double r = std::floor((double)c->rope_p * (double)c->head_dim / 2.0);
    if (r < 0) r = 0;
    if (r > c->head_dim / 2) r = c->head_dim / 2;
    return (int)r;
}

bool chunk_rotated(int c, int d, int R) {
    const int lo = c * 64, hi = lo + 64, h = d / 2;
    return (lo < R) || (lo < h + R && hi > h);
}

// Configuration checks shared by every entry point.
int check_cfg(const g4attn_layer_cfg* c, bool tensor_core_path) {
    if (!c) return G4ATTN_ERR_INVALID_ARG;
    if (c->n_q_heads <= 0 || c->n_kv_heads <= 0 || c->n_q_heads % c->n_kv_heads != 0)
        return G4ATTN_ERR_INVALID_ARG;
    if (c->head_dim <= 0 || (c->head_dim & 1)) return G4ATTN_ERR_INVALID_ARG;
    if (!(c->rope_p >= 0.f && c->rope_p <= 1.f)) return G4ATTN_ERR_INVALID_ARG;
    if (!(c->rope_base > 0.0) || !std::isfinite(c->rope_base)) return G4ATTN_ERR_INVALID_ARG;
    if (c->window < 0) return G4ATTN_ERR_INVALID_ARG;
    if (!std::isfinite(c->scale) || !(c->scale > 0.f)) return G4ATTN_ERR_INVALID_ARG;
    if (c->kv_is_k < 0 || c->kv_is_k > 2) return G4ATTN_ERR_INVALID_ARG;
    if (c->qk_norm != 0 && c->qk_norm != 1) return G4ATTN_ERR_INVALID_ARG;
    if (c->qk_norm && !(c->qk_norm_eps >= 0.f)) return G4ATTN_ERR_INVALID_ARG;
    if (tensor_core_path) {
        if (c->head_dim != 256 && c->head_dim != 512) return G4ATTN_ERR_UNSUPPORTED;
        const int G = c->n_q_heads / c->n_kv_heads;
        if (128 % G != 0) return G4ATTN_ERR_UNSUPPORTED;
    } else if (c->head_dim != 128 && c->head_dim != 256 && c->head_dim != 512) {
        return G4ATTN_ERR_UNSUPPORTED;
    }
    return G4ATTN_OK;
}

// 4-D map over a [B, T, H, d] 16-bit tensor: dims (d, H, T, B), box (64, 1, box_rows, 1),
// 128-byte swizzle, zero fill outside the tensor.
// `T_phys` (default T): rows per batch in memory, when only the first T are exposed (rows
// from T on read as zero).
int encode_rows(CUtensorMap* m, const void* base, int B, int T, int H, int d, bool f16 = false,
                int box_rows = 128, int T_phys = 0) {
    const cuuint64_t tp = (cuuint64_t)(T_phys > 0 ? T_phys : T);
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, tp * H * d * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    CUresult r = g_encode(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                          4, const_cast<void*>(base), dims,
                          strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? G4ATTN_OK : G4ATTN_ERR_CUDA;
}

// 4-D map over an int8 cache [B, T, H, d] as (d, H, T, B), box (64, 1, 64, 1) (64-byte rows),
// 64-byte swizzle, zero fill; `T_phys` as in encode_rows.
int encode_rows_i8(CUtensorMap* m, const void* base, int B, int T, int H, int d, int T_phys) {
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)d, (cuuint64_t)H * d, (cuuint64_t)T_phys * H * d};
    cuuint32_t box[4] = {64, 1, 64, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims,
                          strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? G4ATTN_OK : G4ATTN_ERR_CUDA;
}

// 4-D map over the raw queries [B, T, Hq, d] as (d, Hq, T, B) with box (64, G, 128 / G, 1):
// one box is a 64-dim chunk of a packed row tile (row = token * G + head), 128-byte swizzle.
int encode_q_tile(CUtensorMap* m, const void* q, int B, int T, int Hq, int d, int G) {
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)Hq, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)Hq * d * 2, (cuuint64_t)T * Hq * d * 2};
    cuuint32_t box[4] = {64, (cuuint32_t)G, (cuuint32_t)(128 / G), 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(q), dims, strides,
                          box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? G4ATTN_OK : G4ATTN_ERR_CUDA;
}

// 2-D map over the [T, R] (cos, sin) table as fp32 (2R, T), box (2R, rows).
int encode_cs_rows(CUtensorMap* m, const float2* cs, int T, int R, int rows) {
    cuuint64_t dims[2] = {(cuuint64_t)(2 * R), (cuuint64_t)T};
    cuuint64_t strides[1] = {(cuuint64_t)R * 8};
    cuuint32_t box[2] = {(cuuint32_t)(2 * R), (cuuint32_t)rows};
    cuuint32_t es[2] = {1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float2*>(cs), dims, strides,
                          box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? G4ATTN_OK : G4ATTN_ERR_CUDA;
}

struct PrefillWs {
    size_t kn_off, kr_off, cs_off, v_off, total;
    bool need_kn;
};

// Workspace of an attention pass over Tk key rows per batch: the fp16 normalised keys
// (pre-RoPE copy when some chunk is unrotated or the keys are the values, rotated copy),
// the (cos, sin) table of the Tk positions and, with v_copy, a bf16 copy of the values.
PrefillWs prefill_ws(int B, long long Tk, const g4attn_layer_cfg* c, bool v_copy = false) {
    PrefillWs w{};
    const int d = c->head_dim, R = rope_pairs(c);
    bool any_plain = false;
    for (int ch = 0; ch < d / 64; ++ch) any_plain |= !chunk_rotated(ch, d, R);
    w.need_kn = any_plain || c->kv_is_k == 1;
    const size_t rows = (size_t)B * Tk * c->n_kv_heads * d * 2;
    w.kn_off = 0;
    w.kr_off = w.need_kn ? align256(rows) : 0;
    w.cs_off = w.kr_off + align256(rows);
    w.v_off = w.cs_off + align256((size_t)Tk * (R > 0 ? R : 1) * sizeof(float2));
    w.total = w.v_off + (v_copy && c->kv_is_k == 0 ? align256(rows) : 0);
    return w;
}

constexpr int kDecodeTile = 128;   // keys per decode pair-tile

// Stream-K split of a decode step: the B * Hkv sequences' pair-tiles form one flat range
// of W tiles, cut evenly over P CTA pairs; a sequence is split into one segment per pair
// that touches it, and every segment leaves two partials (one per CTA of its pair).
struct DecodePlan {
    int key_lo, tile_base, splits, tiles_per_seq, n_pairs;
    long long total_tiles;
    size_t o_off, ml_off, total;
};

// Most segments any sequence is cut into when W tiles (nt per sequence) go to P pairs.
int max_segments(long long W, int nt, int nbg, int P) {
    if (W <= 0 || P <= 0) return 0;
    auto pair_of = [&](long long t) { return (int)(((t + 1) * P - 1) / W); };
    int m = 0;
    for (int bg = 0; bg < nbg; ++bg) {
        const long long s0 = (long long)bg * nt;
        const int n = pair_of(s0 + nt - 1) - pair_of(s0) + 1;
        m = n > m ? n : m;
    }
    return m;
}

// ring > 0: the cache is a ring of `ring` rows (position p in row p % ring); the tiles then
// start at the 64-aligned position at or below the window start, so no 64-key box wraps.
DecodePlan decode_plan(int B, int L, const g4attn_layer_cfg* c, int sms, int max_pairs = 0,
                       int ring = 0) {
    DecodePlan p{};
    p.key_lo = (c->window > 0 && L > c->window) ? L - c->window : 0;
    p.tile_base = ring > 0 ? p.key_lo / 64 * 64 : p.key_lo;
    const int len = L - p.tile_base;
    const int nbg = B * c->n_kv_heads;
    p.tiles_per_seq = len > 0 ? (len + kDecodeTile - 1) / kDecodeTile : 0;
    p.total_tiles = (long long)nbg * p.tiles_per_seq;
    long long P = (sms > 1 ? sms : 148) / 2;   // the decode kernel runs on CTA pairs
    if (max_pairs > 0 && P > max_pairs) P = max_pairs;
    if (P > p.total_tiles) P = p.total_tiles;
    p.n_pairs = (int)P;
    p.splits = max_segments(p.total_tiles, p.tiles_per_seq, nbg, p.n_pairs);
    const size_t n = 2 * (size_t)(p.splits > 0 ? p.splits : 1) * B * c->n_q_heads;
    p.o_off = 0;
    p.ml_off = align256(n * c->head_dim * sizeof(float));
    p.total = p.ml_off + align256(n * 2 * sizeof(float));
    return p;
}

g4::Rope make_rope(const g4attn_layer_cfg* c) {
    g4::Rope r;
    r.R = rope_pairs(c);
    r.log2_base = std::log2(c->rope_base);
    return r;
}

int cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return G4ATTN_OK;
    cudaGetLastError();
    return G4ATTN_ERR_CUDA;
}

// Argument checks shared by the decode entry points (before any launch).
int check_decode(const g4attn_bf16* q, const g4attn_bf16* kcache, const g4attn_bf16* vcache,
                 int L, const g4attn_bf16* out, const float* lse, int B,
                 const g4attn_layer_cfg* cfg) {
    int rc = check_cfg(cfg, true);
    if (rc) return rc;
    if (B < 0 || L < 0) return G4ATTN_ERR_INVALID_ARG;
    if (B > 0 && (!q || !out || (L > 0 && !kcache))) return G4ATTN_ERR_INVALID_ARG;
    if ((cfg->kv_is_k == 0) != (vcache != nullptr)) return G4ATTN_ERR_INVALID_ARG;
    const int G = cfg->n_q_heads / cfg->n_kv_heads;
    if (G > 16) return G4ATTN_ERR_UNSUPPORTED;
    if (cfg->kv_is_k == 1) {   // the turned slot of a tile must be a single slot (R <= 64)
        const int R = rope_pairs(cfg);
        int n = 0;
        for (int c = 0; c < cfg->head_dim / 64; ++c) n += chunk_rotated(c, cfg->head_dim, R);
        if (n > 2) return G4ATTN_ERR_UNSUPPORTED;
    }
    const void* ptrs[] = {q, kcache, vcache, out, lse};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return G4ATTN_ERR_MISALIGNED;
    return G4ATTN_OK;
}

// Fills the decode arguments for a planned call and launches decode + combine.
// `rows`: cache rows in memory (L for a linear cache, C for a ring); `ring`: 0 or C.  A ring
// that is not full yet (L < C) exposes only its first L rows to the copies: the last tile's
// positions past L then read zeros instead of never-written rows (whose values, times a zero
// weight, could still be NaN).
int launch_decode_plan(const g4attn_bf16* q, const g4attn_bf16* kcache,
                       const g4attn_bf16* vcache, int L, int rows, int ring, g4attn_bf16* out,
                       float* lse, uint8_t* w, const DecodePlan& plan, int B,
                       const g4attn_layer_cfg* cfg, const DeviceInfo* dev, g4attn_stream_t stream,
                       const g4attn_bf16* vside = nullptr, bool keys_rotated = false,
                       const int8_t* kcodes = nullptr, const float* kscale = nullptr,
                       const int8_t* vcodes = nullptr, const float* vscale = nullptr) {
    g4::DecodeArgs a{};
    const int d = cfg->head_dim, Hkv = cfg->n_kv_heads;
    int rc;
    if (L > 0) {
        const int seen = L < rows ? L : rows;   // rows that hold positions
        if (kcodes) {
            if ((rc = encode_rows_i8(&a.tm_k, kcodes, B, seen, Hkv, d, rows))) return rc;
            if ((rc = encode_rows_i8(&a.tm_v, vcodes ? vcodes : kcodes, B, seen, Hkv, d, rows)))
                return rc;
        } else {
            if ((rc = encode_rows(&a.tm_k, kcache, B, seen, Hkv, d, false, 64, rows))) return rc;
            if ((rc = encode_rows(&a.tm_v, vcache ? vcache : kcache, B, seen, Hkv, d, false, 64,
                                  rows)))
                return rc;
        }
    }
    if (kcodes) {
        a.int8 = 1;
        a.kscale = kscale;
        a.vscale = vscale ? vscale : kscale;
    }
    a.q = q;
    a.part_o = reinterpret_cast<float*>(w + plan.o_off);
    a.part_ml = reinterpret_cast<float*>(w + plan.ml_off);
    a.out = out;
    a.lse = lse;
    a.B = B; a.L = L; a.Hq = cfg->n_q_heads; a.Hkv = Hkv; a.d = d;
    a.G = cfg->n_q_heads / Hkv;
    a.key_lo = plan.key_lo;
    a.tile_base = plan.tile_base;
    a.ring = ring;
    a.splits = plan.splits;
    a.tiles_per_seq = plan.tiles_per_seq;
    a.n_pairs = plan.n_pairs;
    a.total_tiles = plan.total_tiles;
    a.rope = make_rope(cfg);
    if (vside) {
        // split cache: keys arrive rotated, so the kernel turns nothing (R = 0); slot 0's
        // values come from the side copy of the 2R = 128 rotated dims
        if (L > 0) {
            const int seen = L < rows ? L : rows;
            if ((rc = encode_rows(&a.tm_vside, vside, B, seen, Hkv, 128, false, 64, rows)))
                return rc;
        }
        a.split_cache = 1;
        a.rope.R = 0;
    }
    if (keys_rotated) a.rope.R = 0;   // keys stored turned to their positions: no turning
    a.scale_log2 = cfg->scale * 1.4426950408889634f;
    a.kv_is_k = cfg->kv_is_k;
    a.wait_limit = g_wait_limit.load();
    a.status = dev->status;
    return cuda_status(g4::launch_decode(a, reinterpret_cast<cudaStream_t>(stream)));
}

// A ring cache holds the last C positions, C a positive multiple of 64 (pair-tile halves
// never wrap), and must hold the whole window.
int check_ring(int C, const g4attn_layer_cfg* cfg) {
    if (!cfg || C <= 0 || C % 64 != 0) return G4ATTN_ERR_INVALID_ARG;
    if (cfg->window <= 0 || cfg->window > C) return G4ATTN_ERR_INVALID_ARG;
    return G4ATTN_OK;
}

// The fused flash-attention kernel over prepared key rows: kn / kr [B, Tk, Hkv, d] fp16
// (kn may be null when no chunk needs it), v [B, Tk, Hkv, d] bf16 separate values or null,
// cs [Tk, R] (cos, sin); query token t of the T in q sits at key row q_off + t.
int launch_attention(const g4attn_bf16* q, const uint16_t* kn, const uint16_t* kr,
                     const g4attn_bf16* v, const float2* cs, const float* gamma_q,
                     g4attn_bf16* out, float* lse, int B, int T, int Tk, int q_off,
                     const g4attn_layer_cfg* cfg, DeviceInfo* dev, cudaStream_t st) {
    int rc;
    const int d = cfg->head_dim, Hkv = cfg->n_kv_heads;
    g4::PrefillArgs a{};
    const uint16_t* kn_or_kr = kn ? kn : kr;
    if ((rc = encode_rows(&a.tm_kr_s, kr, B, Tk, Hkv, d, true, 64))) return rc;
    if ((rc = encode_rows(&a.tm_kn_s, kn_or_kr, B, Tk, Hkv, d, true, 64))) return rc;
    if ((rc = encode_rows(&a.tm_kr_v, kr, B, Tk, Hkv, d, true, 128))) return rc;
    if ((rc = encode_rows(&a.tm_kn_v, kn_or_kr, B, Tk, Hkv, d, true, 128))) return rc;
    if (v) rc = encode_rows(&a.tm_v, v, B, Tk, Hkv, d, false, 128);
    else rc = encode_rows(&a.tm_v, kn_or_kr, B, Tk, Hkv, d, true, 128);
    if (rc) return rc;
    const int G = cfg->n_q_heads / Hkv;
    if ((rc = encode_q_tile(&a.tm_q, q, B, T, cfg->n_q_heads, d, G))) return rc;
    {
        // the (cos, sin) rows of a row tile go to shared memory by TMA when they fit the
        // staging room (free during the prologue) and the row pitch suits TMA
        const int R = rope_pairs(cfg), rows = 128 / G;
        const size_t bytes = (size_t)rows * R * 8;
        a.cs_tma = R > 0 && R % 2 == 0 && 2 * R <= 256 && rows <= 256 &&
                   bytes <= g4::prefill_cs_stage_bytes(d);
        if (a.cs_tma && (rc = encode_cs_rows(&a.tm_cs, cs, Tk, R, rows))) return rc;
    }
    a.q = q;
    a.gamma_q = gamma_q;
    a.rope_cs = cs;
    a.out = out;
    a.lse = lse;
    a.B = B; a.T = T; a.Hq = cfg->n_q_heads; a.Hkv = Hkv; a.d = d;
    a.Tk = Tk;
    a.q_off = q_off;
    a.G = G;
    a.window = cfg->window;
    a.rope = make_rope(cfg);
    a.qk_norm = cfg->qk_norm;
    a.eps = cfg->qk_norm_eps;
    a.scale_log2 = cfg->scale * 1.4426950408889634f;
    a.kv_is_k = cfg->kv_is_k;
    a.wait_limit = g_wait_limit.load();
    a.status = dev->status;
    return cuda_status(g4::launch_prefill(a, st));
}


// Key rows of a prefill chunk: positions kb .. P + Tn - 1, where kb is the first position
// any of the chunk's queries can see (0 on causal layers, P - W + 1 on window-W layers).
struct ChunkFrame {
    long long kb;
    int Tk, q_off;
};

ChunkFrame chunk_frame(int P, int Tn, const g4attn_layer_cfg* c) {
    ChunkFrame f{};
    f.kb = c->window > 0 ? std::max(0, P - c->window + 1) : 0;
    f.Tk = (int)(P + (long long)Tn - f.kb);
    f.q_off = (int)(P - f.kb);
    return f;
}

int check_chunk(int B, int P, int Tn, int cache_rows, int flags, const g4attn_layer_cfg* c) {
    if (B < 0 || P < 0 || Tn < 0 || cache_rows <= 0) return G4ATTN_ERR_INVALID_ARG;
    if ((long long)P + Tn > INT_MAX / 2) return G4ATTN_ERR_INVALID_ARG;
    if (flags & ~(G4ATTN_CACHE_RING | G4ATTN_CACHE_ROTATED)) return G4ATTN_ERR_INVALID_ARG;
    if ((flags & G4ATTN_CACHE_ROTATED) && c->kv_is_k != 0) return G4ATTN_ERR_INVALID_ARG;
    const bool ring = (flags & G4ATTN_CACHE_RING) != 0;
    if (!ring && (long long)P + Tn > cache_rows) return G4ATTN_ERR_INVALID_ARG;
    if (ring && (c->window <= 0 || c->window > cache_rows)) return G4ATTN_ERR_INVALID_ARG;
    return G4ATTN_OK;
}

}  // namespace

extern "C" {

const char* g4attn_version(void) { return "g4attn 0.1 (sm_100a)"; }

const char* g4attn_status_string(int s) {
    switch (s) {
        case G4ATTN_OK: return "ok";
        case G4ATTN_ERR_INVALID_ARG: return "invalid argument";
        case G4ATTN_ERR_UNSUPPORTED: return "unsupported configuration or device";
        case G4ATTN_ERR_MISALIGNED: return "pointer not 16-byte aligned";
        case G4ATTN_ERR_WORKSPACE: return "workspace missing or too small";
        case G4ATTN_ERR_CUDA: return "CUDA error";
        case G4ATTN_ERR_TIMEOUT: return "device wait timed out";
        case G4ATTN_ERR_TOO_LARGE:
            return "problem needs more than the fixed 8 MiB scratch of g4attn_decode_noalloc";
        default: return "unknown status";
    }
}

int g4attn_wait_selftest(long long polls, g4attn_stream_t stream) {
    DeviceInfo* dev = nullptr;
    const int rc = current_device(&dev);
    if (rc) return rc;
    const long long limit = polls < 1 ? g_wait_limit.load() : polls;
    return cuda_status(g4::launch_wait_selftest(dev->status, limit,
                                                reinterpret_cast<cudaStream_t>(stream)));
}

long long g4attn_set_wait_limit(long long polls) {
    return g_wait_limit.exchange(polls < 1 ? kDefaultWaitLimit : polls);
}

int g4attn_device_status(g4attn_stream_t stream) {
    DeviceInfo* dev = nullptr;
    int rc = current_device(&dev);
    if (rc) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return cuda_status(cudaErrorUnknown);
    int v = 0;
    if (cudaMemcpy(&v, dev->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return cuda_status(cudaErrorUnknown);
    const int zero = 0;
    if (cudaMemcpy(dev->status, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
        return cuda_status(cudaErrorUnknown);
    return v;
}

int g4attn_qknorm_rope(const g4attn_bf16* q_in, const g4attn_bf16* k_in, g4attn_bf16* q_out,
                       g4attn_bf16* kcache_out, g4attn_bf16* krot_out, const float* gamma_q,
                       const float* gamma_k, int B, int T, long long pos0,
                       const g4attn_layer_cfg* cfg, g4attn_stream_t stream) {
    int rc = check_cfg(cfg, false);
    if (rc) return rc;
    if (B < 0 || T < 0 || pos0 < 0) return G4ATTN_ERR_INVALID_ARG;
    if ((q_in && !q_out) || (k_in && !kcache_out && !krot_out)) return G4ATTN_ERR_INVALID_ARG;
    if (cfg->qk_norm && ((q_in && !gamma_q) || (k_in && !gamma_k))) return G4ATTN_ERR_INVALID_ARG;
    const void* ptrs[] = {q_in, k_in, q_out, kcache_out, krot_out, gamma_q, gamma_k};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return G4ATTN_ERR_MISALIGNED;
    if ((long long)B * T == 0 || (!q_in && !k_in)) return G4ATTN_OK;
    DeviceInfo* dev = nullptr;
    if ((rc = current_device(&dev))) return rc;
    g4::QkNormRopeArgs a{};
    a.q_in = q_in;
    a.k_in = k_in;
    a.q_out = q_out;
    a.k_out = k_in ? kcache_out : nullptr;
    a.krot_out = k_in ? krot_out : nullptr;
    a.gamma_q = gamma_q;
    a.gamma_k = gamma_k;
    a.cs_out = nullptr;
    a.B = B; a.T = T; a.Hq = cfg->n_q_heads; a.Hkv = cfg->n_kv_heads; a.d = cfg->head_dim;
    a.pos0 = pos0;
    a.rope = make_rope(cfg);
    a.qk_norm = cfg->qk_norm;
    a.eps = cfg->qk_norm_eps;
    return cuda_status(g4::launch_qknorm_rope(a, reinterpret_cast<cudaStream_t>(stream)));
}

size_t g4attn_prefill_workspace_size(int B, int T, const g4attn_layer_cfg* cfg) {
    if (check_cfg(cfg, true) || B < 0 || T < 0) return 0;
    return prefill_ws(B, T, cfg).total;
}

int g4attn_prefill(const g4attn_bf16* q, const g4attn_bf16* k, const g4attn_bf16* v,
                   const float* gamma_q, const float* gamma_k, g4attn_bf16* out, float* lse,
                   void* workspace, size_t ws_bytes, int B, int T, const g4attn_layer_cfg* cfg,
                   g4attn_stream_t stream) {
    int rc = check_cfg(cfg, true);
    if (rc) return rc;
    if (B < 0 || T < 0) return G4ATTN_ERR_INVALID_ARG;
    if ((long long)B * T == 0) return G4ATTN_OK;
    if (!q || !k || !out) return G4ATTN_ERR_INVALID_ARG;
    if ((cfg->kv_is_k == 0) != (v != nullptr)) return G4ATTN_ERR_INVALID_ARG;
    if (cfg->qk_norm && (!gamma_q || !gamma_k)) return G4ATTN_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, gamma_q, gamma_k, out, lse};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return G4ATTN_ERR_MISALIGNED;
    const PrefillWs ws = prefill_ws(B, T, cfg);
    if (!workspace || ws_bytes < ws.total) return G4ATTN_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return G4ATTN_ERR_MISALIGNED;
    DeviceInfo* dev = nullptr;
    if ((rc = current_device(&dev))) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* w = static_cast<uint8_t*>(workspace);
    uint16_t* kn = ws.need_kn ? reinterpret_cast<uint16_t*>(w + ws.kn_off) : nullptr;
    uint16_t* kr = reinterpret_cast<uint16_t*>(w + ws.kr_off);
    float2* cs = reinterpret_cast<float2*>(w + ws.cs_off);
    const int d = cfg->head_dim, Hkv = cfg->n_kv_heads;

    // 1) normalise the keys once: pre-RoPE copy (the K(=V) values) and the rotated copy,
    //    both fp16, plus the (cos, sin) table of every position for the query prologue
    g4::QkNormRopeArgs ka{};
    ka.k_in = k;
    ka.k_out = kn;
    ka.krot_out = kr;
    ka.gamma_k = gamma_k;
    ka.cs_out = cs;
    ka.k_f16 = 1;   // the prefill keeps its normalised key copies in fp16
    ka.B = B; ka.T = T; ka.Hq = cfg->n_q_heads; ka.Hkv = Hkv; ka.d = d;
    ka.pos0 = 0;
    ka.rope = make_rope(cfg);
    ka.qk_norm = cfg->qk_norm;
    ka.eps = cfg->qk_norm_eps;
    if ((rc = cuda_status(g4::launch_qknorm_rope(ka, st)))) return rc;

    // 2) the fused flash-attention kernel
    return launch_attention(q, kn, kr, v, cs, gamma_q, out, lse, B, T, T, 0, cfg, dev, st);
}

size_t g4attn_prefill_chunk_workspace_size(int B, int P, int Tn, const g4attn_layer_cfg* cfg) {
    if (check_cfg(cfg, true) || B < 0 || P < 0 || Tn < 0) return 0;
    if ((long long)P + Tn > INT_MAX / 2) return 0;
    return prefill_ws(B, chunk_frame(P, Tn, cfg).Tk, cfg, true).total;
}

int g4attn_prefill_chunk(const g4attn_bf16* q, const g4attn_bf16* k, const g4attn_bf16* v,
                         const float* gamma_q, const float* gamma_k, g4attn_bf16* kcache,
                         g4attn_bf16* vcache, int cache_rows, int cache_flags, g4attn_bf16* out,
                         float* lse, void* workspace, size_t ws_bytes, int B, int P, int Tn,
                         const g4attn_layer_cfg* cfg, g4attn_stream_t stream) {
    int rc = check_cfg(cfg, true);
    if (rc) return rc;
    if ((rc = check_chunk(B, P, Tn, cache_rows, cache_flags, cfg))) return rc;
    const bool ring = (cache_flags & G4ATTN_CACHE_RING) != 0;
    const bool rotated = (cache_flags & G4ATTN_CACHE_ROTATED) != 0;
    if ((long long)B * Tn == 0) return G4ATTN_OK;
    if (!q || !k || !out || !kcache) return G4ATTN_ERR_INVALID_ARG;
    const bool sep_v = cfg->kv_is_k == 0;
    if (sep_v != (v != nullptr) || sep_v != (vcache != nullptr)) return G4ATTN_ERR_INVALID_ARG;
    if (cfg->qk_norm && (!gamma_q || !gamma_k)) return G4ATTN_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, gamma_q, gamma_k, kcache, vcache, out, lse};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return G4ATTN_ERR_MISALIGNED;
    const ChunkFrame f = chunk_frame(P, Tn, cfg);
    const PrefillWs ws = prefill_ws(B, f.Tk, cfg, true);
    if (!workspace || ws_bytes < ws.total) return G4ATTN_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return G4ATTN_ERR_MISALIGNED;
    DeviceInfo* dev = nullptr;
    if ((rc = current_device(&dev))) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* w = static_cast<uint8_t*>(workspace);
    uint16_t* kn = ws.need_kn ? reinterpret_cast<uint16_t*>(w + ws.kn_off) : nullptr;
    uint16_t* kr = reinterpret_cast<uint16_t*>(w + ws.kr_off);
    float2* cs = reinterpret_cast<float2*>(w + ws.cs_off);
    uint16_t* vf = sep_v ? reinterpret_cast<uint16_t*>(w + ws.v_off) : nullptr;

    // the key rows of both passes land in one frame of Tk rows per batch, row = position - kb
    g4::QkNormRopeArgs ka{};
    ka.k_out = kn;
    ka.krot_out = kr;
    ka.cs_out = cs;
    ka.v_out = vf;
    ka.k_f16 = 1;
    ka.B = B; ka.Hq = cfg->n_q_heads; ka.Hkv = cfg->n_kv_heads; ka.d = cfg->head_dim;
    ka.rope = make_rope(cfg);
    ka.eps = cfg->qk_norm_eps;
    ka.out_rows = f.Tk;
    ka.out_base = f.kb;

    // 1) the cached positions kb .. P-1: stored normalised, so only turned (and widened); a
    //    cache of turned keys is only widened (its (cos, sin) rows are not needed: the
    //    queries sit at rows q_off and later)
    if (P > f.kb) {
        g4::QkNormRopeArgs ca = ka;
        ca.k_in = kcache;
        ca.v_in = vcache;
        ca.in_rows = cache_rows;
        ca.in_ring = ring ? cache_rows : 0;
        ca.in_base = 0;
        ca.pos0 = f.kb;
        ca.T = (int)(P - f.kb);
        ca.qk_norm = 0;
        if (rotated) ca.rope.R = 0;
        if ((rc = cuda_status(g4::launch_qknorm_rope(ca, st)))) return rc;
    }
    // 2) the chunk's own keys: QKNorm, RoPE, and appended to the cache (values too)
    {
        g4::QkNormRopeArgs na = ka;
        na.k_in = k;
        na.v_in = v;
        na.gamma_k = gamma_k;
        na.in_rows = Tn;
        na.in_base = P;
        na.pos0 = P;
        na.T = Tn;
        na.qk_norm = cfg->qk_norm;
        na.kc_out = kcache;
        na.vc_out = vcache;
        na.kc_rows = cache_rows;
        na.kc_ring = ring ? cache_rows : 0;
        na.kc_rot = rotated ? 1 : 0;
        if ((rc = cuda_status(g4::launch_qknorm_rope(na, st)))) return rc;
    }
    // 3) attention of the chunk's queries (key row q_off + t) over the frame
    return launch_attention(q, kn, kr, vf, cs, gamma_q, out, lse, B, Tn, f.Tk, f.q_off, cfg,
                            dev, st);
}

size_t g4attn_decode_workspace_size(int B, int L, const g4attn_layer_cfg* cfg) {
    if (check_cfg(cfg, true) || B < 0 || L < 0) return 0;
    DeviceInfo* dev = nullptr;
    int sms = 148;
    if (current_device(&dev) == G4ATTN_OK) sms = dev->sms;
    else cudaGetLastError();
    return decode_plan(B, L, cfg, sms).total;
}

int g4attn_decode(const g4attn_bf16* q, const g4attn_bf16* kcache, const g4attn_bf16* vcache,
                  int L, g4attn_bf16* out, float* lse, void* workspace, size_t ws_bytes, int B,
                  const g4attn_layer_cfg* cfg, g4attn_stream_t stream) {
    int rc = check_decode(q, kcache, vcache, L, out, lse, B, cfg);
    if (rc) return rc;
    if (B == 0) return G4ATTN_OK;
    DeviceInfo* dev = nullptr;
    if ((rc = current_device(&dev))) return rc;
    const DecodePlan plan = decode_plan(B, L, cfg, dev->sms);
    if (!workspace || ws_bytes < plan.total) return G4ATTN_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return G4ATTN_ERR_MISALIGNED;
    return launch_decode_plan(q, kcache, vcache, L, L, 0, out, lse,
                              static_cast<uint8_t*>(workspace), plan, B, cfg, dev, stream);
}

size_t g4attn_decode_int8_workspace_size(int B, int L, int C, const g4attn_layer_cfg* cfg) {
    return g4attn_decode_rotated_workspace_size(B, L, C, cfg);
}

int g4attn_decode_int8(const g4attn_bf16* q, const int8_t* kcodes, const float* kscales,
                       const int8_t* vcodes, const float* vscales, int L, int C,
                       g4attn_bf16* out, float* lse, void* workspace, size_t ws_bytes, int B,
                       const g4attn_layer_cfg* cfg, g4attn_stream_t stream) {
    // the bf16 decode's checks, on the code tensors' pointers
    int rc = check_decode(q, reinterpret_cast<const g4attn_bf16*>(kcodes),
                          reinterpret_cast<const g4attn_bf16*>(vcodes), L, out, lse, B, cfg);
    if (rc) return rc;
    if (cfg->n_q_heads / cfg->n_kv_heads > 8) return G4ATTN_ERR_UNSUPPORTED;
    if ((vcodes != nullptr) != (vscales != nullptr)) return G4ATTN_ERR_INVALID_ARG;
    if (B > 0 && L > 0 && !kscales) return G4ATTN_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(kscales) & 3u) || (reinterpret_cast<uintptr_t>(vscales) & 3u))
        return G4ATTN_ERR_MISALIGNED;
    if (C < 0) return G4ATTN_ERR_INVALID_ARG;
    if (C > 0 && (rc = check_ring(C, cfg))) return rc;
    if (B == 0) return G4ATTN_OK;
    DeviceInfo* dev = nullptr;
    if ((rc = current_device(&dev))) return rc;
    const DecodePlan plan = decode_plan(B, L, cfg, dev->sms, 0, C);
    if (!workspace || ws_bytes < plan.total) return G4ATTN_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return G4ATTN_ERR_MISALIGNED;
    return launch_decode_plan(q, nullptr, nullptr, L, C > 0 ? C : L, C, out, lse,
                              static_cast<uint8_t*>(workspace), plan, B, cfg, dev, stream,
                              nullptr, false, kcodes, kscales, vcodes, vscales);
}

int g4attn_decode_split_cache(const g4attn_bf16* q, const g4attn_bf16* krot,
                              const g4attn_bf16* vside, int L, g4attn_bf16* out, float* lse,
                              void* workspace, size_t ws_bytes, int B, const g4attn_layer_cfg* cfg,
                              g4attn_stream_t stream) {
    int rc = check_decode(q, krot, nullptr, L, out, lse, B, cfg);
    if (rc) return rc;
    if (cfg->kv_is_k != 1 || rope_pairs(cfg) != 64) return G4ATTN_ERR_UNSUPPORTED;
    if (B > 0 && L > 0 && !vside) return G4ATTN_ERR_INVALID_ARG;
    if (vside && !aligned16(vside)) return G4ATTN_ERR_MISALIGNED;
    if (B == 0) return G4ATTN_OK;
    DeviceInfo* dev = nullptr;
    if ((rc = current_device(&dev))) return rc;
    const DecodePlan plan = decode_plan(B, L, cfg, dev->sms);
    if (!workspace || ws_bytes < plan.total) return G4ATTN_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return G4ATTN_ERR_MISALIGNED;
    return launch_decode_plan(q, krot, nullptr, L, L, 0, out, lse,
                              static_cast<uint8_t*>(workspace), plan, B, cfg, dev, stream, vside);
}

size_t g4attn_decode_ring_workspace_size(int B, int L, int C, const g4attn_layer_cfg* cfg) {
    if (check_cfg(cfg, true) || check_ring(C, cfg) || B < 0 || L < 0) return 0;
    DeviceInfo* dev = nullptr;
    int sms = 148;
    if (current_device(&dev) == G4ATTN_OK) sms = dev->sms;
    else cudaGetLastError();
    return decode_plan(B, L, cfg, sms, 0, C).total;
}

int g4attn_decode_ring(const g4attn_bf16* q, const g4attn_bf16* kring, const g4attn_bf16* vring,
                       int L, int C, g4attn_bf16* out, float* lse, void* workspace,
                       size_t ws_bytes, int B, const g4attn_layer_cfg* cfg,
                       g4attn_stream_t stream) {
    int rc = check_decode(q, kring, vring, L, out, lse, B, cfg);
    if (rc) return rc;
    if ((rc = check_ring(C, cfg))) return rc;
    if (B == 0) return G4ATTN_OK;
    DeviceInfo* dev = nullptr;
    if ((rc = current_device(&dev))) return rc;
    const DecodePlan plan = decode_plan(B, L, cfg, dev->sms, 0, C);
    if (!workspace || ws_bytes < plan.total) return G4ATTN_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return G4ATTN_ERR_MISALIGNED;
    return launch_decode_plan(q, kring, vring, L, C, C, out, lse,
                              static_cast<uint8_t*>(workspace), plan, B, cfg, dev, stream);
}

size_t g4attn_decode_rotated_workspace_size(int B, int L, int C, const g4attn_layer_cfg* cfg) {
    if (check_cfg(cfg, true) || B < 0 || L < 0 || C < 0) return 0;
    if (C > 0 && check_ring(C, cfg)) return 0;
    DeviceInfo* dev = nullptr;
    int sms = 148;
    if (current_device(&dev) == G4ATTN_OK) sms = dev->sms;
    else cudaGetLastError();
    return decode_plan(B, L, cfg, sms, 0, C).total;
}

int g4attn_decode_rotated(const g4attn_bf16* q, const g4attn_bf16* krot,
                          const g4attn_bf16* vcache, int L, int C, g4attn_bf16* out, float* lse,
                          void* workspace, size_t ws_bytes, int B, const g4attn_layer_cfg* cfg,
                          g4attn_stream_t stream) {
    int rc = check_decode(q, krot, vcache, L, out, lse, B, cfg);
    if (rc) return rc;
    if (cfg->kv_is_k != 0) return G4ATTN_ERR_UNSUPPORTED;   // the values must be their own
    if (C < 0) return G4ATTN_ERR_INVALID_ARG;
    if (C > 0 && (rc = check_ring(C, cfg))) return rc;
    if (B == 0) return G4ATTN_OK;
    DeviceInfo* dev = nullptr;
    if ((rc = current_device(&dev))) return rc;
    const DecodePlan plan = decode_plan(B, L, cfg, dev->sms, 0, C);
    if (!workspace || ws_bytes < plan.total) return G4ATTN_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return G4ATTN_ERR_MISALIGNED;
    return launch_decode_plan(q, krot, vcache, L, C > 0 ? C : L, C, out, lse,
                              static_cast<uint8_t*>(workspace), plan, B, cfg, dev, stream,
                              nullptr, true);
}

int g4attn_quantize_int8(const g4attn_bf16* x, int8_t* codes, float* scales, long long rows,
                         int d, g4attn_stream_t stream) {
    if (rows < 0 || (d != 128 && d != 256 && d != 512)) return G4ATTN_ERR_INVALID_ARG;
    if (rows == 0) return G4ATTN_OK;
    if (!x || !codes || !scales) return G4ATTN_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 3u))
        return G4ATTN_ERR_MISALIGNED;
    DeviceInfo* dev = nullptr;
    int rc;
    if ((rc = current_device(&dev))) return rc;
    return cuda_status(g4::launch_quantize_int8(x, codes, scales, rows, d,
                                                reinterpret_cast<cudaStream_t>(stream)));
}

// Decode with no workspace argument and no allocation: the split partials go to the
// library's fixed device scratch.  The number of CTA pairs (and with it the segments per
// sequence) is lowered until the partials fit; a problem whose single-segment partials
// (2 * B * Hq * (d + 2) fp32: one set per CTA of the pair) exceed the scratch is refused.
int g4attn_decode_noalloc(const g4attn_bf16* q, const g4attn_bf16* kcache,
                          const g4attn_bf16* vcache, int L, g4attn_bf16* out, float* lse, int B,
                          const g4attn_layer_cfg* cfg, g4attn_stream_t stream) {
    int rc = check_decode(q, kcache, vcache, L, out, lse, B, cfg);
    if (rc) return rc;
    if (B == 0) return G4ATTN_OK;
    DeviceInfo* dev = nullptr;
    if ((rc = current_device(&dev))) return rc;
    const size_t cap = g4::decode_scratch_bytes();
    const size_t per_split = 2 * (size_t)B * cfg->n_q_heads;   // two partials per segment
    if (align256(per_split * cfg->head_dim * sizeof(float)) + align256(per_split * 2 * sizeof(float)) >
        cap)
        return G4ATTN_ERR_TOO_LARGE;
    // the most CTA pairs whose partials fit: every pair count from the full split down is
    // tried (a count that divides the sequences evenly can fit where its neighbours cut
    // sequences in two), so the decode keeps as many SMs as the scratch allows
    DecodePlan plan = decode_plan(B, L, cfg, dev->sms);
    for (int p = plan.n_pairs - 1; plan.total > cap && p >= 1; --p)
        plan = decode_plan(B, L, cfg, dev->sms, p);
    if (plan.total > cap) return G4ATTN_ERR_TOO_LARGE;
    if (!dev->scratch) return G4ATTN_ERR_CUDA;
    return launch_decode_plan(q, kcache, vcache, L, L, 0, out, lse,
                              static_cast<uint8_t*>(dev->scratch), plan, B, cfg, dev, stream);
}

}  // extern "C"

// qknorm_rope.cu -- standalone QKNorm + p-RoPE prologue (memory-bound).
//
// One CTA per token (b, t).  The CTA first evaluates the R rotary (cos, sin) pairs of the
// token's position once (they are shared by every head), then each warp normalises whole
// head rows: RMS over head_dim in fp32 with the learned gain (Gemma 4 report section 2,
// QKNorm), then turns the pairs (i, i + d/2), i < R (p-RoPE).  Lane l owns elements
// [l*E, l*E + E) of both halves of the row, so a pair never leaves its lane.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kernels.h"
#include "rope.cuh"

namespace g4 {
namespace {

constexpr int kThreads = 256;

template <int E>
struct Vec;
template <>
struct Vec<8> { using T = uint4; };
template <>
struct Vec<4> { using T = uint2; };
template <>
struct Vec<2> { using T = uint32_t; };

template <int E>
__device__ __forceinline__ void load_bf16(const uint16_t* p, float* v) {
    typename Vec<E>::T raw = *reinterpret_cast<const typename Vec<E>::T*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < E / 2; ++i) {
        float2 f = __bfloat1622float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

template <int E>
__device__ __forceinline__ void store_bf16(uint16_t* p, const float* v) {
    typename Vec<E>::T raw;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < E / 2; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    *reinterpret_cast<typename Vec<E>::T*>(p) = raw;
}

template <int E>
__device__ __forceinline__ void store_f16(uint16_t* p, const float* v) {
    typename Vec<E>::T raw;
    __half2* h = reinterpret_cast<__half2*>(&raw);
#pragma unroll
    for (int i = 0; i < E / 2; ++i) h[i] = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
    *reinterpret_cast<typename Vec<E>::T*>(p) = raw;
}

template <int E>
__device__ __forceinline__ void store_row_half(uint16_t* p, const float* v, bool f16) {
    if (f16) store_f16<E>(p, v);
    else store_bf16<E>(p, v);
}

template <int E>
__global__ void __launch_bounds__(kThreads) qknorm_rope_kernel(QkNormRopeArgs a) {
    extern __shared__ float2 cs[];   // [R] (cos, sin) of this token's position
    const int d = 64 * E;
    const int half = d / 2;
    const int b = (int)(blockIdx.x / a.T);
    const int t = (int)(blockIdx.x % a.T);
    const long long pos = a.pos0 + t;
    // rows of this token in the inputs, the outputs and the cache copies
    const long long in_row = (long long)b * a.in_rows + (a.in_ring ? pos % a.in_ring : pos - a.in_base);
    const long long out_row = (long long)b * a.out_rows + (pos - a.out_base);
    const bool kc_live = !a.kc_ring || t >= a.T - a.kc_ring;   // not overwritten by a later token
    const long long kc_row = (long long)b * a.kc_rows + (a.kc_ring ? pos % a.kc_ring : pos);
    for (int i = threadIdx.x; i < a.rope.R; i += kThreads) {
        cs[i] = rope_cos_sin(pos, i, d, a.rope.log2_base);
        if (a.cs_out && b == 0) a.cs_out[(size_t)(pos - a.out_base) * a.rope.R + i] = cs[i];
    }
    __syncthreads();

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nq = a.q_in ? a.Hq : 0;
    const int nk = a.k_in ? a.Hkv : 0;
    const int nv = a.v_in ? a.Hkv : 0;
    for (int r = warp; r < nq + nk + nv; r += kThreads / 32) {
        if (r >= nq + nk) {   // values: a plain copy of the row
            const int h = r - nq - nk;
            const uint16_t* src = a.v_in + (in_row * a.Hkv + h) * (long long)d;
            uint16_t* dst = a.v_out ? a.v_out + (out_row * a.Hkv + h) * (long long)d : nullptr;
            uint16_t* cdst = a.vc_out && kc_live ? a.vc_out + (kc_row * a.Hkv + h) * (long long)d
                                                 : nullptr;
            for (int c = lane; c < d / 8; c += 32) {
                const uint4 x = reinterpret_cast<const uint4*>(src)[c];
                if (dst) reinterpret_cast<uint4*>(dst)[c] = x;
                if (cdst) reinterpret_cast<uint4*>(cdst)[c] = x;
            }
            continue;
        }
        const bool is_q = r < nq;
        const int h = is_q ? r : r - nq;
        const uint16_t* src = is_q ? a.q_in + (in_row * a.Hq + h) * (long long)d
                                   : a.k_in + (in_row * a.Hkv + h) * (long long)d;
        const float* gamma = is_q ? a.gamma_q : a.gamma_k;
        float x0[E], x1[E];
        load_bf16<E>(src + lane * E, x0);
        load_bf16<E>(src + half + lane * E, x1);
        if (a.qk_norm) {
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) ss += x0[e] * x0[e] + x1[e] * x1[e];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            const float inv = 1.0f / sqrtf(ss / (float)d + a.eps);
#pragma unroll
            for (int e = 0; e < E; ++e) {
                x0[e] = x0[e] * inv * gamma[lane * E + e];
                x1[e] = x1[e] * inv * gamma[half + lane * E + e];
            }
        }
        const bool f16 = !is_q && a.k_f16;
        if (!is_q && a.k_out) {
            uint16_t* dst = a.k_out + (out_row * a.Hkv + h) * (long long)d;
            store_row_half<E>(dst + lane * E, x0, f16);
            store_row_half<E>(dst + half + lane * E, x1, f16);
        }
        uint16_t* const kc_dst = !is_q && a.kc_out && kc_live
                                     ? a.kc_out + (kc_row * a.Hkv + h) * (long long)d
                                     : nullptr;
        if (kc_dst && !a.kc_rot) {
            store_bf16<E>(kc_dst + lane * E, x0);
            store_bf16<E>(kc_dst + half + lane * E, x1);
        }
        uint16_t* rdst = is_q ? (a.q_out ? a.q_out + (out_row * a.Hq + h) * (long long)d : nullptr)
                              : (a.krot_out ? a.krot_out + (out_row * a.Hkv + h) * (long long)d
                                            : nullptr);
        if (rdst || (kc_dst && a.kc_rot)) {
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const int i = lane * E + e;
                if (i < a.rope.R) {
                    const float2 c = cs[i];
                    const float u = x0[e], w = x1[e];
                    x0[e] = u * c.x - w * c.y;
                    x1[e] = u * c.y + w * c.x;
                }
            }
            if (rdst) {
                store_row_half<E>(rdst + lane * E, x0, f16);
                store_row_half<E>(rdst + half + lane * E, x1, f16);
            }
            if (kc_dst && a.kc_rot) {
                store_bf16<E>(kc_dst + lane * E, x0);
                store_bf16<E>(kc_dst + half + lane * E, x1);
            }
        }
    }
}

}  // namespace

cudaError_t launch_qknorm_rope(const QkNormRopeArgs& in, cudaStream_t stream) {
    const long long blocks = (long long)in.B * in.T;
    if (blocks == 0) return cudaSuccess;
    QkNormRopeArgs a = in;   // zero placement fields: the dense [B, T, H, d] layout
    if (a.in_rows == 0 && a.in_ring == 0) {
        a.in_rows = a.T;
        a.in_base = a.pos0;
    }
    if (a.out_rows == 0) {
        a.out_rows = a.T;
        a.out_base = a.pos0;
    }
    const size_t smem = sizeof(float2) * (size_t)(a.rope.R > 0 ? a.rope.R : 1);
    switch (a.d) {
        case 512: qknorm_rope_kernel<8><<<(unsigned)blocks, kThreads, smem, stream>>>(a); break;
        case 256: qknorm_rope_kernel<4><<<(unsigned)blocks, kThreads, smem, stream>>>(a); break;
        case 128: qknorm_rope_kernel<2><<<(unsigned)blocks, kThreads, smem, stream>>>(a); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace g4

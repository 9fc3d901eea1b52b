// quant.cu -- writer of the int8 KV cache: one fp32 scale per row (a position of one kv
// head), symmetric codes in [-127, 127].
//
// The Gemma 4 report's memory table counts the KV cache in int8 without giving the scheme;
// the one built here: scale = max |x| / 127, code = round-half-even(x / scale), clamped; a
// row of zeros keeps scale 0 and codes 0.  Both integer decisions use IEEE fp32 division
// rounded to nearest, so the codes are reproducible on any IEEE machine.  A row holding an
// infinity or a NaN has no such scale: it gets scale NaN and codes 0, so every element it
// stands for (scale * code) reads as NaN rather than as a wrong finite value.
//
// Memory-bound: one warp per row, each lane a contiguous run of d/32 elements (vector loads of
// 8-32 bytes, stores of 4-16 bytes), the row maximum by warp shuffles.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace g4 {
namespace {

constexpr int kQuantThreads = 256;   // 8 rows per block

template <int E>
struct QuantVec;
template <>
struct QuantVec<4> { using In = uint2; };
template <>
struct QuantVec<8> { using In = uint4; };
template <>
struct QuantVec<16> { using In = uint4; };   // two loads of 8 elements

// four codes into one little-endian word
__device__ __forceinline__ uint32_t pack4(const int* c) {
    return (uint32_t)(c[0] & 0xff) | ((uint32_t)(c[1] & 0xff) << 8) |
           ((uint32_t)(c[2] & 0xff) << 16) | ((uint32_t)(c[3] & 0xff) << 24);
}

template <int E>
__global__ void __launch_bounds__(kQuantThreads)
    quantize_int8_kernel(const uint16_t* __restrict__ x, int8_t* __restrict__ codes,
                         float* __restrict__ scales, long long rows) {
    constexpr int D = 32 * E;
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * (kQuantThreads / 32) + (threadIdx.x >> 5);
    if (row >= rows) return;
    const uint16_t* src = x + row * D + lane * E;
    float v[E];
    if constexpr (E == 16) {
        const uint4 a = reinterpret_cast<const uint4*>(src)[0];
        const uint4 b = reinterpret_cast<const uint4*>(src)[1];
        const __nv_bfloat162* ha = reinterpret_cast<const __nv_bfloat162*>(&a);
        const __nv_bfloat162* hb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 fa = __bfloat1622float2(ha[i]), fb = __bfloat1622float2(hb[i]);
            v[2 * i] = fa.x;
            v[2 * i + 1] = fa.y;
            v[8 + 2 * i] = fb.x;
            v[8 + 2 * i + 1] = fb.y;
        }
    } else {
        const typename QuantVec<E>::In a = *reinterpret_cast<const typename QuantVec<E>::In*>(src);
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&a);
#pragma unroll
        for (int i = 0; i < E / 2; ++i) {
            const float2 f = __bfloat1622float2(h[i]);
            v[2 * i] = f.x;
            v[2 * i + 1] = f.y;
        }
    }
    float amax = 0.f;
    bool finite = true;
#pragma unroll
    for (int i = 0; i < E; ++i) {
        amax = fmaxf(amax, fabsf(v[i]));
        finite &= isfinite(v[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    finite = __all_sync(0xffffffffu, finite);
    const float s = finite ? __fdiv_rn(amax, 127.0f) : __int_as_float(0x7fc00000);   // NaN
    int c[E];
#pragma unroll
    for (int i = 0; i < E; ++i) {
        float r = s > 0.f ? rintf(__fdiv_rn(v[i], s)) : 0.f;   // NaN scale: codes 0
        r = fminf(fmaxf(r, -127.f), 127.f);
        c[i] = (int)r;
    }
    int8_t* dst = codes + row * D + lane * E;
    if constexpr (E == 4) {
        *reinterpret_cast<uint32_t*>(dst) = pack4(c);
    } else if constexpr (E == 8) {
        *reinterpret_cast<uint2*>(dst) = make_uint2(pack4(c), pack4(c + 4));
    } else {
        *reinterpret_cast<uint4*>(dst) = make_uint4(pack4(c), pack4(c + 4), pack4(c + 8), pack4(c + 12));
    }
    if (lane == 0) scales[row] = s;
}

}  // namespace

cudaError_t launch_quantize_int8(const uint16_t* x, int8_t* codes, float* scales, long long rows,
                                 int d, cudaStream_t stream) {
    if (rows == 0) return cudaSuccess;
    const long long blocks = (rows + kQuantThreads / 32 - 1) / (kQuantThreads / 32);
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    switch (d) {
        case 128: quantize_int8_kernel<4><<<(unsigned)blocks, kQuantThreads, 0, stream>>>(x, codes, scales, rows); break;
        case 256: quantize_int8_kernel<8><<<(unsigned)blocks, kQuantThreads, 0, stream>>>(x, codes, scales, rows); break;
        case 512: quantize_int8_kernel<16><<<(unsigned)blocks, kQuantThreads, 0, stream>>>(x, codes, scales, rows); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace g4

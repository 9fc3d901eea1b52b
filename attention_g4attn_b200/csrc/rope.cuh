// rope.cuh -- RoPE angle evaluation shared by the kernels.
#pragma once

#include <cuda_runtime.h>

namespace g4 {

// (cos, sin) of phi = pos * base^(-2i/d), rotary pair i of a d-dim head
// (Gemma 4 report section 2: RoPE base 1e6 on global and 1e4 on local layers;
// explainer "p-RoPE": the first pair turns fastest).  The angle is formed and reduced
// modulo 2*pi in double precision, so positions up to 2^17 and beyond keep ~1e-7 rad of
// accuracy; the reduced angle (|r| <= pi) then goes through the fp32 sincosf.
__device__ __forceinline__ float2 rope_cos_sin(long long pos, int i, int d, double log2_base) {
    const double kTwoPi = 6.283185307179586;
    const double kInvTwoPi = 0.15915494309189535;
    double theta = exp2(-(2.0 * (double)i / (double)d) * log2_base);
    double phi = (double)pos * theta;
    double turns = rint(phi * kInvTwoPi);
    double r = fma(-turns, kTwoPi, phi);
    float s, c;
    sincosf((float)r, &s, &c);
    return make_float2(c, s);
}

}  // namespace g4

// rope_math.cuh -- the RoPE arithmetic shared by the rope_apply pass and the
// prefill kernel's fused Q rotation, so that both produce the same bits
// ("Transformer Architecture Breakdown ...", section 3.1; "Coding interview
// (14)", section 3.5): theta_i = base^(-2i/d), angle t * theta_i formed and
// reduced in fp64, cos/sin stored fp32, each pair (a, b) rotated to
// (a cos - b sin, a sin + b cos) in fp32 with every product and sum rounded
// separately (no contraction into FMAs), then rounded to bf16.
#pragma once

#include <cuda_runtime.h>

namespace attn {

// (cos, sin) of position t for frequency index i (0 <= i < d/2).
__device__ __forceinline__ float2 rope_cos_sin(long long t, int i, int d, double base) {
  const double theta = pow(base, -2.0 * (double)i / (double)d);
  const double ang = (double)t * theta;
  double s, c;
  sincos(ang, &s, &c);
  return make_float2((float)c, (float)s);
}

__device__ __forceinline__ void rope_rotate(float a, float b, float2 cs, float& ra, float& rb) {
  ra = __fsub_rn(__fmul_rn(a, cs.x), __fmul_rn(b, cs.y));
  rb = __fadd_rn(__fmul_rn(a, cs.y), __fmul_rn(b, cs.x));
}

}  // namespace attn

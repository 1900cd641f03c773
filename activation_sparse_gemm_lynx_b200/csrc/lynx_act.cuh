// lynx_act.cuh -- activations the GEMM epilogues apply to a finished output
// value, in fp32, before its one bf16 rounding.
#pragma once

#include "lynx_internal.h"

namespace lynx {

// GELU, tanh form (Hendrycks & Gimpel, "Gaussian Error Linear Units"):
//   gelu(v) = v/2 (1 + tanh u),  u = sqrt(2/pi) (v + 0.044715 v^3),
// evaluated through the identity (1 + tanh u)/2 = 1/(1 + e^(-2u)):
//   e^(-2u) = 2^x,  x = v (1 + 0.044715 v^2) * (-2 sqrt(2/pi) log2 e),
// then v / (1 + 2^x), with the hardware base-2 exponential and reciprocal
// (ex2.approx, rcp.approx; a few fp32 ulps).  Eight instructions per value:
// the epilogue runs next to a GEMM that is close to the board's power limit,
// and every instruction it adds there costs clock (a form with a sign select
// and a full divide ran the layer about 6% slower).  Both ends are exact in
// the limit: 2^x -> 0 gives v, 2^x -> inf gives 0; very negative v (|gelu(v)|
// below the fp32 normal range) gives zero.
__device__ __forceinline__ float gelu_tanh(float v) {
  const float x = v * __fmaf_rn(v * v, 0.044715f, 1.0f) * -2.3022081981f;
  float e, r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(x));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.0f + e));
  return v * r;
}

template <int ACT>
__device__ __forceinline__ float apply_act(float v) {
  if constexpr (ACT == kActGeluTanh) {
    return gelu_tanh(v);
  } else {
    return v;
  }
}

}  // namespace lynx

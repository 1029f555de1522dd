// Element-pair arithmetic and the gate activations of librn's row kernels
// (RL-Kernel PR #468, "[WS1][CUDA][Qwen3-Next] Gated RMSNorm CUDA kernel for
// the GDN block", Summary, "Activation" bullet).  Shared by the row kernels and
// the library's test entry points, so a test sees the very code the kernels run.
#pragma once

#include "rn_common.cuh"

namespace rn_detail {

// ---------------------------------------------------------------------------
// arithmetic of element pairs, written with explicit roundings
// ---------------------------------------------------------------------------
// Packed fp32 pairs (sm_100's two-lane fp32 instructions): each lane is the
// IEEE fp32 operation rounded to nearest even, so a pair op gives the bits of
// the two scalar ops it replaces and halves the instructions issued.  Adds
// stay scalar __fadd_rn: a product followed by a packed add was observed to
// come out fused (one rounding instead of two), which changed dw's bits, while
// __fadd_rn is never merged into a multiply-add.
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  return make_float2(__fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y));
}
__device__ __forceinline__ float2 bc2(float a) { return make_float2(a, a); }
__device__ __forceinline__ float2 neg2(float2 a) { return make_float2(-a.x, -a.y); }

// s(z) = 1 / (1 + exp(-z)) of both lanes   (PR #468 Summary, "Activation" bullet)
// Evaluated as 1/(1+e) for z >= 0 and e/(1+e) for z < 0 with e = exp(-|z|) in
// (0, 1]: the same function, but exp never overflows, so for z < -88.7 the
// sigmoid is the fp32 subnormal e^z rather than 1/inf = 0 (outlier gates reach
// there, and x*rstd*w*z*s(z) can still be a normal bf16 number).  1/(1+e) is
// rcp.approx refined by kRcpSteps Newton steps (rcp_1to2's operations).  e is
// CUDA's accurate expf, not the fast-math exponential: the operator's strict
// mode turns fast math off, and PR #468 ("Activation" bullet) uses expf.
__device__ __forceinline__ float2 sigmoid2(float2 z) {
  const float2 e = make_float2(expf(-fabsf(z.x)), expf(-fabsf(z.y)));
  const float2 d = add2(bc2(1.0f), e);
  float2 y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y.x) : "f"(d.x));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y.y) : "f"(d.y));
#pragma unroll
  for (int i = 0; i < kRcpSteps; ++i) y = fma2(y, fma2(neg2(d), y, bc2(1.0f)), y);
  const float2 er = mul2(e, y);
  return make_float2(z.x >= 0.0f ? y.x : er.x, z.y >= 0.0f ? y.y : er.y);
}

// a(z) from z and s = s(z): silu(z) = z * s(z), or the sigmoid itself
template <int ACT>
__device__ __forceinline__ float2 gate2(float2 z, float2 s) {
  return ACT == kActSilu ? mul2(z, s) : s;
}
// a'(z) / s(z): 1 + z * (1 - s) for silu, 1 - s for the sigmoid (1 + (-s)
// is the IEEE difference 1 - s exactly)
template <int ACT>
__device__ __forceinline__ float2 gate_slope_over_s2(float2 z, float2 s) {
  const float2 one_minus_s = add2(bc2(1.0f), neg2(s));
  return ACT == kActSilu ? fma2(z, one_minus_s, bc2(1.0f)) : one_minus_s;
}

}  // namespace rn_detail

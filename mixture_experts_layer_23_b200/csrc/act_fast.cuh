// Activation functions for the bf16 tensor-core epilogues, where outputs are rounded to bf16
// (8-bit mantissa): short instruction sequences with errors far below bf16 resolution.
//
// erf uses the rational approximation of Abramowitz & Stegun, Handbook of Mathematical
// Functions, formula 7.1.26 (|error| <= 1.5e-7 for x >= 0; odd extension for x < 0), with the
// exponential and the reciprocal as single approximate hardware operations (each element costs
// two special-function-unit operations and a handful of FMAs).  The fp32 layers keep the library
// math functions (see common.cuh).
#pragma once

#ifndef MOE_ACT_HOST_TEST
#include <cuda_runtime.h>
#define MOE_ACT_FN __device__ __forceinline__
#define MOE_EXP(x) __expf(x)
#define MOE_RCP(x) moe::fast::rcp_approx(x)
namespace moe {
namespace fast {
// single-instruction approximate reciprocal (rcp.approx: relative error within 1 ulp-ish of fp32,
// far below bf16 resolution)
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
}  // namespace fast
}  // namespace moe
#else
#include <math.h>
#define MOE_ACT_FN inline
#define MOE_EXP(x) expf(x)
#define MOE_RCP(x) (1.0f / (x))
#endif

namespace moe {
namespace fast {

// erf(|x|) and exp(-x^2) of x = |u| / sqrt(2), the two pieces GELU and its derivative share.
struct ErfParts {
  float erf_abs;  // erf(|u| / sqrt 2)
  float e;        // exp(-u^2 / 2)
};

MOE_ACT_FN ErfParts erf_parts(float u) {
  const float x = fabsf(u) * 0.70710678118654752f;
  const float t = MOE_RCP(fmaf(0.3275911f, x, 1.0f));
  float p = fmaf(t, 1.061405429f, -1.453152027f);
  p = fmaf(t, p, 1.421413741f);
  p = fmaf(t, p, -0.284496736f);
  p = fmaf(t, p, 0.254829592f);
  p *= t;
  const float e = MOE_EXP(-x * x);
  return ErfParts{fmaf(-p, e, 1.0f), e};
}

// u * Phi(u) = 0.5 u (1 + erf(u / sqrt 2))
MOE_ACT_FN float gelu(float u) {
  const ErfParts q = erf_parts(u);
  const float erf_u = copysignf(q.erf_abs, u);
  return 0.5f * u * (1.0f + erf_u);
}

// d/du [u Phi(u)] = Phi(u) + u phi(u),  phi(u) = exp(-u^2/2) / sqrt(2 pi)
MOE_ACT_FN float gelu_grad(float u) {
  const ErfParts q = erf_parts(u);
  const float erf_u = copysignf(q.erf_abs, u);
  return fmaf(0.5f, erf_u, 0.5f) + u * (0.39894228040143268f * q.e);
}

MOE_ACT_FN float sigmoid(float z) { return MOE_RCP(1.0f + MOE_EXP(-z)); }

}  // namespace fast
}  // namespace moe

// common.cuh -- device helpers shared by the sm_100a kernels of this library.
//
// Gate activation (CKDA review, "Method steps", step 1):
//   KDA   alpha = sigma(a),        beta = sigma(b)
//   CKDA  alpha = 2 sigma(a) - 1,  beta = 2 sigma(b)
//   raw   alpha = a,               beta = b
// Accurate libdevice functions (expf, expm1f, log1pf, logf, tanhf) are used:
// this file is compiled without fast-math.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ckda.h"

namespace ckda {

constexpr float kLn2 = 0.693147180559945309f;
constexpr float kInvLn2 = 1.442695040888963407f;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Gate forms: signed_gate 0 (KDA) widens no range and 1 (CKDA) both; 3 widens the gate range
// alone and 4 the strength range alone (the single-range variants of the CKDA review's
// Figure 6); 2 passes raw values.  The gate is sigma / 2 sigma - 1 / raw for alpha_form
// 0 / 1 / 2, the strength sigma / 2 sigma / raw for beta_form 0 / 1 / 2.
__host__ __device__ __forceinline__ constexpr int alpha_form(int signed_gate) {
  return signed_gate == 3 ? 1 : (signed_gate == 4 ? 0 : signed_gate);
}
__host__ __device__ __forceinline__ constexpr int beta_form(int signed_gate) {
  return signed_gate == 3 ? 0 : (signed_gate == 4 ? 1 : signed_gate);
}

// Linear gate value alpha (decode path).  Exact at +-inf: sigma 1/0, 2 sigma - 1 +-1.
__device__ __forceinline__ float gate_alpha(float a, int signed_gate) {
  const int f = alpha_form(signed_gate);
  if (f == 0) return 1.0f / (1.0f + expf(-a));
  if (f == 1) return tanhf(0.5f * a);  // 2 sigma(a) - 1 == tanh(a/2)
  return a;
}

// Strength beta.  Exact at +-inf: sigma 1/0, 2 sigma 2/0.
__device__ __forceinline__ float gate_beta(float b, int signed_gate) {
  const int f = beta_form(signed_gate);
  if (f == 0) return 1.0f / (1.0f + expf(-b));
  if (f == 1) return 2.0f / (1.0f + expf(-b));
  return b;
}

// Log-space gate: log2|alpha| (finite unless is_zero), sign bit, exact-zero flag.
//   KDA : log sigma(a) = -softplus(-a);       zero iff a == -inf
//   CKDA: log |tanh(a/2)| = log(-expm1(-|a|)) - log1p(exp(-|a|));  zero iff a == 0
//   raw : log |a|;                            zero iff a == 0
__device__ __forceinline__ void gate_log2(float a, int signed_gate, float &log2abs, bool &is_zero,
                                          bool &is_neg) {
  const int f = alpha_form(signed_gate);
  if (f == 0) {
    is_neg = false;
    is_zero = (a == -INFINITY);
    const float x = -a;  // softplus(x) = max(x, 0) + log1p(exp(-|x|))
    const float sp = fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x)));
    log2abs = is_zero ? 0.0f : -sp * kInvLn2;
  } else if (f == 1) {
    is_neg = (a < 0.0f);
    is_zero = (a == 0.0f);
    const float x = fabsf(a);
    log2abs = is_zero ? 0.0f : (logf(-expm1f(-x)) - log1pf(expf(-x))) * kInvLn2;
  } else {
    is_neg = (a < 0.0f);
    is_zero = (a == 0.0f);
    log2abs = is_zero ? 0.0f : log2f(fabsf(a));
  }
}

// Derivatives of the activations with respect to their logits (backward):
// d sigma(x) / dx = sigma(x) sigma(-x) = e^{-|x|} / (1 + e^{-|x|})^2 (0 at +-inf), doubled for
// 2 sigma - 1 and 2 sigma, 1 for raw values.
__device__ __forceinline__ float dsigmoid(float x) {
  const float e = expf(-fabsf(x));
  const float d = 1.0f + e;
  return e / (d * d);
}
__device__ __forceinline__ float dalpha_da(float a, int signed_gate) {
  const int f = alpha_form(signed_gate);
  return f == 2 ? 1.0f : (f == 1 ? 2.0f : 1.0f) * dsigmoid(a);
}
__device__ __forceinline__ float dbeta_db(float b, int signed_gate) {
  const int f = beta_form(signed_gate);
  return f == 2 ? 1.0f : (f == 1 ? 2.0f : 1.0f) * dsigmoid(b);
}

// Records the first device-detected error in the workspace status word.
__device__ __forceinline__ void set_status(int *status, int code) {
  if (status) atomicCAS(status, 0, code);
}

}  // namespace ckda

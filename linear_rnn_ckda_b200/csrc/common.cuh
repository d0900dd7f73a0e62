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

// Gate forms (signed_gate & kGateFormMask): 0 (KDA) widens no range and 1 (CKDA) both; 3 widens
// the gate range alone and 4 the strength range alone (the single-range variants of the CKDA
// review's Figure 6); 2 passes raw values.  The gate is sigma / 2 sigma - 1 / raw for alpha_form
// 0 / 1 / 2, the strength sigma / 2 sigma / raw for beta_form 0 / 1 / 2.  Two flag bits ride
// above the form: kFlagPerHeadGate (one gate per token and head, GDN-style: a is [B,T,H] and
// the gate is broadcast over the key channels) and kFlagQkL2Norm (q and k are divided by
// their L2 norm over the key channels inside the kernel).
constexpr int kGateFormMask = 15;
constexpr int kFlagPerHeadGate = CKDA_GATE_PER_HEAD;
constexpr int kFlagQkL2Norm = CKDA_QK_L2NORM;
constexpr int kFlagProduct2 = CKDA_DELTA_PRODUCT2;
__host__ __device__ __forceinline__ constexpr int alpha_form(int signed_gate) {
  return (signed_gate & kGateFormMask) == 3 ? 1
         : (signed_gate & kGateFormMask) == 4 ? 0 : (signed_gate & kGateFormMask);
}
__host__ __device__ __forceinline__ constexpr int beta_form(int signed_gate) {
  return (signed_gate & kGateFormMask) == 3 ? 0
         : (signed_gate & kGateFormMask) == 4 ? 1 : (signed_gate & kGateFormMask);
}
__host__ __device__ __forceinline__ constexpr bool per_head_gate(int signed_gate) {
  return (signed_gate & kFlagPerHeadGate) != 0;
}
__host__ __device__ __forceinline__ constexpr bool qk_l2norm(int signed_gate) {
  return (signed_gate & kFlagQkL2Norm) != 0;
}
__host__ __device__ __forceinline__ constexpr bool delta_product2(int signed_gate) {
  return (signed_gate & kFlagProduct2) != 0;
}
// 1 / ||x|| from the sum of squares, 0 for a zero vector (which then stays zero)
__device__ __forceinline__ float inv_norm(float sumsq) { return sumsq > 0.f ? rsqrtf(sumsq) : 0.f; }

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

// Divides rows 0..rows-1 of the fp32 tiles X and Y (row stride ld, n columns) by their L2
// norms (a zero row stays zero); the factors go to inv_x / inv_y when given.  One warp per
// row, the whole block takes part; the caller synchronises before and after.
__device__ __forceinline__ void l2norm_rows2(float *X, float *Y, int ld, int rows, int n,
                                             float *inv_x, float *inv_y) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  for (int r = warp; r < rows; r += nw) {
    float sx = 0.f, sy = 0.f;
    for (int c = lane; c < n; c += 32) {
      const float x = X[r * ld + c], y = Y[r * ld + c];
      sx = fmaf(x, x, sx);
      sy = fmaf(y, y, sy);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      sx += __shfl_xor_sync(0xffffffffu, sx, off);
      sy += __shfl_xor_sync(0xffffffffu, sy, off);
    }
    const float ix = inv_norm(sx), iy = inv_norm(sy);
    for (int c = lane; c < n; c += 32) {
      X[r * ld + c] *= ix;
      Y[r * ld + c] *= iy;
    }
    if (lane == 0 && inv_x) {
      inv_x[r] = ix;
      inv_y[r] = iy;
    }
  }
}

// Records the first device-detected error in the workspace status word.
__device__ __forceinline__ void set_status(int *status, int code) {
  if (status) atomicCAS(status, 0, code);
}

}  // namespace ckda

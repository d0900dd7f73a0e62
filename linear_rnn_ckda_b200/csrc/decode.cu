// decode.cu -- one recurrent decode step on sm_100a (HBM-bound).
//
// Per head:  S' = Diag(alpha) S;  p = S'^T k;  S = S' + beta k (v - p)^T;  o = S^T q
// which is S_t = (I - beta k k^T) Diag(alpha) S_{t-1} + beta k v^T, o_t = S_t^T q_t
// (CKDA review, section "Diagonal-plus-rank-one (DPR1) transition"; the
// review notes the extended ranges add no per-token inference cost).
//
// Each head's fp32 state [dk][dv] is read once and written once, in 16-byte
// vectors.  A warp owns 16 state columns: lane l holds columns
// 16*w + 4*(l%4) .. +3 for rows l/4 + 8*m (m = 0 .. dk/8-1), so one warp load
// instruction covers 8 rows x 64 contiguous bytes, and the reductions over the
// key channel (k . S' and q . S) are in-thread sums followed by three xor
// shuffles across the 8 lanes that share a column group.  No shared-memory
// reduction and no block barrier touch the state.
#include "common.cuh"
#include "internal.h"

namespace ckda {
namespace {

constexpr int kDecodeThreads = 256;

template <int DK, int DV, typename TIn, typename TOut>
__global__ void __launch_bounds__(kDecodeThreads)
    decode_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k, const TIn *__restrict__ v,
                  const TIn *__restrict__ a, const float *__restrict__ b, float *__restrict__ S,
                  TOut *__restrict__ o, int n_heads, int H, int signed_gate) {
  constexpr int kWarpsPerHead = DV / 16;
  constexpr int kHeadsPerBlock = (kDecodeThreads / 32) / kWarpsPerHead;
  constexpr int kRows = DK / 8;  // state rows per thread
  __shared__ float s_q[kHeadsPerBlock][DK];
  __shared__ float s_k[kHeadsPerBlock][DK];
  __shared__ float s_al[kHeadsPerBlock][DK];
  __shared__ float s_k2[kHeadsPerBlock][DK];     // DeltaProduct2: the token's second key
  __shared__ float s_beta[kHeadsPerBlock][2];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hl = warp / kWarpsPerHead;
  const int head = blockIdx.x * kHeadsPerBlock + hl;
  const int gtid = threadIdx.x - hl * kWarpsPerHead * 32;  // thread index within the head group
  const int cq = lane & 3, r0 = lane >> 2;
  const int col = (warp % kWarpsPerHead) * 16 + cq * 4;
  float *Sh = S + (size_t)head * DK * DV;

  // The state loads go first: they do not depend on the staging below and stay in flight
  // across it.
  float4 st[kRows];
  if (head < n_heads) {
#pragma unroll
    for (int m = 0; m < kRows; ++m)
      st[m] = *reinterpret_cast<const float4 *>(Sh + (size_t)(r0 + 8 * m) * DV + col);
  }

  // Stage q, k and the activated gate for this head group (one gate per head with
  // CKDA_GATE_PER_HEAD: a is [B, H]).
  // (DeltaProduct2: k, v, b hold two rows per token, [B, 2, H, .]; key j of this head is
  // row (head / H * 2 + j) * H + head % H)
  const bool per_head = per_head_gate(signed_gate), prod2 = delta_product2(signed_gate);
  const size_t krow1 = prod2 ? ((size_t)(head / H) * 2) * H + head % H : (size_t)head;
  const size_t krow2 = krow1 + H;
  if (head < n_heads) {
    for (int i = gtid; i < DK; i += kWarpsPerHead * 32) {
      const size_t e = (size_t)head * DK + i;
      s_q[hl][i] = to_f32(q[e]);
      s_k[hl][i] = to_f32(k[krow1 * DK + i]);
      if (prod2) s_k2[hl][i] = to_f32(k[krow2 * DK + i]);
      s_al[hl][i] = gate_alpha(to_f32(a[per_head ? (size_t)head : e]), signed_gate);
    }
    if (gtid == 0) {
      s_beta[hl][0] = gate_beta(b[krow1], signed_gate);
      if (prod2) s_beta[hl][1] = gate_beta(b[krow2], signed_gate);
    }
  }
  __syncthreads();
  if (qk_l2norm(signed_gate)) {
    // q and k divided by their norms over the key channels (the head group's first warp)
    if (head < n_heads && gtid < 32) {
      float sq = 0.f, sk = 0.f, sk2 = 0.f;
      for (int i = gtid; i < DK; i += 32) {
        sq = fmaf(s_q[hl][i], s_q[hl][i], sq);
        sk = fmaf(s_k[hl][i], s_k[hl][i], sk);
        if (prod2) sk2 = fmaf(s_k2[hl][i], s_k2[hl][i], sk2);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        sq += __shfl_xor_sync(0xffffffffu, sq, off);
        sk += __shfl_xor_sync(0xffffffffu, sk, off);
        sk2 += __shfl_xor_sync(0xffffffffu, sk2, off);
      }
      const float iq = inv_norm(sq), ik = inv_norm(sk), ik2 = inv_norm(sk2);
      for (int i = gtid; i < DK; i += 32) {
        s_q[hl][i] *= iq;
        s_k[hl][i] *= ik;
        if (prod2) s_k2[hl][i] *= ik2;
      }
    }
    __syncthreads();
  }
  if (head >= n_heads) return;

  // S' = Diag(alpha) S and p = S'^T k (partial over this thread's rows)
  float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
#pragma unroll
  for (int m = 0; m < kRows; ++m) {
    const int i = r0 + 8 * m;
    const float al = s_al[hl][i], ki = s_k[hl][i];
    st[m].x *= al; st[m].y *= al; st[m].z *= al; st[m].w *= al;
    p0 = fmaf(ki, st[m].x, p0); p1 = fmaf(ki, st[m].y, p1);
    p2 = fmaf(ki, st[m].z, p2); p3 = fmaf(ki, st[m].w, p3);
  }
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    p0 += __shfl_xor_sync(0xffffffffu, p0, off);
    p1 += __shfl_xor_sync(0xffffffffu, p1, off);
    p2 += __shfl_xor_sync(0xffffffffu, p2, off);
    p3 += __shfl_xor_sync(0xffffffffu, p3, off);
  }

  // u = beta (v - p)
  const float beta = s_beta[hl][0];
  const TIn *vh = v + krow1 * DV + col;
  float u0 = beta * (to_f32(vh[0]) - p0), u1 = beta * (to_f32(vh[1]) - p1);
  float u2 = beta * (to_f32(vh[2]) - p2), u3 = beta * (to_f32(vh[3]) - p3);
  if (prod2) {
    // DeltaProduct2: the first update, then the second key's read p' = S''^T k2 and its update
    float q0 = 0.f, q1 = 0.f, q2 = 0.f, q3 = 0.f;
#pragma unroll
    for (int m = 0; m < kRows; ++m) {
      const int i = r0 + 8 * m;
      const float ki = s_k[hl][i], k2i = s_k2[hl][i];
      st[m].x = fmaf(ki, u0, st[m].x); st[m].y = fmaf(ki, u1, st[m].y);
      st[m].z = fmaf(ki, u2, st[m].z); st[m].w = fmaf(ki, u3, st[m].w);
      q0 = fmaf(k2i, st[m].x, q0); q1 = fmaf(k2i, st[m].y, q1);
      q2 = fmaf(k2i, st[m].z, q2); q3 = fmaf(k2i, st[m].w, q3);
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      q0 += __shfl_xor_sync(0xffffffffu, q0, off);
      q1 += __shfl_xor_sync(0xffffffffu, q1, off);
      q2 += __shfl_xor_sync(0xffffffffu, q2, off);
      q3 += __shfl_xor_sync(0xffffffffu, q3, off);
    }
    const float beta2 = s_beta[hl][1];
    const TIn *vh2 = v + krow2 * DV + col;
    u0 = beta2 * (to_f32(vh2[0]) - q0); u1 = beta2 * (to_f32(vh2[1]) - q1);
    u2 = beta2 * (to_f32(vh2[2]) - q2); u3 = beta2 * (to_f32(vh2[3]) - q3);
  }
  const float(*kw)[DK] = prod2 ? s_k2 : s_k;   // the key of the last update

  // S = S' + k u^T, written back; o = S^T q
  float r0s = 0.f, r1s = 0.f, r2s = 0.f, r3s = 0.f;
#pragma unroll
  for (int m = 0; m < kRows; ++m) {
    const int i = r0 + 8 * m;
    const float ki = kw[hl][i], qi = s_q[hl][i];
    st[m].x = fmaf(ki, u0, st[m].x); st[m].y = fmaf(ki, u1, st[m].y);
    st[m].z = fmaf(ki, u2, st[m].z); st[m].w = fmaf(ki, u3, st[m].w);
    *reinterpret_cast<float4 *>(Sh + (size_t)i * DV + col) = st[m];
    r0s = fmaf(qi, st[m].x, r0s); r1s = fmaf(qi, st[m].y, r1s);
    r2s = fmaf(qi, st[m].z, r2s); r3s = fmaf(qi, st[m].w, r3s);
  }
  if (o == nullptr) return;
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    r0s += __shfl_xor_sync(0xffffffffu, r0s, off);
    r1s += __shfl_xor_sync(0xffffffffu, r1s, off);
    r2s += __shfl_xor_sync(0xffffffffu, r2s, off);
    r3s += __shfl_xor_sync(0xffffffffu, r3s, off);
  }
  if (r0 == 0) {
    TOut *oh = o + (size_t)head * DV + col;
    oh[0] = from_f32<TOut>(r0s); oh[1] = from_f32<TOut>(r1s);
    oh[2] = from_f32<TOut>(r2s); oh[3] = from_f32<TOut>(r3s);
  }
}

template <int DK, int DV, typename TIn, typename TOut>
int launch_typed(const DecodeArgs &g, cudaStream_t stream) {
  const int n_heads = g.B * g.H;
  constexpr int kHeadsPerBlock = (kDecodeThreads / 32) / (DV / 16);
  const int blocks = (n_heads + kHeadsPerBlock - 1) / kHeadsPerBlock;
  decode_kernel<DK, DV, TIn, TOut><<<blocks, kDecodeThreads, 0, stream>>>(
      static_cast<const TIn *>(g.q), static_cast<const TIn *>(g.k), static_cast<const TIn *>(g.v),
      static_cast<const TIn *>(g.a), g.b, g.S, static_cast<TOut *>(g.o), n_heads, g.H,
      g.signed_gate);
  return cudaGetLastError() == cudaSuccess ? CKDA_OK : CKDA_ERR_CUDA;
}

template <int DK, int DV>
int launch_dims(const DecodeArgs &g, cudaStream_t s) {
  const bool in_bf = g.io_dtype == CKDA_BF16, out_bf = g.o_dtype == CKDA_BF16;
  if (in_bf && out_bf) return launch_typed<DK, DV, __nv_bfloat16, __nv_bfloat16>(g, s);
  if (in_bf) return launch_typed<DK, DV, __nv_bfloat16, float>(g, s);
  if (out_bf) return launch_typed<DK, DV, float, __nv_bfloat16>(g, s);
  return launch_typed<DK, DV, float, float>(g, s);
}

template <int DK>
int launch_dv(const DecodeArgs &g, cudaStream_t s) {
  switch (g.dv) {
    case 16: return launch_dims<DK, 16>(g, s);
    case 32: return launch_dims<DK, 32>(g, s);
    case 64: return launch_dims<DK, 64>(g, s);
    case 128: return launch_dims<DK, 128>(g, s);
  }
  return CKDA_ERR_DIM;
}

}  // namespace

int launch_decode(const DecodeArgs &g, cudaStream_t s) {
  if (g.B * g.H == 0) return CKDA_OK;
  switch (g.dk) {
    case 16: return launch_dv<16>(g, s);
    case 32: return launch_dv<32>(g, s);
    case 64: return launch_dv<64>(g, s);
    case 128: return launch_dv<128>(g, s);
  }
  return CKDA_ERR_DIM;
}

}  // namespace ckda

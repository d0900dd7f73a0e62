// chunk_simt.cu -- exact fp32 chunkwise (WY / UT-transform) forward, CUDA cores.
//
// This is the library's fp32 path (any dk, dv in {16..128}, chunk in {16,32,64}):
// every product runs in fp32 FMA, the within-chunk gate products are formed in
// log space with a sign-parity bit and an exact-zero count, so alpha = 0,
// alpha = +-1 and arbitrarily strong decay are all exact.
//
// Chunkwise form (the CKDA review states the DPR1 transition keeps WY
// chunk-wise parallelism, section "Diagonal-plus-rank-one (DPR1) transition").
// For a chunk with incoming state S0 and positions r = 0..C-1, let
// g(r,j) = prod_{s=j+1..r} alpha_s per channel and G_r = g(r,-1).  Then
//   A[r,j] = beta_r sum_c k_rc k_jc g(r,j)_c    (j < r)
//   P[r,j] =        sum_c q_rc k_jc g(r,j)_c    (j <= r)
//   Tm     = (I + A)^{-1} Diag(beta)
//   U      = Tm (V - (K*G) S0)
//   O      = (Q*G) S0 + P U
//   S_C    = Diag(G_{C-1}) S0 + (K * g(C-1, .))^T U
// with g(r,j)_c = 0 when a zero gate lies in (j, r], else
// (-1)^(parity_r xor parity_j) 2^(L_r - L_j), L the prefix of log2|alpha|.
//
// One CTA owns one (sequence, head, dv-slice of <= 64 columns); chunks of a
// sequence run in order, the state slice stays in shared memory.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace ckda {
namespace {

constexpr int kSimtThreads = 256;

struct SimtParams {
  const void *q, *k, *v, *a;
  const float *b, *S0;
  const int32_t *cu;
  void *o;
  float *S_T;
  int *status;
  int n_seqs, T, H, dk, dv, C, dvs, signed_gate;
};

__host__ __device__ inline size_t simt_smem_floats(int dk, int dvs, int C) {
  const int ldk = dk + 1, ldz = dk + 4;
  return (size_t)dk * dvs + 3 * (size_t)C * ldk + ((size_t)C * ldz) / 4 + 2 * (size_t)C * dvs +
         2 * (size_t)C * C + C + 3 * (size_t)dk;
}

template <typename TIn, typename TOut>
__global__ void __launch_bounds__(kSimtThreads, 1) chunk_simt_kernel(SimtParams p) {
  extern __shared__ float smem[];
  const int dk = p.dk, dvs = p.dvs, C = p.C, H = p.H, dv = p.dv;
  const int ldk = dk + 1, ldz = dk + 4;
  const int tid = threadIdx.x;
  float *sS = smem;                       // [dk][dvs] state slice
  float *sQ = sS + (size_t)dk * dvs;      // [C][ldk]  q, then q*G
  float *sK = sQ + (size_t)C * ldk;       // [C][ldk]  k, then k*G
  float *sL = sK + (size_t)C * ldk;       // [C][ldk]  raw a, then L, then k*g(C-1,.)
  uint8_t *sZ = reinterpret_cast<uint8_t *>(sL + (size_t)C * ldk);  // [C][ldz] zero count<<1 | parity
  float *sV = reinterpret_cast<float *>(sZ + (size_t)C * ldz);      // [C][dvs] v, then V - (K*G) S
  float *sU = sV + (size_t)C * dvs;       // [C][dvs]
  float *sA = sU + (size_t)C * dvs;       // [C][C]    A, then Tm
  float *sP = sA + (size_t)C * C;         // [C][C]
  float *sBeta = sP + (size_t)C * C;      // [C]
  float *sG = sBeta + C;                  // [dk] G_{C-1}
  float *sLC = sG + dk;                   // [dk] L_{C-1}
  int *sZC = reinterpret_cast<int *>(sLC + dk);  // [dk] zero count and parity at C-1

  const TIn *q = static_cast<const TIn *>(p.q);
  const TIn *k = static_cast<const TIn *>(p.k);
  const TIn *v = static_cast<const TIn *>(p.v);
  const TIn *a = static_cast<const TIn *>(p.a);
  TOut *o = static_cast<TOut *>(p.o);

  const bool per_head = per_head_gate(p.signed_gate), l2 = qk_l2norm(p.signed_gate);
  // DeltaProduct2: the kernel walks two rows per token (k, v, b are [rows of tokens x 2]);
  // row 2t carries the gate of token t, row 2t + 1 a gate of 1 and the read-out
  const int rpt = delta_product2(p.signed_gate) ? 2 : 1;
  const float unit_logit = alpha_form(p.signed_gate) == 2 ? 1.f : INFINITY;
  const int unit = blockIdx.x;
  const int n = unit / H, h = unit % H;
  const int j0 = blockIdx.y * dvs;
  long t0, t1, bofs;
  if (p.cu) {
    t0 = p.cu[n];
    t1 = p.cu[n + 1];
    bofs = 0;
    if (t0 < 0 || t1 < t0 || t1 > p.T || (n == 0 && t0 != 0) || (n == p.n_seqs - 1 && t1 != p.T)) {
      if (tid == 0) set_status(p.status, CKDA_ERR_SEQLENS);
      return;
    }
  } else {
    t0 = 0;
    t1 = p.T;
    bofs = (long)n * p.T;
  }
  // from here on t0, t1, bofs count kernel rows (two per token for DeltaProduct2)
  t0 *= rpt;
  t1 *= rpt;
  bofs *= rpt;
  const size_t sbase = ((size_t)n * H + h) * dk * dv;

  for (int e = tid; e < dk * dvs; e += kSimtThreads) {
    const int c = e / dvs, j = e % dvs;
    sS[e] = p.S0 ? p.S0[sbase + (size_t)c * dv + j0 + j] : 0.f;
  }

  for (long cs = t0; cs < t1; cs += C) {
    const int nrows = (int)(t1 - cs < C ? t1 - cs : C);
    __syncthreads();
    // ---- load q, k, raw a (rows past the sequence end: q = k = 0, alpha = 1)
    for (int e = tid; e < C * dk; e += kSimtThreads) {
      const int r = e / dk, c = e % dk;
      float qv = 0.f, kv = 0.f, av = 0.f;
      if (r < nrows) {
        const long kr = bofs + cs + r;                    // kernel row
        const size_t row = (size_t)kr * H + h;            // its k, v, b row
        const size_t trow = (size_t)(kr / rpt) * H + h;   // its token's q, a, o row
        const bool first = kr % rpt == 0, last = kr % rpt == rpt - 1;
        qv = last ? to_f32(q[trow * dk + c]) : 0.f;
        kv = to_f32(k[row * dk + c]);
        av = first ? to_f32(a[per_head ? trow : trow * dk + c]) : unit_logit;
      }
      sQ[r * ldk + c] = qv;
      sK[r * ldk + c] = kv;
      sL[r * ldk + c] = av;
    }
    for (int e = tid; e < C * dvs; e += kSimtThreads) {
      const int r = e / dvs, j = e % dvs;
      sV[e] = r < nrows ? to_f32(v[((size_t)(bofs + cs + r) * H + h) * dv + j0 + j]) : 0.f;
    }
    for (int r = tid; r < C; r += kSimtThreads)
      sBeta[r] = r < nrows ? gate_beta(p.b[(size_t)(bofs + cs + r) * H + h], p.signed_gate) : 0.f;
    __syncthreads();
    if (l2) {   // q, k divided by their norms over the key channels
      l2norm_rows2(sQ, sK, ldk, nrows, dk, nullptr, nullptr);
      __syncthreads();
    }
    // ---- gate prefix per channel: L_r, zero count, parity (in place over raw a)
    for (int c = tid; c < dk; c += kSimtThreads) {
      float L = 0.f;
      int zc = 0, par = 0;
      for (int r = 0; r < C; ++r) {
        if (r < nrows) {
          float l;
          bool z, neg;
          gate_log2(sL[r * ldk + c], p.signed_gate, l, z, neg);
          if (z) {
            ++zc;
          } else {
            L += l;
            par ^= (int)neg;
          }
        }
        sL[r * ldk + c] = L;
        sZ[r * ldz + c] = (uint8_t)((zc << 1) | par);
      }
      sLC[c] = L;
      sZC[c] = (zc << 1) | par;
      sG[c] = zc ? 0.f : (par ? -exp2f(L) : exp2f(L));
    }
    __syncthreads();
    // ---- A (strictly lower) and P (lower incl. diagonal), exact pair factors
    const int npairs = C * (C + 1) / 2;
    for (int e = tid; e < npairs; e += kSimtThreads) {
      int r = (int)((sqrtf(8.f * e + 1.f) - 1.f) * 0.5f);
      while (r * (r + 1) / 2 > e) --r;
      while ((r + 1) * (r + 2) / 2 <= e) ++r;
      const int j = e - r * (r + 1) / 2;
      float accA = 0.f, accP = 0.f;
      for (int c = 0; c < dk; ++c) {
        const int zr = sZ[r * ldz + c], zj = sZ[j * ldz + c];
        if ((zr >> 1) != (zj >> 1)) continue;
        float f = exp2f(sL[r * ldk + c] - sL[j * ldk + c]);
        if ((zr ^ zj) & 1) f = -f;
        const float kj = sK[j * ldk + c] * f;
        accA = fmaf(sK[r * ldk + c], kj, accA);
        accP = fmaf(sQ[r * ldk + c], kj, accP);
      }
      sA[r * C + j] = (j < r) ? sBeta[r] * accA : 0.f;
      sP[r * C + j] = accP;
      if (j < r) {  // zero the mirrored upper entries
        sA[j * C + r] = 0.f;
        sP[j * C + r] = 0.f;
      }
    }
    __syncthreads();
    // ---- q*G, k*G, k*g(C-1, .)
    for (int e = tid; e < C * dk; e += kSimtThreads) {
      const int r = e / dk, c = e % dk;
      const int z = sZ[r * ldz + c];
      const float L = sL[r * ldk + c];
      const float g = (z >> 1) ? 0.f : ((z & 1) ? -exp2f(L) : exp2f(L));
      const int zC = sZC[c];
      float gb = 0.f;
      if ((z >> 1) == (zC >> 1)) {
        gb = exp2f(sLC[c] - L);
        if ((z ^ zC) & 1) gb = -gb;
      }
      const float kv = sK[r * ldk + c];
      sQ[r * ldk + c] *= g;
      sK[r * ldk + c] = kv * g;
      sL[r * ldk + c] = kv * gb;
    }
    // ---- Tm = (I + A)^{-1} Diag(beta): forward substitution, row by row
    for (int r = 1; r < C; ++r) {
      __syncthreads();
      float x = 0.f;
      const int m = tid;
      if (m < r) {
        x = -sA[r * C + m];
        for (int j = m + 1; j < r; ++j) x = fmaf(-sA[r * C + j], sA[j * C + m], x);
      }
      __syncthreads();
      if (m < r) sA[r * C + m] = x;
    }
    __syncthreads();
    for (int e = tid; e < C * C; e += kSimtThreads) {
      const int r = e / C, m = e % C;
      sA[e] = (m < r) ? sA[e] * sBeta[m] : (m == r ? sBeta[r] : 0.f);
    }
    __syncthreads();
    // ---- Y = V - (K*G) S  (in place over V)
    for (int e = tid; e < C * dvs; e += kSimtThreads) {
      const int r = e / dvs, j = e % dvs;
      float acc = sV[e];
      for (int c = 0; c < dk; ++c) acc = fmaf(-sK[r * ldk + c], sS[c * dvs + j], acc);
      sV[e] = acc;
    }
    __syncthreads();
    // ---- U = Tm Y
    for (int e = tid; e < C * dvs; e += kSimtThreads) {
      const int r = e / dvs, j = e % dvs;
      float acc = 0.f;
      for (int m = 0; m <= r; ++m) acc = fmaf(sA[r * C + m], sV[m * dvs + j], acc);
      sU[e] = acc;
    }
    __syncthreads();
    // ---- O = (Q*G) S + P U
    if (o) {
      for (int e = tid; e < nrows * dvs; e += kSimtThreads) {
        const int r = e / dvs, j = e % dvs;
        const long kr = bofs + cs + r;
        if (kr % rpt != rpt - 1) continue;   // DeltaProduct2: read out after a token's last update
        float acc = 0.f;
        for (int c = 0; c < dk; ++c) acc = fmaf(sQ[r * ldk + c], sS[c * dvs + j], acc);
        for (int m = 0; m <= r; ++m) acc = fmaf(sP[r * C + m], sU[m * dvs + j], acc);
        o[((size_t)(kr / rpt) * H + h) * dv + j0 + j] = from_f32<TOut>(acc);
      }
    }
    __syncthreads();
    // ---- S = Diag(G_{C-1}) S + (K * g(C-1,.))^T U
    for (int e = tid; e < dk * dvs; e += kSimtThreads) {
      const int c = e / dvs, j = e % dvs;
      float acc = sG[c] * sS[e];
      for (int r = 0; r < C; ++r) acc = fmaf(sL[r * ldk + c], sU[r * dvs + j], acc);
      sS[e] = acc;
    }
  }
  __syncthreads();
  if (p.S_T) {
    for (int e = tid; e < dk * dvs; e += kSimtThreads) {
      const int c = e / dvs, j = e % dvs;
      p.S_T[sbase + (size_t)c * dv + j0 + j] = sS[e];
    }
  }
}

template <typename TIn, typename TOut>
int launch_typed(const ChunkArgs &g, cudaStream_t stream) {
  SimtParams p;
  p.q = g.q; p.k = g.k; p.v = g.v; p.a = g.a; p.b = g.b; p.S0 = g.S0; p.cu = g.cu_seqlens;
  p.o = g.o; p.S_T = g.S_T; p.status = g.status;
  p.n_seqs = g.n_seqs; p.T = g.T; p.H = g.H; p.dk = g.dk; p.dv = g.dv; p.C = g.chunk;
  p.dvs = std::min(g.dv, 64);
  p.signed_gate = g.signed_gate;
  const size_t smem = simt_smem_floats(p.dk, p.dvs, p.C) * sizeof(float);
  auto kern = chunk_simt_kernel<TIn, TOut>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return CKDA_ERR_CUDA;
  dim3 grid((unsigned)(g.n_seqs * g.H), (unsigned)(g.dv / p.dvs));
  kern<<<grid, kSimtThreads, smem, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? CKDA_OK : CKDA_ERR_CUDA;
}

}  // namespace

int launch_chunk_simt(const ChunkArgs &g, cudaStream_t s) {
  if (g.n_seqs * g.H == 0) return CKDA_OK;
  const bool in_bf = g.io_dtype == CKDA_BF16, out_bf = g.o_dtype == CKDA_BF16;
  if (in_bf && out_bf) return launch_typed<__nv_bfloat16, __nv_bfloat16>(g, s);
  if (in_bf) return launch_typed<__nv_bfloat16, float>(g, s);
  if (out_bf) return launch_typed<float, __nv_bfloat16>(g, s);
  return launch_typed<float, float>(g, s);
}

}  // namespace ckda

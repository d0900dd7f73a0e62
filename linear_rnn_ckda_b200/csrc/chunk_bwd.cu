// chunk_bwd.cu -- exact fp32 chunkwise backward of the gated delta rule (CUDA cores).
//
// Gradients of L = sum dO . o + sum dS_T . S_T with respect to q, k, v, the gate and
// strength logits a, b and the initial state S0, for the forward of ckda_chunk_fwd.  The
// CKDA review measures its kernels forward plus backward (Figure 5); the pages give no
// backward formulas, so this is the chain rule of the chunkwise (UT) form, walked in reverse.
//
// Per chunk (rows r = 0..C-1, incoming state S, per-channel signed products
// G_r = prod_{s<=r} alpha_s, g = G_{C-1}, g(t, j) = prod_{s=j+1..t} alpha_s):
//   Kr = K*G   Qr = Q*G   Kd = K*g(C-1, .)       M = tril(Kr-pairs, -1), P = tril(Q-pairs)
//   M_rj = sum_c K_rc K_jc g(r,j)_c   P_rj = sum_c Q_rc K_jc g(r,j)_c   A = Diag(beta) M
//   Li = (I + A)^{-1}   T = Li Diag(beta)   V' = V - Kr S   U = T V'
//   O = Qr S + P U      S' = Diag(g) S + Kd^T U
// Reverse, given dO and dS' (the gradient of the outgoing state):
//   dU = Kd dS' + P^T dO        dV = dV' = T^T dU
//   dS = Diag(g) dS' + Qr^T dO - Kr^T dV'                       (the only sequential step)
//   dKd = U dS'^T   dQr = dO S^T   dKr = -dV' S^T   dP = tril(dO U^T)   dT = dU V'^T
//   dLi = dT Diag(beta), dbeta_j = sum_r Li_rj dT_rj;  dA = -Li^T dLi Li^T (strictly lower)
//   dbeta_r += sum_j dA_rj M_rj;  dM = Diag(beta) dA
//   dQ = dQr*G + sum_{j<=r} dP_rj K_j g(r,j)
//   dK = dKr*G + dKd*g(C-1,.) + sum_{j<r} dM_rj K_j g(r,j) + sum_{t>r} dM_tr K_t g(t,r)
//        + sum_{t>=r} dP_tr Q_t g(t,r)
//   d log|alpha_s| = sum_{t>=s} (dKr_t Kr_t + dQr_t Qr_t)           (state read)
//                  + sum_{t>=s>j} (dM_tj K_t K_j + dP_tj Q_t K_j) g(t,j)   (pairs across s)
//                  + sum_{t<s} dKd_t Kd_t + g (sum_j dS'_.j S_.j)   (state write, carry)
//   dalpha_s = d log|alpha_s| / alpha_s
// The gate gradient is formed from these terms only (each gate factor a product of |alpha|
// <= 1 over the rows it spans), never as a suffix sum of dG G, whose terms cancel pairwise.
// The kernel forms dalpha_s itself, not d log|alpha_s|: the derivative of each term's gate
// factor with respect to alpha_s is the product of the factor's other gates, so nothing is
// divided by alpha_s and an exact zero gate (where L, affine in each gate, still has its
// derivative) needs no special case.  Every gate product is exact (log-space prefixes with a
// zero count and a sign parity, as the exact forward).
//
// Passes: (1) the exact forward kernel, chunk 32, saves each chunk's incoming state;
// (2) bwd_reverse_kernel, one block per (sequence, head), walks the chunks last to first
// and saves each chunk's outgoing-state gradient dS'; (3) bwd_grad_kernel, one block per
// (chunk, head), forms every other gradient of its rows.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace ckda {
namespace {

constexpr int kBC = 32;          // backward chunk rows
constexpr int kBThreads = 256;
constexpr int kJS = 32;          // value columns per slice in the gradient pass

struct BwdParams {
  const void *q, *k, *v, *a, *dO;
  const float *b, *S0, *dS_T;
  const int32_t *cu;
  float *gq, *gk, *gv, *ga, *gb, *gS0;   // gradients (fp32)
  const float *S_in;   // [slot][H][dk][dv] incoming state of every chunk (pass 1)
  float *dS_out;       // [slot][H][dk][dv] gradient of every chunk's outgoing state (pass 2)
  int *status;
  int n_seqs, T, H, dk, dv, signed_gate;
  long n_slots;
};

// The sequence's token range; false (status recorded by the first pass) if its offsets are bad.
__device__ __forceinline__ bool seq_range(const BwdParams &p, int n, long &t0, long &t1,
                                          long &bofs) {
  if (p.cu) {
    t0 = p.cu[n];
    t1 = p.cu[n + 1];
    bofs = 0;
    return !(t0 < 0 || t1 < t0 || t1 > p.T || (n == 0 && t0 != 0) ||
             (n == p.n_seqs - 1 && t1 != p.T));
  }
  t0 = 0;
  t1 = p.T;
  bofs = (long)n * p.T;
  return true;
}

// Shared chunk set-up of passes 2 and 3: q, k and the gate prefix of a chunk's rows.
//   sQ, sK [kBC][ldk]: q, k (rows past the end: 0)
//   sL     [kBC][ldk]: L_r = sum of log2|alpha| over the non-zero gates of rows 0..r
//   sZ     [kBC][ldz]: (zero count << 1) | sign parity of rows 0..r
//   sBeta  [kBC], sGC [dk] = g (exact), sLC [dk], sZC [dk]
//   (CKDA_QK_L2NORM: q and k divided by their norms; the factors go to sInvQ / sInvK)
template <typename TIn>
__device__ void load_chunk(const BwdParams &p, long row0, int nrows, int h, float *sQ, float *sK,
                           float *sL, uint8_t *sZ, float *sBeta, float *sGC, float *sLC, int *sZC,
                           float *sInvQ, float *sInvK) {
  const bool per_head = per_head_gate(p.signed_gate);
  const int dk = p.dk, ldk = dk + 1, ldz = dk + 4, H = p.H, tid = threadIdx.x;
  const TIn *q = static_cast<const TIn *>(p.q);
  const TIn *k = static_cast<const TIn *>(p.k);
  const TIn *a = static_cast<const TIn *>(p.a);
  for (int e = tid; e < kBC * dk; e += kBThreads) {
    const int r = e / dk, c = e % dk;
    float qv = 0.f, kv = 0.f, av = 0.f;
    if (r < nrows) {
      const size_t row = (size_t)(row0 + r) * H + h;
      qv = to_f32(q[row * dk + c]);
      kv = to_f32(k[row * dk + c]);
      av = to_f32(a[per_head ? row : row * dk + c]);
    }
    sQ[r * ldk + c] = qv;
    sK[r * ldk + c] = kv;
    sL[r * ldk + c] = av;
  }
  for (int r = tid; r < kBC; r += kBThreads)
    sBeta[r] = r < nrows ? gate_beta(p.b[(size_t)(row0 + r) * H + h], p.signed_gate) : 0.f;
  __syncthreads();
  for (int c = tid; c < dk; c += kBThreads) {
    float L = 0.f;
    int zc = 0, par = 0;
    for (int r = 0; r < kBC; ++r) {
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
    sGC[c] = zc ? 0.f : (par ? -exp2f(L) : exp2f(L));
  }
  __syncthreads();
  if (qk_l2norm(p.signed_gate)) {
    l2norm_rows2(sQ, sK, ldk, nrows, dk, sInvQ, sInvK);
    __syncthreads();
  }
}

// g(t, j)_c from the prefixes (exact: 0 when a zero gate lies in (j, t])
__device__ __forceinline__ float pair_gate(const float *sL, const uint8_t *sZ, int ldk, int ldz,
                                           int t, int j, int c) {
  const int zt = sZ[t * ldz + c], zj = sZ[j * ldz + c];
  if ((zt >> 1) != (zj >> 1)) return 0.f;
  const float f = exp2f(sL[t * ldk + c] - sL[j * ldk + c]);
  return ((zt ^ zj) & 1) ? -f : f;
}
// G_r (exact) and g(C-1, r) (exact)
__device__ __forceinline__ float prefix_gate(const float *sL, const uint8_t *sZ, int ldk, int ldz,
                                             int r, int c) {
  const int z = sZ[r * ldz + c];
  if (z >> 1) return 0.f;
  const float f = exp2f(sL[r * ldk + c]);
  return (z & 1) ? -f : f;
}
__device__ __forceinline__ float suffix_gate(const float *sL, const uint8_t *sZ, const float *sLC,
                                             const int *sZC, int ldk, int ldz, int r, int c) {
  const int z = sZ[r * ldz + c], zC = sZC[c];
  if ((z >> 1) != (zC >> 1)) return 0.f;
  const float f = exp2f(sLC[c] - sL[r * ldk + c]);
  return ((z ^ zC) & 1) ? -f : f;
}

// M (strictly lower, without beta) and P (lower, diagonal included), exact pair factors
__device__ void pair_products(int dk, const float *sQ, const float *sK, const float *sL,
                              const uint8_t *sZ, float *sM, float *sP) {
  const int ldk = dk + 1, ldz = dk + 4, tid = threadIdx.x;
  const int npairs = kBC * (kBC + 1) / 2;
  for (int e = tid; e < npairs; e += kBThreads) {
    int r = (int)((sqrtf(8.f * e + 1.f) - 1.f) * 0.5f);
    while (r * (r + 1) / 2 > e) --r;
    while ((r + 1) * (r + 2) / 2 <= e) ++r;
    const int j = e - r * (r + 1) / 2;
    float accM = 0.f, accP = 0.f;
    for (int c = 0; c < dk; ++c) {
      const float f = pair_gate(sL, sZ, ldk, ldz, r, j, c);
      if (f == 0.f) continue;
      const float kj = sK[j * ldk + c] * f;
      accM = fmaf(sK[r * ldk + c], kj, accM);
      accP = fmaf(sQ[r * ldk + c], kj, accP);
    }
    sM[r * kBC + j] = (j < r) ? accM : 0.f;
    sP[r * kBC + j] = accP;
    if (j < r) {
      sM[j * kBC + r] = 0.f;
      sP[j * kBC + r] = 0.f;
    }
  }
  __syncthreads();
}

// Li = (I + Diag(beta) M)^{-1} (unit lower triangular), forward substitution row by row
__device__ void unit_lower_inverse(const float *sM, const float *sBeta, float *sLi) {
  const int tid = threadIdx.x;
  for (int e = tid; e < kBC * kBC; e += kBThreads) {
    const int r = e / kBC, m = e % kBC;
    sLi[e] = (r == m) ? 1.f : 0.f;
  }
  __syncthreads();
  // row r: Li_rm = -sum_{m <= j < r} A_rj Li_jm   (A_rj = beta_r M_rj)
  for (int r = 1; r < kBC; ++r) {
    float x = 0.f;
    const int m = tid;
    if (m < r) {
      for (int j = m; j < r; ++j) x = fmaf(sBeta[r] * sM[r * kBC + j], sLi[j * kBC + m], x);
    }
    __syncthreads();
    if (m < r) sLi[r * kBC + m] = -x;
    __syncthreads();
  }
}

// ------------------------------------------------------------------ pass 2: dS, last chunk first
template <typename TIn, typename TG>
__global__ void __launch_bounds__(kBThreads, 1) bwd_reverse_kernel(BwdParams p) {
  extern __shared__ float smem[];
  const int dk = p.dk, dv = p.dv, ldk = dk + 1, ldz = dk + 4, H = p.H, tid = threadIdx.x;
  float *sdS = smem;                                  // [dk][dv]
  float *sQ = sdS + (size_t)dk * dv;                  // [kBC][ldk] q, then Qr
  float *sK = sQ + kBC * ldk;                         // [kBC][ldk] k, then Kr
  float *sL = sK + kBC * ldk;                         // [kBC][ldk] prefix, then Kd
  uint8_t *sZ = reinterpret_cast<uint8_t *>(sL + kBC * ldk);
  float *sM = reinterpret_cast<float *>(sZ + kBC * ldz);  // [kBC][kBC] M, then T
  float *sP = sM + kBC * kBC;
  float *sLi = sP + kBC * kBC;
  float *sdO = sLi + kBC * kBC;                       // [kBC][dv]
  float *sdU = sdO + kBC * dv;                        // [kBC][dv]
  float *sdV = sdU + kBC * dv;                        // [kBC][dv]
  float *sBeta = sdV + kBC * dv;
  float *sGC = sBeta + kBC;
  float *sLC = sGC + dk;
  float *sInv = sLC + dk;                             // [2][kBC] 1 / row norms of q and k
  int *sZC = reinterpret_cast<int *>(sInv + 2 * kBC);

  const int unit = blockIdx.x, n = unit / H, h = unit % H;
  long t0, t1, bofs;
  if (!seq_range(p, n, t0, t1, bofs)) return;
  const size_t sofs = ((size_t)n * H + h) * dk * dv;
  const long slot0 = chunk_slot_base(p.cu, n, p.T, kBC);
  const TG *dO = static_cast<const TG *>(p.dO);

  for (int e = tid; e < dk * dv; e += kBThreads) sdS[e] = p.dS_T ? p.dS_T[sofs + e] : 0.f;
  const long nch = (t1 - t0 + kBC - 1) / kBC;
  for (long ci = nch - 1; ci >= 0; --ci) {
    const long cs = t0 + ci * kBC;
    const int nrows = (int)(t1 - cs < kBC ? t1 - cs : kBC);
    __syncthreads();
    load_chunk<TIn>(p, bofs + cs, nrows, h, sQ, sK, sL, sZ, sBeta, sGC, sLC, sZC, sInv,
                    sInv + kBC);
    for (int e = tid; e < kBC * dv; e += kBThreads) {
      const int r = e / dv, j = e % dv;
      sdO[e] = (r < nrows && dO) ? to_f32(dO[((size_t)(bofs + cs + r) * H + h) * dv + j]) : 0.f;
    }
    pair_products(dk, sQ, sK, sL, sZ, sM, sP);
    unit_lower_inverse(sM, sBeta, sLi);
    // T = Li Diag(beta) over M; Qr, Kr, Kd in place
    for (int e = tid; e < kBC * kBC; e += kBThreads) sM[e] = sLi[e] * sBeta[e % kBC];
    for (int e = tid; e < kBC * dk; e += kBThreads) {
      const int r = e / dk, c = e % dk;
      const float G = prefix_gate(sL, sZ, ldk, ldz, r, c);
      const float gd = suffix_gate(sL, sZ, sLC, sZC, ldk, ldz, r, c);
      const float kv = sK[r * ldk + c];
      sQ[r * ldk + c] *= G;
      sK[r * ldk + c] = kv * G;
      sL[r * ldk + c] = kv * gd;
    }
    // the gradient of this chunk's outgoing state, for the gradient pass
    float *dst = p.dS_out + ((size_t)(slot0 + ci) * H + h) * dk * dv;
    for (int e = tid; e < dk * dv; e += kBThreads) dst[e] = sdS[e];
    __syncthreads();
    // dU = Kd dS' + P^T dO
    for (int e = tid; e < kBC * dv; e += kBThreads) {
      const int r = e / dv, j = e % dv;
      float acc = 0.f;
      for (int c = 0; c < dk; ++c) acc = fmaf(sL[r * ldk + c], sdS[c * dv + j], acc);
      for (int t = r; t < kBC; ++t) acc = fmaf(sP[t * kBC + r], sdO[t * dv + j], acc);
      sdU[e] = acc;
    }
    __syncthreads();
    // dV' = T^T dU
    for (int e = tid; e < kBC * dv; e += kBThreads) {
      const int r = e / dv, j = e % dv;
      float acc = 0.f;
      for (int t = r; t < kBC; ++t) acc = fmaf(sM[t * kBC + r], sdU[t * dv + j], acc);
      sdV[e] = acc;
    }
    __syncthreads();
    // dS = Diag(g) dS' + Qr^T dO - Kr^T dV'
    for (int e = tid; e < dk * dv; e += kBThreads) {
      const int c = e / dv, j = e % dv;
      float acc = sGC[c] * sdS[e];
      for (int r = 0; r < kBC; ++r) {
        acc = fmaf(sQ[r * ldk + c], sdO[r * dv + j], acc);
        acc = fmaf(-sK[r * ldk + c], sdV[r * dv + j], acc);
      }
      sdS[e] = acc;
    }
  }
  __syncthreads();
  if (p.gS0)
    for (int e = tid; e < dk * dv; e += kBThreads) p.gS0[sofs + e] = sdS[e];
}

// ------------------------------------------------------------------ pass 3: gradients of a chunk
template <typename TIn, typename TG>
__global__ void __launch_bounds__(kBThreads, 1) bwd_grad_kernel(BwdParams p) {
  extern __shared__ float smem[];
  const int dk = p.dk, dv = p.dv, ldk = dk + 1, ldz = dk + 4, H = p.H, tid = threadIdx.x;
  float *sQ = smem;                                   // [kBC][ldk] q
  float *sK = sQ + kBC * ldk;                         // [kBC][ldk] k
  float *sL = sK + kBC * ldk;                         // [kBC][ldk] gate prefix
  float *sKr = sL + kBC * ldk;                        // [kBC][ldk] K*G
  float *sKd = sKr + kBC * ldk;                       // [kBC][ldk] K*g(C-1,.)
  float *sdKr = sKd + kBC * ldk;                      // [kBC][ldk] accumulators
  float *sdQr = sdKr + kBC * ldk;
  float *sdKd = sdQr + kBC * ldk;
  uint8_t *sZ = reinterpret_cast<uint8_t *>(sdKd + kBC * ldk);
  float *sM = reinterpret_cast<float *>(sZ + kBC * ldz);  // [kBC][kBC]
  float *sP = sM + kBC * kBC;
  float *sLi = sP + kBC * kBC;
  float *sdP = sLi + kBC * kBC;
  float *sdT = sdP + kBC * kBC;                        // dT, then dLi, then X, then dA
  float *sX = sdT + kBC * kBC;                         // scratch [kBC][kBC]
  float *sS = sX + kBC * kBC;                          // [dk][kJS] slice of S
  float *sdS = sS + dk * kJS;                          // [dk][kJS] slice of dS'
  float *sVp = sdS + dk * kJS;                         // [kBC][kJS] V, then V'
  float *sU = sVp + kBC * kJS;
  float *sdO = sU + kBC * kJS;
  float *sdU = sdO + kBC * kJS;
  float *sdV = sdU + kBC * kJS;
  float *sBeta = sdV + kBC * kJS;
  float *sdBeta = sBeta + kBC;
  float *sGC = sdBeta + kBC;
  float *sLC = sGC + dk;
  float *sCarry = sLC + dk;                            // sum_j dS'_cj S_cj
  float *sInvQ = sCarry + dk;                          // [kBC] 1 / ||q_r|| (CKDA_QK_L2NORM)
  float *sInvK = sInvQ + kBC;                          // [kBC] 1 / ||k_r||
  float *sDaRow = sInvK + kBC;                         // [kBC] per-head gate gradient
  int *sZC = reinterpret_cast<int *>(sDaRow + kBC);

  // slot -> (sequence, chunk)
  const long slot = blockIdx.x;
  const int h = blockIdx.y;
  int n;
  if (p.cu) {
    int lo = 0, hi = p.n_seqs - 1;   // the last sequence whose base is <= slot
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (chunk_slot_base(p.cu, mid, p.T, kBC) <= slot) lo = mid; else hi = mid - 1;
    }
    n = lo;
  } else {
    n = (int)(slot / ((p.T + kBC - 1) / kBC));
  }
  if (n < 0 || n >= p.n_seqs) return;
  long t0, t1, bofs;
  if (!seq_range(p, n, t0, t1, bofs)) return;
  const long ci = slot - chunk_slot_base(p.cu, n, p.T, kBC);
  const long cs = t0 + ci * kBC;
  if (ci < 0 || cs >= t1) return;   // a slot between two sequences' chunks
  const int nrows = (int)(t1 - cs < kBC ? t1 - cs : kBC);
  const long row0 = bofs + cs;
  const TIn *v = static_cast<const TIn *>(p.v);
  const TIn *a = static_cast<const TIn *>(p.a);
  const TG *dO = static_cast<const TG *>(p.dO);
  const float *S_in = p.S_in + ((size_t)slot * H + h) * dk * dv;
  const float *dSo = p.dS_out + ((size_t)slot * H + h) * dk * dv;

  const bool per_head = per_head_gate(p.signed_gate), l2 = qk_l2norm(p.signed_gate);
  load_chunk<TIn>(p, row0, nrows, h, sQ, sK, sL, sZ, sBeta, sGC, sLC, sZC, sInvQ, sInvK);
  for (int r = tid; r < kBC; r += kBThreads) sDaRow[r] = 0.f;
  pair_products(dk, sQ, sK, sL, sZ, sM, sP);
  unit_lower_inverse(sM, sBeta, sLi);
  for (int e = tid; e < kBC * dk; e += kBThreads) {
    const int r = e / dk, c = e % dk;
    const float kv = sK[r * ldk + c];
    sKr[r * ldk + c] = kv * prefix_gate(sL, sZ, ldk, ldz, r, c);
    sKd[r * ldk + c] = kv * suffix_gate(sL, sZ, sLC, sZC, ldk, ldz, r, c);
    sdKr[r * ldk + c] = 0.f;
    sdQr[r * ldk + c] = 0.f;
    sdKd[r * ldk + c] = 0.f;
  }
  for (int e = tid; e < kBC * kBC; e += kBThreads) {
    sdP[e] = 0.f;
    sdT[e] = 0.f;
  }
  for (int c = tid; c < dk; c += kBThreads) sCarry[c] = 0.f;
  __syncthreads();

  // ---- value-column slices: V', U, dU, dV' (-> dv) and the sums over value columns
  for (int j0 = 0; j0 < dv; j0 += kJS) {
    const int js = min(kJS, dv - j0);
    for (int e = tid; e < dk * js; e += kBThreads) {
      const int c = e / js, j = e % js;
      sS[c * kJS + j] = S_in[(size_t)c * dv + j0 + j];
      sdS[c * kJS + j] = dSo[(size_t)c * dv + j0 + j];
    }
    for (int e = tid; e < kBC * js; e += kBThreads) {
      const int r = e / js, j = e % js;
      const size_t idx = ((size_t)(row0 + r) * H + h) * dv + j0 + j;
      sVp[r * kJS + j] = r < nrows ? to_f32(v[idx]) : 0.f;
      sdO[r * kJS + j] = (r < nrows && dO) ? to_f32(dO[idx]) : 0.f;
    }
    __syncthreads();
    // V' = V - Kr S
    for (int e = tid; e < kBC * js; e += kBThreads) {
      const int r = e / js, j = e % js;
      float acc = sVp[r * kJS + j];
      for (int c = 0; c < dk; ++c) acc = fmaf(-sKr[r * ldk + c], sS[c * kJS + j], acc);
      sVp[r * kJS + j] = acc;
    }
    __syncthreads();
    // U = Li Diag(beta) V';  dU = Kd dS' + P^T dO
    for (int e = tid; e < kBC * js; e += kBThreads) {
      const int r = e / js, j = e % js;
      float u = 0.f;
      for (int m = 0; m <= r; ++m) u = fmaf(sLi[r * kBC + m] * sBeta[m], sVp[m * kJS + j], u);
      sU[r * kJS + j] = u;
      float du = 0.f;
      for (int c = 0; c < dk; ++c) du = fmaf(sKd[r * ldk + c], sdS[c * kJS + j], du);
      for (int t = r; t < kBC; ++t) du = fmaf(sP[t * kBC + r], sdO[t * kJS + j], du);
      sdU[r * kJS + j] = du;
    }
    __syncthreads();
    // dV' = T^T dU = Diag(beta) Li^T dU  (the gradient of v)
    for (int e = tid; e < kBC * js; e += kBThreads) {
      const int r = e / js, j = e % js;
      float acc = 0.f;
      for (int t = r; t < kBC; ++t) acc = fmaf(sLi[t * kBC + r], sdU[t * kJS + j], acc);
      acc *= sBeta[r];
      sdV[r * kJS + j] = acc;
      if (r < nrows) p.gv[((size_t)(row0 + r) * H + h) * dv + j0 + j] = acc;
    }
    __syncthreads();
    // sums over this slice's value columns
    for (int e = tid; e < kBC * dk; e += kBThreads) {
      const int r = e / dk, c = e % dk;
      float akd = 0.f, aqr = 0.f, akr = 0.f;
      for (int j = 0; j < js; ++j) {
        const float s = sS[c * kJS + j];
        akd = fmaf(sU[r * kJS + j], sdS[c * kJS + j], akd);
        aqr = fmaf(sdO[r * kJS + j], s, aqr);
        akr = fmaf(-sdV[r * kJS + j], s, akr);
      }
      sdKd[r * ldk + c] += akd;
      sdQr[r * ldk + c] += aqr;
      sdKr[r * ldk + c] += akr;
    }
    for (int e = tid; e < kBC * kBC; e += kBThreads) {
      const int r = e / kBC, m = e % kBC;
      if (m > r) continue;
      float adp = 0.f, adt = 0.f;
      for (int j = 0; j < js; ++j) {
        adp = fmaf(sdO[r * kJS + j], sU[m * kJS + j], adp);
        adt = fmaf(sdU[r * kJS + j], sVp[m * kJS + j], adt);
      }
      sdP[e] += adp;
      sdT[e] += adt;
    }
    for (int c = tid; c < dk; c += kBThreads) {
      float acc = 0.f;
      for (int j = 0; j < js; ++j) acc = fmaf(sdS[c * kJS + j], sS[c * kJS + j], acc);
      sCarry[c] += acc;
    }
    __syncthreads();
  }

  // ---- through T = Li Diag(beta) and Li = (I + A)^{-1}
  // dbeta_m = sum_r Li_rm dT_rm;  dLi = dT Diag(beta) (in place)
  for (int m = tid; m < kBC; m += kBThreads) {
    float acc = 0.f;
    for (int r = m; r < kBC; ++r) acc = fmaf(sLi[r * kBC + m], sdT[r * kBC + m], acc);
    sdBeta[m] = acc;
  }
  __syncthreads();
  for (int e = tid; e < kBC * kBC; e += kBThreads) sdT[e] *= sBeta[e % kBC];
  __syncthreads();
  // X = dLi Li^T
  for (int e = tid; e < kBC * kBC; e += kBThreads) {
    const int r = e / kBC, m = e % kBC;
    float acc = 0.f;
    for (int j = 0; j < kBC; ++j) acc = fmaf(sdT[r * kBC + j], sLi[m * kBC + j], acc);
    sX[e] = acc;
  }
  __syncthreads();
  // dA = -Li^T X, strictly lower (over dT); dbeta_r += sum_j dA_rj M_rj; dM = beta_r dA (over dT)
  for (int e = tid; e < kBC * kBC; e += kBThreads) {
    const int r = e / kBC, j = e % kBC;
    float acc = 0.f;
    if (j < r)
      for (int t = 0; t < kBC; ++t) acc = fmaf(sLi[t * kBC + r], sX[t * kBC + j], acc);
    sdT[e] = -acc;
  }
  __syncthreads();
  for (int r = tid; r < kBC; r += kBThreads) {
    float acc = 0.f;
    for (int j = 0; j < r; ++j) acc = fmaf(sdT[r * kBC + j], sM[r * kBC + j], acc);
    sdBeta[r] += acc;
  }
  __syncthreads();
  for (int e = tid; e < kBC * kBC; e += kBThreads) sdT[e] *= sBeta[e / kBC];   // dM
  __syncthreads();
  const float *sdM = sdT;

  // ---- dq, dk of the rows
  for (int e = tid; e < kBC * dk; e += kBThreads) {
    const int r = e / dk, c = e % dk;
    if (r >= nrows) continue;
    const float G = prefix_gate(sL, sZ, ldk, ldz, r, c);
    const float gd = suffix_gate(sL, sZ, sLC, sZC, ldk, ldz, r, c);
    float dqv = sdQr[r * ldk + c] * G;
    float dkv = sdKr[r * ldk + c] * G + sdKd[r * ldk + c] * gd;
    for (int j = 0; j <= r; ++j) {
      const float f = pair_gate(sL, sZ, ldk, ldz, r, j, c);
      dqv = fmaf(sdP[r * kBC + j] * sK[j * ldk + c], f, dqv);
      if (j < r) dkv = fmaf(sdM[r * kBC + j] * sK[j * ldk + c], f, dkv);
    }
    for (int t = r; t < kBC; ++t) {
      const float f = pair_gate(sL, sZ, ldk, ldz, t, r, c);
      float w = sdP[t * kBC + r] * sQ[t * ldk + c];
      if (t > r) w = fmaf(sdM[t * kBC + r], sK[t * ldk + c], w);
      dkv = fmaf(w, f, dkv);
    }
    if (l2) {   // gradients of the normalised q, k: the chain through the norm follows
      sKr[r * ldk + c] = dqv;
      sKd[r * ldk + c] = dkv;
    } else {
      const size_t idx = ((size_t)(row0 + r) * H + h) * dk + c;
      p.gq[idx] = dqv;
      p.gk[idx] = dkv;
    }
  }
  if (l2) {
    // x = y / ||y||:  dy = (dx - x (x . dx)) / ||y||   (one warp per row)
    __syncthreads();
    const int warp = tid >> 5, lane = tid & 31;
    for (int r = warp; r < nrows; r += kBThreads / 32) {
      float dq_dot = 0.f, dk_dot = 0.f;
      for (int c = lane; c < dk; c += 32) {
        dq_dot = fmaf(sQ[r * ldk + c], sKr[r * ldk + c], dq_dot);
        dk_dot = fmaf(sK[r * ldk + c], sKd[r * ldk + c], dk_dot);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        dq_dot += __shfl_xor_sync(0xffffffffu, dq_dot, off);
        dk_dot += __shfl_xor_sync(0xffffffffu, dk_dot, off);
      }
      for (int c = lane; c < dk; c += 32) {
        const size_t idx = ((size_t)(row0 + r) * H + h) * dk + c;
        p.gq[idx] = sInvQ[r] * fmaf(-sQ[r * ldk + c], dq_dot, sKr[r * ldk + c]);
        p.gk[idx] = sInvK[r] * fmaf(-sK[r * ldk + c], dk_dot, sKd[r * ldk + c]);
      }
    }
  }

  // ---- gate gradient, one thread per channel.  dL/dalpha_s is the derivative of the gate
  // factors of the terms above with respect to alpha_s, every factor a product over rows
  // other than s (so nothing is divided by alpha_s, and an exact zero gate needs no care):
  //   dalpha_s = G_{s-1} RS(s) + g(C-1,s) WS(s) + sum_{t>=s} g(t,s) inner_t(s)
  //              + G_{s-1} g(C-1,s) carry
  //   x_t = dKr_t K_t + dQr_t Q_t        RS(s) = sum_{t>=s} x_t g(t,s) = x_s + alpha_{s+1} RS(s+1)
  //   z_t = dKd_t K_t                    WS(s) = sum_{t<s} z_t g(s-1,t): WS(s+1) = z_s + alpha_s WS(s)
  //   c_tj = (dM_tj K_t + dP_tj Q_t) K_j inner_t(s) = sum_{j<s} c_tj g(s-1,j):
  //                                      inner_t(s+1) = c_ts + alpha_s inner_t(s)
  // Every sum is accumulated term by term (no total minus a prefix, which cancels when a
  // chunk's gates decay strongly).
  for (int c = tid; c < dk; c += kBThreads) {
    float RS[kBC];
    float run = 0.f;
#pragma unroll
    for (int t = kBC - 1; t >= 0; --t) {
      const float x = sdKr[t * ldk + c] * sK[t * ldk + c] + sdQr[t * ldk + c] * sQ[t * ldk + c];
      const float al_next = t + 1 < kBC ? pair_gate(sL, sZ, ldk, ldz, t + 1, t, c) : 0.f;
      run = fmaf(al_next, run, x);
      RS[t] = run;
    }
    float inner[kBC];
#pragma unroll
    for (int t = 0; t < kBC; ++t) inner[t] = 0.f;
    float WS = 0.f;
    const float carry = sCarry[c];
#pragma unroll
    for (int s = 0; s < kBC; ++s) {
      if (s < nrows) {
        const float Gp = s > 0 ? prefix_gate(sL, sZ, ldk, ldz, s - 1, c) : 1.f;
        const float gd = suffix_gate(sL, sZ, sLC, sZC, ldk, ldz, s, c);
        float pairs = 0.f;
#pragma unroll
        for (int t = s; t < kBC; ++t) {
          const float f = t == s ? 1.f : pair_gate(sL, sZ, ldk, ldz, t, s, c);
          pairs = fmaf(f, inner[t], pairs);
        }
        const float dalpha = fmaf(Gp, RS[s], fmaf(gd, WS, fmaf(Gp * gd, carry, pairs)));
        if (per_head) {
          atomicAdd(&sDaRow[s], dalpha);   // one gate shared by every key channel
        } else {
          const size_t idx = ((size_t)(row0 + s) * H + h) * dk + c;
          p.ga[idx] = dalpha * dalpha_da(to_f32(a[idx]), p.signed_gate);
        }
      }
      // advance WS and inner_t past row s
      const float al = s > 0 ? pair_gate(sL, sZ, ldk, ldz, s, s - 1, c) : prefix_gate(sL, sZ, ldk, ldz, 0, c);
      const float z = sdKd[s * ldk + c] * sK[s * ldk + c];
      WS = fmaf(al, WS, z);
      const float ks = sK[s * ldk + c];
#pragma unroll
      for (int t = s + 1; t < kBC; ++t) {
        const float cts = (sdM[t * kBC + s] * sK[t * ldk + c] + sdP[t * kBC + s] * sQ[t * ldk + c]) * ks;
        inner[t] = fmaf(al, inner[t], cts);
      }
    }
  }
  __syncthreads();
  for (int r = tid; r < nrows; r += kBThreads) {
    const size_t row = (size_t)(row0 + r) * H + h;
    p.gb[row] = sdBeta[r] * dbeta_db(p.b[row], p.signed_gate);
    if (per_head) p.ga[row] = sDaRow[r] * dalpha_da(to_f32(a[row]), p.signed_gate);
  }
}

size_t reverse_smem(int dk, int dv) {
  const int ldk = dk + 1, ldz = dk + 4;
  return sizeof(float) * ((size_t)dk * dv + 3 * kBC * ldk + 3 * kBC * kBC + 3 * kBC * dv + kBC +
                          2 * dk + 2 * kBC) +
         (size_t)kBC * ldz + sizeof(int) * dk + 64;
}
size_t grad_smem(int dk) {
  const int ldk = dk + 1, ldz = dk + 4;
  return sizeof(float) * ((size_t)8 * kBC * ldk + 6 * kBC * kBC + 2 * dk * kJS + 5 * kBC * kJS +
                          2 * kBC + 3 * dk + 3 * kBC) +
         (size_t)kBC * ldz + sizeof(int) * dk + 64;
}

template <typename TIn, typename TG>
int launch_typed(const BwdArgs &g, cudaStream_t stream) {
  BwdParams p;
  p.q = g.q; p.k = g.k; p.v = g.v; p.a = g.a; p.dO = g.dO; p.b = g.b; p.S0 = g.S0;
  p.dS_T = g.dS_T; p.cu = g.cu_seqlens;
  p.gq = g.gq; p.gk = g.gk; p.gv = g.gv; p.ga = g.ga; p.gb = g.gb; p.gS0 = g.gS0;
  p.S_in = g.S_chunks; p.dS_out = g.dS_chunks; p.status = g.status;
  p.n_seqs = g.n_seqs; p.T = g.T; p.H = g.H; p.dk = g.dk; p.dv = g.dv;
  p.signed_gate = g.signed_gate; p.n_slots = g.n_slots;
  const size_t sr = reverse_smem(g.dk, g.dv), sg = grad_smem(g.dk);
  auto kr = bwd_reverse_kernel<TIn, TG>;
  auto kg = bwd_grad_kernel<TIn, TG>;
  if (cudaFuncSetAttribute(kr, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sr) !=
          cudaSuccess ||
      cudaFuncSetAttribute(kg, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sg) != cudaSuccess)
    return CKDA_ERR_CUDA;
  kr<<<(unsigned)(g.n_seqs * g.H), kBThreads, sr, stream>>>(p);
  if (cudaGetLastError() != cudaSuccess) return CKDA_ERR_CUDA;
  if (g.n_slots > 0) {
    kg<<<dim3((unsigned)g.n_slots, (unsigned)g.H), kBThreads, sg, stream>>>(p);
    if (cudaGetLastError() != cudaSuccess) return CKDA_ERR_CUDA;
  }
  return CKDA_OK;
}

}  // namespace

int bwd_chunk_rows() { return kBC; }

int launch_chunk_bwd(const BwdArgs &g, cudaStream_t s) {
  if (g.n_seqs * g.H == 0) return CKDA_OK;
  // pass 1: the exact forward at the backward's chunk size, saving every chunk's state
  ChunkArgs f;
  f.q = g.q; f.k = g.k; f.v = g.v; f.a = g.a; f.b = g.b; f.S0 = g.S0; f.cu_seqlens = g.cu_seqlens;
  f.o = nullptr; f.S_T = nullptr; f.n_seqs = g.n_seqs; f.B = g.B; f.T = g.T; f.H = g.H;
  f.dk = g.dk; f.dv = g.dv; f.chunk = kBC; f.signed_gate = g.signed_gate;
  f.io_dtype = g.io_dtype; f.o_dtype = CKDA_F32; f.status = g.status; f.workspace = nullptr;
  f.workspace_bytes = 0; f.inject_chunk = -1; f.inject_wait_ns = 0; f.S_chunks = g.S_chunks;
  const int rc = launch_chunk_simt(f, s);
  if (rc != CKDA_OK) return rc;
  const bool in_bf = g.io_dtype == CKDA_BF16, do_bf = g.do_dtype == CKDA_BF16;
  if (in_bf && do_bf) return launch_typed<__nv_bfloat16, __nv_bfloat16>(g, s);
  if (in_bf) return launch_typed<__nv_bfloat16, float>(g, s);
  if (do_bf) return launch_typed<float, __nv_bfloat16>(g, s);
  return launch_typed<float, float>(g, s);
}

}  // namespace ckda

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
// Passes (all exact fp32):
//   (1) bwd_prep_kernel, one block per (chunk, head): the chunk's state-independent factors
//       (Kr, Kd, Qr, Li, P, M, beta, g) into a per-chunk record;
//   (2) bwd_state_fwd_kernel, one block per (sequence, head, value slice): the forward state
//       walk, first chunk to last, saving each chunk's incoming state S;
//   (3) bwd_state_rev_kernel, one block per (sequence, head, value slice): the reverse walk,
//       last chunk to first, saving each chunk's outgoing-state gradient dS';
//   (4) bwd_grad_kernel, one block per (chunk, head): every other gradient of its rows.
// The state passes are the only sequential steps; they read each chunk's record with one bulk
// copy and do three products per chunk, and the state's value columns evolve independently
// (S' = Diag(g) S + Kd^T U acts column by column), so a sequence's walk is split over slices
// of value columns.
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace ckda {
namespace {

using namespace sm100;

constexpr int kBC = 32;          // backward chunk rows
constexpr int kBThreads = 256;   // the state passes
constexpr int kGThreads = 512;   // the record and gradient passes (one chunk per block)
constexpr int kJS = 32;          // value columns per slice in the gradient pass
constexpr int kJP = kJS + 4;     // their row stride: 16-byte rows that start on distinct 16-byte bank groups
constexpr int kBP = kBC + 1;     // row stride of the gradient pass's [kBC][kBC] arrays (the same)
constexpr uint64_t kWaitNs = 2000000000ull;   // bound on a record copy's wait (2 s)

// Offsets (floats) of the factors in one (chunk slot, head) record; the forward state pass
// copies [kr, qr), the reverse pass [kr, m).
struct RecLayout {
  int kr, kd, li, beta, g, qr, pp, m, size;
};
__host__ __device__ __forceinline__ RecLayout rec_layout(int dk) {
  RecLayout L;
  L.kr = 0;
  L.kd = kBC * dk;
  L.li = 2 * kBC * dk;
  L.beta = L.li + kBC * kBC;
  L.g = L.beta + kBC;
  L.qr = L.g + dk;
  L.pp = L.qr + kBC * dk;
  L.m = L.pp + kBC * kBC;
  L.size = (int)bwd_record_floats(kBC, dk);
  return L;
}

struct BwdParams {
  const void *q, *k, *v, *a, *dO;
  const float *b, *S0, *dS_T;
  const int32_t *cu;
  float *gq, *gk, *gv, *ga, *gb, *gS0;   // gradients (fp32)
  float *S_in;         // [slot][H][dk][dv] incoming state of every chunk (pass 2)
  float *dS_out;       // [slot][H][dk][dv] gradient of every chunk's outgoing state (pass 3)
  float *rec;          // [slot][H][record] state-independent factors of every chunk (pass 1)
  int *status;
  int n_seqs, T, H, dk, dv, dvs, signed_gate;
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

// The chunk held by backward slot `slot`: its sequence n, the sequence's token range and the
// chunk's index ci in it.  False for a slot between two sequences' chunks (or past the last)
// and for a sequence with bad offsets.
__device__ __forceinline__ bool slot_chunk(const BwdParams &p, long slot, int &n, long &t0,
                                           long &t1, long &bofs, long &ci) {
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
  if (n < 0 || n >= p.n_seqs) return false;
  if (!seq_range(p, n, t0, t1, bofs)) return false;
  ci = slot - chunk_slot_base(p.cu, n, p.T, kBC);
  return ci >= 0 && t0 + ci * kBC < t1;
}

// Shared chunk set-up of the record and gradient passes: q, k and the gate prefix of a chunk's rows.
//   sQ, sK [kBC][ldk]: q, k (rows past the end: 0)
//   sL     [kBC][ldk]: L_r = sum of log2|alpha| over the non-zero gates of rows 0..r
//   sZ     [kBC][ldz]: (zero count << 1) | sign parity of rows 0..r
//   sBeta  [kBC], sGC [dk] = g (exact), sLC [dk], sZC [dk]
//   (CKDA_QK_L2NORM: q and k divided by their norms; the factors go to sInvQ / sInvK)
template <typename TIn>
__device__ void load_chunk(const BwdParams &p, long row0, int nrows, int h, int ldk, float *sQ,
                           float *sK, float *sL, uint8_t *sZ, float *sBeta, float *sGC, float *sLC,
                           int *sZC, float *sInvQ, float *sInvK) {
  const bool per_head = per_head_gate(p.signed_gate);
  const int dk = p.dk, ldz = dk + 4, H = p.H, tid = threadIdx.x;
  const TIn *q = static_cast<const TIn *>(p.q);
  const TIn *k = static_cast<const TIn *>(p.k);
  const TIn *a = static_cast<const TIn *>(p.a);
  for (int e = tid; e < kBC * dk; e += blockDim.x) {
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
  for (int r = tid; r < kBC; r += blockDim.x)
    sBeta[r] = r < nrows ? gate_beta(p.b[(size_t)(row0 + r) * H + h], p.signed_gate) : 0.f;
  __syncthreads();
  for (int c = tid; c < dk; c += blockDim.x) {
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
  for (int e = tid; e < npairs; e += blockDim.x) {
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

// Li = (I + Diag(beta) M)^{-1} (unit lower triangular) by one warp: lane m keeps column m in
// registers and finishes the rows in order, Li_rm = -beta_r sum_{m <= j < r} M_rj Li_jm (the
// rows of M read as broadcasts; no block barrier).  The caller synchronises after.
__device__ __forceinline__ void unit_lower_inverse_warp(const float *sM, const float *sBeta,
                                                        float *sLi) {
  const int m = threadIdx.x & 31;
  float col[kBC];
#pragma unroll
  for (int r = 0; r < kBC; ++r) {
    float x = 0.f;
#pragma unroll
    for (int j = 0; j < r; ++j) x = fmaf(sM[r * kBC + j], col[j], x);   // col[j] = 0 for j < m
    col[r] = r == m ? 1.f : (r < m ? 0.f : -sBeta[r] * x);
  }
#pragma unroll
  for (int r = 0; r < kBC; ++r) sLi[r * kBC + m] = col[r];
}

// ------------------------------------------------------------------ pass 1: chunk records
// One block per (chunk slot, head): Kr = K*G, Kd = K*g(C-1,.), Qr = Q*G, Li, P, M, beta, g.
template <typename TIn>
__global__ void __launch_bounds__(kGThreads) bwd_prep_kernel(BwdParams p) {
  extern __shared__ float smem[];
  const int dk = p.dk, ldk = dk + 1, ldz = dk + 4, H = p.H, tid = threadIdx.x;
  float *sQ = smem;                                   // [kBC][ldk] q
  float *sK = sQ + kBC * ldk;                         // [kBC][ldk] k
  float *sL = sK + kBC * ldk;                         // [kBC][ldk] gate prefix
  uint8_t *sZ = reinterpret_cast<uint8_t *>(sL + kBC * ldk);
  float *sM = reinterpret_cast<float *>(sZ + kBC * ldz);  // [kBC][kBC]
  float *sP = sM + kBC * kBC;
  float *sLi = sP + kBC * kBC;
  float *sBeta = sLi + kBC * kBC;
  float *sGC = sBeta + kBC;
  float *sLC = sGC + dk;
  float *sInv = sLC + dk;                             // [2][kBC]
  int *sZC = reinterpret_cast<int *>(sInv + 2 * kBC);

  const long slot = blockIdx.x;
  const int h = blockIdx.y;
  int n;
  long t0, t1, bofs, ci;
  if (!slot_chunk(p, slot, n, t0, t1, bofs, ci)) return;
  const long cs = t0 + ci * kBC;
  const int nrows = (int)(t1 - cs < kBC ? t1 - cs : kBC);
  load_chunk<TIn>(p, bofs + cs, nrows, h, ldk, sQ, sK, sL, sZ, sBeta, sGC, sLC, sZC, sInv,
                  sInv + kBC);
  pair_products(dk, sQ, sK, sL, sZ, sM, sP);
  // warp 0 inverts while the others write the gated rows
  if (tid < 32) unit_lower_inverse_warp(sM, sBeta, sLi);
  const RecLayout R = rec_layout(dk);
  float *rec = p.rec + ((size_t)slot * H + h) * R.size;
  for (int e = tid; e < kBC * dk; e += kGThreads) {
    const int r = e / dk, c = e % dk;
    const float G = prefix_gate(sL, sZ, ldk, ldz, r, c);
    const float gd = suffix_gate(sL, sZ, sLC, sZC, ldk, ldz, r, c);
    const float kv = sK[r * ldk + c];
    rec[R.kr + e] = kv * G;
    rec[R.kd + e] = kv * gd;
    rec[R.qr + e] = sQ[r * ldk + c] * G;
  }
  __syncthreads();
  for (int e = tid; e < kBC * kBC; e += kGThreads) {
    rec[R.li + e] = sLi[e];
    rec[R.pp + e] = sP[e];
    rec[R.m + e] = sM[e];
  }
  for (int r = tid; r < kBC; r += kGThreads) rec[R.beta + r] = sBeta[r];
  for (int c = tid; c < dk; c += kGThreads) rec[R.g + c] = sGC[c];
}

// The state passes read each chunk's record (floats [0, nfl)) into shared memory with one bulk
// copy, issued by thread 0 a chunk ahead into the other of two buffers.  Every thread waits on
// the copy's barrier and the block agrees on the outcome; on a wait that runs out (a copy that
// never lands: not expected) the status records CKDA_ERR_TIMEOUT and thread 0 waits once more
// for that copy (the only one in flight: the next is issued after a successful wait), so that
// none is in flight when the block exits.
__device__ __forceinline__ void issue_record(const float *src, float *dst, int nfl, uint64_t *bar) {
  fence_proxy_async();   // earlier reads of dst by this block precede the copy's writes
  mbar_arrive_expect_tx(bar, (uint32_t)nfl * sizeof(float));
  bulk_load(dst, src, (uint32_t)nfl * sizeof(float), bar);
}
__device__ __forceinline__ bool wait_record(const BwdParams &p, uint64_t *bar, uint32_t parity) {
  const bool ok = __syncthreads_and(mbar_wait(bar, parity, kWaitNs));
  if (!ok && threadIdx.x == 0) {
    set_status(p.status, CKDA_ERR_TIMEOUT);
    mbar_wait(bar, parity, kWaitNs);
  }
  return ok;
}

// ------------------------------------------------------------------ pass 2: the state, forward
// Block (sequence x head, slice of dvs value columns from j0): per chunk
//   V' = V - Kr S,   U = Li Diag(beta) V',   S <- Diag(g) S + Kd^T U
// saving the incoming S of every chunk.
template <typename TIn>
__global__ void __launch_bounds__(kBThreads) bwd_state_fwd_kernel(BwdParams p) {
  extern __shared__ __align__(16) float smem[];
  const int dk = p.dk, dv = p.dv, dvs = p.dvs, H = p.H, tid = threadIdx.x;
  const RecLayout R = rec_layout(dk);
  float *sRec2 = smem;                         // [2] floats [kr, qr) of a chunk's record
  float *sS = sRec2 + 2 * R.qr;                // [dk][dvs] state slice
  float *sV = sS + dk * dvs;                   // [kBC][dvs] v, then V'
  float *sU = sV + kBC * dvs;                  // [kBC][dvs]
  uint64_t *bar = reinterpret_cast<uint64_t *>(sU + kBC * dvs);   // [2]

  const int unit = blockIdx.x, n = unit / H, h = unit % H, j0 = blockIdx.y * dvs;
  long t0, t1, bofs;
  if (!seq_range(p, n, t0, t1, bofs)) {
    if (tid == 0 && blockIdx.y == 0) set_status(p.status, CKDA_ERR_SEQLENS);
    return;
  }
  const size_t sofs = ((size_t)n * H + h) * dk * dv;
  const long slot0 = chunk_slot_base(p.cu, n, p.T, kBC);
  const TIn *v = static_cast<const TIn *>(p.v);
  const long nch = (t1 - t0 + kBC - 1) / kBC;
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_init(bar + 1, 1);
    mbar_fence_init();
    if (nch > 0) issue_record(p.rec + ((size_t)slot0 * H + h) * R.size, sRec2, R.qr, bar);
  }
  for (int e = tid; e < dk * dvs; e += kBThreads) {
    const int c = e / dvs, j = e % dvs;
    sS[e] = p.S0 ? p.S0[sofs + (size_t)c * dv + j0 + j] : 0.f;
  }
  __syncthreads();
  for (long ci = 0; ci < nch; ++ci) {
    const long cs = t0 + ci * kBC;
    const int nrows = (int)(t1 - cs < kBC ? t1 - cs : kBC);
    const size_t slot = (size_t)(slot0 + ci);
    const int buf = (int)(ci & 1);
    for (int e = tid; e < kBC * dvs; e += kBThreads) {
      const int r = e / dvs, j = e % dvs;
      sV[e] = r < nrows ? to_f32(v[((size_t)(bofs + cs + r) * H + h) * dv + j0 + j]) : 0.f;
    }
    float *dst = p.S_in + (slot * H + h) * dk * dv;
    for (int e = tid; e < dk * dvs; e += kBThreads) {
      const int c = e / dvs, j = e % dvs;
      dst[(size_t)c * dv + j0 + j] = sS[e];
    }
    if (!wait_record(p, bar + buf, (uint32_t)((ci >> 1) & 1))) return;
    if (tid == 0 && ci + 1 < nch)
      issue_record(p.rec + ((slot + 1) * H + h) * R.size, sRec2 + (buf ^ 1) * R.qr, R.qr,
                   bar + (buf ^ 1));
    const float *sRec = sRec2 + buf * R.qr;
    const float *sKr = sRec + R.kr, *sKd = sRec + R.kd, *sLi = sRec + R.li,
                *sBeta = sRec + R.beta, *sG = sRec + R.g;
    // V' = V - Kr S: rows r0, r0 + 1 and columns jj, jj + 1 per thread
    for (int ti = tid; ti < (kBC / 2) * (dvs / 2); ti += kBThreads) {
      const int r0 = 2 * (ti / (dvs / 2)), jj = 2 * (ti % (dvs / 2));
      float a00 = sV[r0 * dvs + jj], a01 = sV[r0 * dvs + jj + 1];
      float a10 = sV[(r0 + 1) * dvs + jj], a11 = sV[(r0 + 1) * dvs + jj + 1];
      const float *k0 = sKr + r0 * dk, *k1 = k0 + dk;
      for (int c = 0; c < dk; c += 4) {
        const float4 x0 = *reinterpret_cast<const float4 *>(k0 + c);
        const float4 x1 = *reinterpret_cast<const float4 *>(k1 + c);
        const float xa[4] = {x0.x, x0.y, x0.z, x0.w}, xb[4] = {x1.x, x1.y, x1.z, x1.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 sv = *reinterpret_cast<const float2 *>(sS + (c + i) * dvs + jj);
          a00 = fmaf(-xa[i], sv.x, a00);
          a01 = fmaf(-xa[i], sv.y, a01);
          a10 = fmaf(-xb[i], sv.x, a10);
          a11 = fmaf(-xb[i], sv.y, a11);
        }
      }
      *reinterpret_cast<float2 *>(sV + r0 * dvs + jj) = make_float2(a00, a01);
      *reinterpret_cast<float2 *>(sV + (r0 + 1) * dvs + jj) = make_float2(a10, a11);
    }
    __syncthreads();
    // U = Li Diag(beta) V'  (Li lower triangular, zeros above the diagonal)
    for (int ti = tid; ti < (kBC / 2) * (dvs / 2); ti += kBThreads) {
      const int r0 = 2 * (ti / (dvs / 2)), jj = 2 * (ti % (dvs / 2));
      float a00 = 0.f, a01 = 0.f, a10 = 0.f, a11 = 0.f;
      for (int m = 0; m < r0 + 2; m += 4) {
        const float4 l0 = *reinterpret_cast<const float4 *>(sLi + r0 * kBC + m);
        const float4 l1 = *reinterpret_cast<const float4 *>(sLi + (r0 + 1) * kBC + m);
        const float4 bt = *reinterpret_cast<const float4 *>(sBeta + m);
        const float la[4] = {l0.x * bt.x, l0.y * bt.y, l0.z * bt.z, l0.w * bt.w};
        const float lb[4] = {l1.x * bt.x, l1.y * bt.y, l1.z * bt.z, l1.w * bt.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 vv = *reinterpret_cast<const float2 *>(sV + (m + i) * dvs + jj);
          a00 = fmaf(la[i], vv.x, a00);
          a01 = fmaf(la[i], vv.y, a01);
          a10 = fmaf(lb[i], vv.x, a10);
          a11 = fmaf(lb[i], vv.y, a11);
        }
      }
      *reinterpret_cast<float2 *>(sU + r0 * dvs + jj) = make_float2(a00, a01);
      *reinterpret_cast<float2 *>(sU + (r0 + 1) * dvs + jj) = make_float2(a10, a11);
    }
    __syncthreads();
    // S <- Diag(g) S + Kd^T U: key channels c0 .. c0 + 3, columns jj .. jj + 3 per thread
    for (int ti = tid; ti < (dk / 4) * (dvs / 4); ti += kBThreads) {
      const int c0 = 4 * (ti / (dvs / 4)), jj = 4 * (ti % (dvs / 4));
      float acc[4][4];
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const float4 sv = *reinterpret_cast<const float4 *>(sS + (c0 + x) * dvs + jj);
        const float gx = sG[c0 + x];
        acc[x][0] = gx * sv.x;
        acc[x][1] = gx * sv.y;
        acc[x][2] = gx * sv.z;
        acc[x][3] = gx * sv.w;
      }
      for (int r = 0; r < kBC; ++r) {
        const float4 kd = *reinterpret_cast<const float4 *>(sKd + r * dk + c0);
        const float4 u = *reinterpret_cast<const float4 *>(sU + r * dvs + jj);
        const float ka[4] = {kd.x, kd.y, kd.z, kd.w}, ua[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(ka[x], ua[y], acc[x][y]);
      }
#pragma unroll
      for (int x = 0; x < 4; ++x)
        *reinterpret_cast<float4 *>(sS + (c0 + x) * dvs + jj) =
            make_float4(acc[x][0], acc[x][1], acc[x][2], acc[x][3]);
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------ pass 3: the state gradient
// Block (sequence x head, value slice), last chunk first: with dS' the gradient of the chunk's
// outgoing state (saved),
//   dU = Kd dS' + P^T dO,   dV' = Diag(beta) Li^T dU,   dS = Diag(g) dS' + Qr^T dO - Kr^T dV'
template <typename TIn, typename TG>
__global__ void __launch_bounds__(kBThreads) bwd_state_rev_kernel(BwdParams p) {
  extern __shared__ __align__(16) float smem[];
  const int dk = p.dk, dv = p.dv, dvs = p.dvs, H = p.H, tid = threadIdx.x;
  const RecLayout R = rec_layout(dk);
  float *sRec2 = smem;                         // [2] floats [kr, m) of a chunk's record
  float *sdS = sRec2 + 2 * R.m;                // [dk][dvs]
  float *sdO = sdS + dk * dvs;                 // [kBC][dvs]
  float *sdU = sdO + kBC * dvs;
  float *sdV = sdU + kBC * dvs;
  uint64_t *bar = reinterpret_cast<uint64_t *>(sdV + kBC * dvs);   // [2]

  const int unit = blockIdx.x, n = unit / H, h = unit % H, j0 = blockIdx.y * dvs;
  long t0, t1, bofs;
  if (!seq_range(p, n, t0, t1, bofs)) return;   // recorded by the forward state pass
  const size_t sofs = ((size_t)n * H + h) * dk * dv;
  const long slot0 = chunk_slot_base(p.cu, n, p.T, kBC);
  const TG *dO = static_cast<const TG *>(p.dO);
  const long nch = (t1 - t0 + kBC - 1) / kBC;
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_init(bar + 1, 1);
    mbar_fence_init();
    if (nch > 0) issue_record(p.rec + ((size_t)(slot0 + nch - 1) * H + h) * R.size, sRec2, R.m, bar);
  }
  for (int e = tid; e < dk * dvs; e += kBThreads) {
    const int c = e / dvs, j = e % dvs;
    sdS[e] = p.dS_T ? p.dS_T[sofs + (size_t)c * dv + j0 + j] : 0.f;
  }
  __syncthreads();
  for (long ci = nch - 1; ci >= 0; --ci) {
    const long cs = t0 + ci * kBC;
    const int nrows = (int)(t1 - cs < kBC ? t1 - cs : kBC);
    const size_t slot = (size_t)(slot0 + ci);
    const long it = nch - 1 - ci;   // iteration: buffer it & 1, its (it >> 1)-th use
    const int buf = (int)(it & 1);
    for (int e = tid; e < kBC * dvs; e += kBThreads) {
      const int r = e / dvs, j = e % dvs;
      sdO[e] = (r < nrows && dO) ? to_f32(dO[((size_t)(bofs + cs + r) * H + h) * dv + j0 + j]) : 0.f;
    }
    float *dst = p.dS_out + (slot * H + h) * dk * dv;
    for (int e = tid; e < dk * dvs; e += kBThreads) {
      const int c = e / dvs, j = e % dvs;
      dst[(size_t)c * dv + j0 + j] = sdS[e];
    }
    if (!wait_record(p, bar + buf, (uint32_t)((it >> 1) & 1))) return;
    if (tid == 0 && ci > 0)
      issue_record(p.rec + ((slot - 1) * H + h) * R.size, sRec2 + (buf ^ 1) * R.m, R.m,
                   bar + (buf ^ 1));
    const float *sRec = sRec2 + buf * R.m;
    const float *sKr = sRec + R.kr, *sKd = sRec + R.kd, *sLi = sRec + R.li,
                *sBeta = sRec + R.beta, *sG = sRec + R.g, *sQr = sRec + R.qr, *sP = sRec + R.pp;
    // dU = Kd dS' + P^T dO
    for (int ti = tid; ti < (kBC / 2) * (dvs / 2); ti += kBThreads) {
      const int r0 = 2 * (ti / (dvs / 2)), jj = 2 * (ti % (dvs / 2));
      float a00 = 0.f, a01 = 0.f, a10 = 0.f, a11 = 0.f;
      const float *k0 = sKd + r0 * dk, *k1 = k0 + dk;
      for (int c = 0; c < dk; c += 4) {
        const float4 x0 = *reinterpret_cast<const float4 *>(k0 + c);
        const float4 x1 = *reinterpret_cast<const float4 *>(k1 + c);
        const float xa[4] = {x0.x, x0.y, x0.z, x0.w}, xb[4] = {x1.x, x1.y, x1.z, x1.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 sv = *reinterpret_cast<const float2 *>(sdS + (c + i) * dvs + jj);
          a00 = fmaf(xa[i], sv.x, a00);
          a01 = fmaf(xa[i], sv.y, a01);
          a10 = fmaf(xb[i], sv.x, a10);
          a11 = fmaf(xb[i], sv.y, a11);
        }
      }
      for (int t = r0; t < kBC; ++t) {   // P lower triangular: P[t][r0 + 1] = 0 at t = r0
        const float2 pt = *reinterpret_cast<const float2 *>(sP + t * kBC + r0);
        const float2 o = *reinterpret_cast<const float2 *>(sdO + t * dvs + jj);
        a00 = fmaf(pt.x, o.x, a00);
        a01 = fmaf(pt.x, o.y, a01);
        a10 = fmaf(pt.y, o.x, a10);
        a11 = fmaf(pt.y, o.y, a11);
      }
      *reinterpret_cast<float2 *>(sdU + r0 * dvs + jj) = make_float2(a00, a01);
      *reinterpret_cast<float2 *>(sdU + (r0 + 1) * dvs + jj) = make_float2(a10, a11);
    }
    __syncthreads();
    // dV' = Diag(beta) Li^T dU
    for (int ti = tid; ti < (kBC / 2) * (dvs / 2); ti += kBThreads) {
      const int r0 = 2 * (ti / (dvs / 2)), jj = 2 * (ti % (dvs / 2));
      float a00 = 0.f, a01 = 0.f, a10 = 0.f, a11 = 0.f;
      for (int t = r0; t < kBC; ++t) {   // Li[r0][r0 + 1] = 0
        const float2 lt = *reinterpret_cast<const float2 *>(sLi + t * kBC + r0);
        const float2 du = *reinterpret_cast<const float2 *>(sdU + t * dvs + jj);
        a00 = fmaf(lt.x, du.x, a00);
        a01 = fmaf(lt.x, du.y, a01);
        a10 = fmaf(lt.y, du.x, a10);
        a11 = fmaf(lt.y, du.y, a11);
      }
      const float b0 = sBeta[r0], b1 = sBeta[r0 + 1];
      *reinterpret_cast<float2 *>(sdV + r0 * dvs + jj) = make_float2(b0 * a00, b0 * a01);
      *reinterpret_cast<float2 *>(sdV + (r0 + 1) * dvs + jj) = make_float2(b1 * a10, b1 * a11);
    }
    __syncthreads();
    // dS = Diag(g) dS' + Qr^T dO - Kr^T dV'
    for (int ti = tid; ti < (dk / 4) * (dvs / 4); ti += kBThreads) {
      const int c0 = 4 * (ti / (dvs / 4)), jj = 4 * (ti % (dvs / 4));
      float acc[4][4];
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const float4 sv = *reinterpret_cast<const float4 *>(sdS + (c0 + x) * dvs + jj);
        const float gx = sG[c0 + x];
        acc[x][0] = gx * sv.x;
        acc[x][1] = gx * sv.y;
        acc[x][2] = gx * sv.z;
        acc[x][3] = gx * sv.w;
      }
      for (int r = 0; r < kBC; ++r) {
        const float4 qv = *reinterpret_cast<const float4 *>(sQr + r * dk + c0);
        const float4 kv = *reinterpret_cast<const float4 *>(sKr + r * dk + c0);
        const float4 o = *reinterpret_cast<const float4 *>(sdO + r * dvs + jj);
        const float4 w = *reinterpret_cast<const float4 *>(sdV + r * dvs + jj);
        const float qa[4] = {qv.x, qv.y, qv.z, qv.w}, ka[4] = {kv.x, kv.y, kv.z, kv.w};
        const float oa[4] = {o.x, o.y, o.z, o.w}, wa[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int y = 0; y < 4; ++y)
            acc[x][y] = fmaf(qa[x], oa[y], fmaf(-ka[x], wa[y], acc[x][y]));
      }
#pragma unroll
      for (int x = 0; x < 4; ++x)
        *reinterpret_cast<float4 *>(sdS + (c0 + x) * dvs + jj) =
            make_float4(acc[x][0], acc[x][1], acc[x][2], acc[x][3]);
    }
    __syncthreads();
  }
  if (p.gS0)
    for (int e = tid; e < dk * dvs; e += kBThreads) {
      const int c = e / dvs, j = e % dvs;
      p.gS0[sofs + (size_t)c * dv + j0 + j] = sdS[e];
    }
}

// ------------------------------------------------------------------ pass 4: gradients of a chunk
template <typename TIn, typename TG>
__global__ void __launch_bounds__(kGThreads, 1) bwd_grad_kernel(BwdParams p) {
  extern __shared__ float smem[];
  // rows of dk + 8 floats: 16-byte aligned, and the gate gradient's four threads per channel
  // read rows t = 4i + sub, which then fall on distinct banks for the eight channels of a warp
  const int dk = p.dk, dv = p.dv, ldk = dk + 8, ldz = dk + 4, H = p.H, tid = threadIdx.x;
  float *sQ = smem;                                   // [kBC][ldk] q
  float *sK = sQ + kBC * ldk;                         // [kBC][ldk] k
  float *sL = sK + kBC * ldk;                         // [kBC][ldk] gate prefix
  float *sKr = sL + kBC * ldk;                        // [kBC][ldk] K*G
  float *sKd = sKr + kBC * ldk;                       // [kBC][ldk] K*g(C-1,.)
  float *sdKr = sKd + kBC * ldk;                      // [kBC][ldk] accumulators
  float *sdQr = sdKr + kBC * ldk;
  float *sdKd = sdQr + kBC * ldk;
  uint8_t *sZ = reinterpret_cast<uint8_t *>(sdKd + kBC * ldk);
  // [kBC][kBP] arrays (rows padded to 33: threads that differ in the row hit distinct banks)
  float *sM = reinterpret_cast<float *>(sZ + kBC * ldz);
  float *sP = sM + kBC * kBP;
  float *sLi = sP + kBC * kBP;
  float *sdP = sLi + kBC * kBP;
  float *sdT = sdP + kBC * kBP;                        // dT, then dLi, then X, then dA
  float *sX = sdT + kBC * kBP;                         // scratch
  float *sS = sX + kBC * kBP;                          // [dk][kJP] slice of S
  float *sdS = sS + dk * kJP;                          // [dk][kJP] slice of dS'
  float *sVp = sdS + dk * kJP;                         // [kBC][kJP] V, then V'
  float *sU = sVp + kBC * kJP;
  float *sdO = sU + kBC * kJP;
  float *sdU = sdO + kBC * kJP;
  float *sdV = sdU + kBC * kJP;
  float *sBeta = sdV + kBC * kJP;
  float *sdBeta = sBeta + kBC;
  float *sGC = sdBeta + kBC;
  float *sLC = sGC + dk;
  float *sCarry = sLC + dk;                            // sum_j dS'_cj S_cj
  float *sInvQ = sCarry + dk;                          // [kBC] 1 / ||q_r|| (CKDA_QK_L2NORM)
  float *sInvK = sInvQ + kBC;                          // [kBC] 1 / ||k_r||
  float *sDaRow = sInvK + kBC;                         // [kBC] per-head gate gradient
  int *sZC = reinterpret_cast<int *>(sDaRow + kBC);

  const long slot = blockIdx.x;
  const int h = blockIdx.y;
  int n;
  long t0, t1, bofs, ci;
  if (!slot_chunk(p, slot, n, t0, t1, bofs, ci)) return;
  const long cs = t0 + ci * kBC;
  const int nrows = (int)(t1 - cs < kBC ? t1 - cs : kBC);
  const long row0 = bofs + cs;
  const TIn *v = static_cast<const TIn *>(p.v);
  const TIn *a = static_cast<const TIn *>(p.a);
  const TG *dO = static_cast<const TG *>(p.dO);
  const float *S_in = p.S_in + ((size_t)slot * H + h) * dk * dv;
  const float *dSo = p.dS_out + ((size_t)slot * H + h) * dk * dv;

  const bool per_head = per_head_gate(p.signed_gate), l2 = qk_l2norm(p.signed_gate);
  load_chunk<TIn>(p, row0, nrows, h, ldk, sQ, sK, sL, sZ, sBeta, sGC, sLC, sZC, sInvQ, sInvK);
  for (int r = tid; r < kBC; r += kGThreads) sDaRow[r] = 0.f;
  // M, P, Li, Kr and Kd from the chunk's record
  const RecLayout R = rec_layout(dk);
  const float *rec = p.rec + ((size_t)slot * H + h) * R.size;
  for (int e = tid; e < kBC * kBC; e += kGThreads) {
    const int q = (e / kBC) * kBP + e % kBC;
    sM[q] = rec[R.m + e];
    sP[q] = rec[R.pp + e];
    sLi[q] = rec[R.li + e];
  }
  for (int e = tid; e < kBC * dk; e += kGThreads) {
    const int r = e / dk, c = e % dk;
    sKr[r * ldk + c] = rec[R.kr + e];
    sKd[r * ldk + c] = rec[R.kd + e];
    sdKr[r * ldk + c] = 0.f;
    sdQr[r * ldk + c] = 0.f;
    sdKd[r * ldk + c] = 0.f;
  }
  for (int e = tid; e < kBC * kBP; e += kGThreads) {
    sdP[e] = 0.f;
    sdT[e] = 0.f;
  }
  for (int c = tid; c < dk; c += kGThreads) sCarry[c] = 0.f;
  __syncthreads();

  // ---- value-column slices: V', U, dU, dV' (-> dv) and the sums over value columns
  for (int j0 = 0; j0 < dv; j0 += kJS) {
    const int js = min(kJS, dv - j0);
    for (int e = tid; e < dk * js; e += kGThreads) {
      const int c = e / js, j = e % js;
      sS[c * kJP + j] = S_in[(size_t)c * dv + j0 + j];
      sdS[c * kJP + j] = dSo[(size_t)c * dv + j0 + j];
    }
    for (int e = tid; e < kBC * js; e += kGThreads) {
      const int r = e / js, j = e % js;
      const size_t idx = ((size_t)(row0 + r) * H + h) * dv + j0 + j;
      sVp[r * kJP + j] = r < nrows ? to_f32(v[idx]) : 0.f;
      sdO[r * kJP + j] = (r < nrows && dO) ? to_f32(dO[idx]) : 0.f;
    }
    __syncthreads();
    // Products over one slice, two rows (r0, r0 + 1) and one column j per thread.
    // V' = V - Kr S
    for (int ti = tid; ti < (kBC / 2) * js; ti += kGThreads) {
      const int r0 = 2 * (ti / js), j = ti % js;
      float a0 = sVp[r0 * kJP + j], a1 = sVp[(r0 + 1) * kJP + j];
      const float *k0 = sKr + r0 * ldk, *k1 = k0 + ldk;   // rows 16-byte aligned (ldk % 4 == 0)
      for (int c = 0; c < dk; c += 4) {
        const float4 x0 = *reinterpret_cast<const float4 *>(k0 + c);
        const float4 x1 = *reinterpret_cast<const float4 *>(k1 + c);
        const float xa[4] = {x0.x, x0.y, x0.z, x0.w}, xb[4] = {x1.x, x1.y, x1.z, x1.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float sv = sS[(c + i) * kJP + j];
          a0 = fmaf(-xa[i], sv, a0);
          a1 = fmaf(-xb[i], sv, a1);
        }
      }
      sVp[r0 * kJP + j] = a0;
      sVp[(r0 + 1) * kJP + j] = a1;
    }
    __syncthreads();
    // U = Li Diag(beta) V';  dU = Kd dS' + P^T dO
    for (int ti = tid; ti < (kBC / 2) * js; ti += kGThreads) {
      const int r0 = 2 * (ti / js), j = ti % js;
      float u0 = 0.f, u1 = 0.f;
      for (int m = 0; m <= r0 + 1; ++m) {   // Li[r0][r0 + 1] = 0
        const float vm = sBeta[m] * sVp[m * kJP + j];
        u0 = fmaf(sLi[r0 * kBP + m], vm, u0);
        u1 = fmaf(sLi[(r0 + 1) * kBP + m], vm, u1);
      }
      sU[r0 * kJP + j] = u0;
      sU[(r0 + 1) * kJP + j] = u1;
      float d0 = 0.f, d1 = 0.f;
      const float *k0 = sKd + r0 * ldk, *k1 = k0 + ldk;
      for (int c = 0; c < dk; c += 4) {
        const float4 x0 = *reinterpret_cast<const float4 *>(k0 + c);
        const float4 x1 = *reinterpret_cast<const float4 *>(k1 + c);
        const float xa[4] = {x0.x, x0.y, x0.z, x0.w}, xb[4] = {x1.x, x1.y, x1.z, x1.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float sv = sdS[(c + i) * kJP + j];
          d0 = fmaf(xa[i], sv, d0);
          d1 = fmaf(xb[i], sv, d1);
        }
      }
      for (int t = r0; t < kBC; ++t) {   // P[r0][r0 + 1] = 0
        const float o = sdO[t * kJP + j];
        d0 = fmaf(sP[t * kBP + r0], o, d0);
        d1 = fmaf(sP[t * kBP + r0 + 1], o, d1);
      }
      sdU[r0 * kJP + j] = d0;
      sdU[(r0 + 1) * kJP + j] = d1;
    }
    __syncthreads();
    // dV' = T^T dU = Diag(beta) Li^T dU  (the gradient of v)
    for (int ti = tid; ti < (kBC / 2) * js; ti += kGThreads) {
      const int r0 = 2 * (ti / js), j = ti % js;
      float a0 = 0.f, a1 = 0.f;
      for (int t = r0; t < kBC; ++t) {
        const float du = sdU[t * kJP + j];
        a0 = fmaf(sLi[t * kBP + r0], du, a0);
        a1 = fmaf(sLi[t * kBP + r0 + 1], du, a1);
      }
      a0 *= sBeta[r0];
      a1 *= sBeta[r0 + 1];
      sdV[r0 * kJP + j] = a0;
      sdV[(r0 + 1) * kJP + j] = a1;
      if (r0 < nrows) p.gv[((size_t)(row0 + r0) * H + h) * dv + j0 + j] = a0;
      if (r0 + 1 < nrows) p.gv[((size_t)(row0 + r0 + 1) * H + h) * dv + j0 + j] = a1;
    }
    __syncthreads();
    // sums over this slice's value columns: rows r0, r0 + 1 and the key channels
    // cl, cl + 32, cl + 64, cl + 96 per thread, four columns per step (16-byte loads)
    for (int ti = tid; ti < (kBC / 2) * 32; ti += kGThreads) {
      const int r0 = 2 * (ti >> 5), cl = ti & 31;
      float akd[2][4], aqr[2][4], akr[2][4];
#pragma unroll
      for (int y = 0; y < 2; ++y)
#pragma unroll
        for (int x = 0; x < 4; ++x) akd[y][x] = aqr[y][x] = akr[y][x] = 0.f;
      for (int j = 0; j < js; j += 4) {
        const float4 u0 = *reinterpret_cast<const float4 *>(sU + r0 * kJP + j);
        const float4 u1 = *reinterpret_cast<const float4 *>(sU + (r0 + 1) * kJP + j);
        const float4 o0 = *reinterpret_cast<const float4 *>(sdO + r0 * kJP + j);
        const float4 o1 = *reinterpret_cast<const float4 *>(sdO + (r0 + 1) * kJP + j);
        const float4 w0 = *reinterpret_cast<const float4 *>(sdV + r0 * kJP + j);
        const float4 w1 = *reinterpret_cast<const float4 *>(sdV + (r0 + 1) * kJP + j);
        const float ua[2][4] = {{u0.x, u0.y, u0.z, u0.w}, {u1.x, u1.y, u1.z, u1.w}};
        const float oa[2][4] = {{o0.x, o0.y, o0.z, o0.w}, {o1.x, o1.y, o1.z, o1.w}};
        const float wa[2][4] = {{w0.x, w0.y, w0.z, w0.w}, {w1.x, w1.y, w1.z, w1.w}};
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int c = cl + 32 * x;
          if (c < dk) {
            const float4 sv = *reinterpret_cast<const float4 *>(sS + c * kJP + j);
            const float4 dv4 = *reinterpret_cast<const float4 *>(sdS + c * kJP + j);
            const float sa[4] = {sv.x, sv.y, sv.z, sv.w}, da[4] = {dv4.x, dv4.y, dv4.z, dv4.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
              for (int y = 0; y < 2; ++y) {
                akd[y][x] = fmaf(ua[y][i], da[i], akd[y][x]);
                aqr[y][x] = fmaf(oa[y][i], sa[i], aqr[y][x]);
                akr[y][x] = fmaf(-wa[y][i], sa[i], akr[y][x]);
              }
          }
        }
      }
#pragma unroll
      for (int y = 0; y < 2; ++y)
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int c = cl + 32 * x;
          if (c < dk) {
            sdKd[(r0 + y) * ldk + c] += akd[y][x];
            sdQr[(r0 + y) * ldk + c] += aqr[y][x];
            sdKr[(r0 + y) * ldk + c] += akr[y][x];
          }
        }
    }
    for (int e = tid; e < kBC * kBC; e += kGThreads) {
      const int r = e / kBC, m = e % kBC;
      if (m > r) continue;
      float adp = 0.f, adt = 0.f;
      for (int j = 0; j < js; j += 4) {
        const float4 o = *reinterpret_cast<const float4 *>(sdO + r * kJP + j);
        const float4 u = *reinterpret_cast<const float4 *>(sU + m * kJP + j);
        const float4 du = *reinterpret_cast<const float4 *>(sdU + r * kJP + j);
        const float4 vp = *reinterpret_cast<const float4 *>(sVp + m * kJP + j);
        adp = fmaf(o.x, u.x, fmaf(o.y, u.y, fmaf(o.z, u.z, fmaf(o.w, u.w, adp))));
        adt = fmaf(du.x, vp.x, fmaf(du.y, vp.y, fmaf(du.z, vp.z, fmaf(du.w, vp.w, adt))));
      }
      sdP[r * kBP + m] += adp;
      sdT[r * kBP + m] += adt;
    }
    for (int c = tid; c < dk; c += kGThreads) {
      float acc = 0.f;
      for (int j = 0; j < js; j += 4) {
        const float4 a4 = *reinterpret_cast<const float4 *>(sdS + c * kJP + j);
        const float4 b4 = *reinterpret_cast<const float4 *>(sS + c * kJP + j);
        acc = fmaf(a4.x, b4.x, fmaf(a4.y, b4.y, fmaf(a4.z, b4.z, fmaf(a4.w, b4.w, acc))));
      }
      sCarry[c] += acc;
    }
    __syncthreads();
  }

  // ---- through T = Li Diag(beta) and Li = (I + A)^{-1}
  // dbeta_m = sum_r Li_rm dT_rm;  dLi = dT Diag(beta) (in place)
  for (int m = tid; m < kBC; m += kGThreads) {
    float acc = 0.f;
    for (int r = m; r < kBC; ++r) acc = fmaf(sLi[r * kBP + m], sdT[r * kBP + m], acc);
    sdBeta[m] = acc;
  }
  __syncthreads();
  for (int e = tid; e < kBC * kBC; e += kGThreads) sdT[(e / kBC) * kBP + e % kBC] *= sBeta[e % kBC];
  __syncthreads();
  // X = dLi Li^T
  for (int e = tid; e < kBC * kBC; e += kGThreads) {
    const int r = e / kBC, m = e % kBC;
    float acc = 0.f;
    for (int j = 0; j < kBC; ++j) acc = fmaf(sdT[r * kBP + j], sLi[m * kBP + j], acc);
    sX[r * kBP + m] = acc;
  }
  __syncthreads();
  // dA = -Li^T X, strictly lower (over dT); dbeta_r += sum_j dA_rj M_rj; dM = beta_r dA (over dT)
  for (int e = tid; e < kBC * kBC; e += kGThreads) {
    const int r = e / kBC, j = e % kBC;
    float acc = 0.f;
    if (j < r)
      for (int t = 0; t < kBC; ++t) acc = fmaf(sLi[t * kBP + r], sX[t * kBP + j], acc);
    sdT[r * kBP + j] = -acc;
  }
  __syncthreads();
  for (int r = tid; r < kBC; r += kGThreads) {
    float acc = 0.f;
    for (int j = 0; j < r; ++j) acc = fmaf(sdT[r * kBP + j], sM[r * kBP + j], acc);
    sdBeta[r] += acc;
  }
  __syncthreads();
  for (int e = tid; e < kBC * kBC; e += kGThreads) sdT[(e / kBC) * kBP + e % kBC] *= sBeta[e / kBC];   // dM
  __syncthreads();
  const float *sdM = sdT;

  // ---- dq, dk of the rows.  The pair factors g(r, j) run as products of the single gates
  // (g(r, j) = g(r, j+1) alpha_{j+1} walking j down from r, g(t, r) = g(t-1, r) alpha_t walking t
  // up), exact to a few ulp; a zero gate makes every factor across it zero, as it should.
  float *sAl = sS;   // [kBC][ldk] the gates (the slice buffers are dead)
  for (int e = tid; e < kBC * dk; e += kGThreads) {
    const int r = e / dk, c = e % dk;
    sAl[r * ldk + c] = r > 0 ? pair_gate(sL, sZ, ldk, ldz, r, r - 1, c)
                             : prefix_gate(sL, sZ, ldk, ldz, 0, c);
  }
  __syncthreads();
  for (int e = tid; e < kBC * dk; e += kGThreads) {
    const int r = e / dk, c = e % dk;
    if (r >= nrows) continue;
    const float G = prefix_gate(sL, sZ, ldk, ldz, r, c);
    const float gd = suffix_gate(sL, sZ, sLC, sZC, ldk, ldz, r, c);
    float dqv = sdQr[r * ldk + c] * G;
    float dkv = sdKr[r * ldk + c] * G + sdKd[r * ldk + c] * gd;
    dqv = fmaf(sdP[r * kBP + r], sK[r * ldk + c], dqv);   // j = r: factor 1
    float f = 1.f;
    for (int j = r - 1; j >= 0; --j) {
      f *= sAl[(j + 1) * ldk + c];
      const float kj = sK[j * ldk + c] * f;
      dqv = fmaf(sdP[r * kBP + j], kj, dqv);
      dkv = fmaf(sdM[r * kBP + j], kj, dkv);
    }
    dkv = fmaf(sdP[r * kBP + r], sQ[r * ldk + c], dkv);   // t = r: factor 1
    f = 1.f;
    for (int t = r + 1; t < kBC; ++t) {
      f *= sAl[t * ldk + c];
      const float w = fmaf(sdM[t * kBP + r], sK[t * ldk + c], sdP[t * kBP + r] * sQ[t * ldk + c]);
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
    for (int r = warp; r < nrows; r += kGThreads / 32) {
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

  // ---- gate gradient, four threads per channel (lanes 4c' .. 4c' + 3 of a warp; thread sub
  // owns the rows t = sub, sub + 4, ... of the inner sums).  dL/dalpha_s is the derivative of the gate
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
  static_assert(kGThreads >= 4 * 128, "four threads per key channel");
  if ((tid >> 2) < dk) {   // whole warps (dk is a multiple of 16)
    const int c = tid >> 2, sub = tid & 3;
    float RS[kBC];
    float run = 0.f;
#pragma unroll
    for (int t = kBC - 1; t >= 0; --t) {
      const float x = sdKr[t * ldk + c] * sK[t * ldk + c] + sdQr[t * ldk + c] * sQ[t * ldk + c];
      const float al_next = t + 1 < kBC ? sAl[(t + 1) * ldk + c] : 0.f;
      run = fmaf(al_next, run, x);
      RS[t] = run;
    }
    float inner[kBC / 4];   // inner_t for t = 4i + sub
#pragma unroll
    for (int i = 0; i < kBC / 4; ++i) inner[i] = 0.f;
    float WS = 0.f;
    const float carry = sCarry[c];
#pragma unroll
    for (int s = 0; s < kBC; ++s) {
      // sum over this thread's t >= s of g(t, s) inner_t, g(t, s) walked up from g(s, s) = 1
      float pairs = (s & 3) == sub ? inner[s >> 2] : 0.f;
      float f = 1.f;
#pragma unroll
      for (int t = s + 1; t < kBC; ++t) {
        f *= sAl[t * ldk + c];
        if ((t & 3) == sub) pairs = fmaf(f, inner[t >> 2], pairs);
      }
      pairs += __shfl_xor_sync(0xffffffffu, pairs, 1);
      pairs += __shfl_xor_sync(0xffffffffu, pairs, 2);
      if (s < nrows && sub == 0) {
        const float Gp = s > 0 ? prefix_gate(sL, sZ, ldk, ldz, s - 1, c) : 1.f;
        const float gd = suffix_gate(sL, sZ, sLC, sZC, ldk, ldz, s, c);
        const float dalpha = fmaf(Gp, RS[s], fmaf(gd, WS, fmaf(Gp * gd, carry, pairs)));
        if (per_head) {
          atomicAdd(&sDaRow[s], dalpha);   // one gate shared by every key channel
        } else {
          const size_t idx = ((size_t)(row0 + s) * H + h) * dk + c;
          p.ga[idx] = dalpha * dalpha_da(to_f32(a[idx]), p.signed_gate);
        }
      }
      // advance WS and inner_t past row s
      const float al = sAl[s * ldk + c];
      const float z = sdKd[s * ldk + c] * sK[s * ldk + c];
      WS = fmaf(al, WS, z);
      const float ks = sK[s * ldk + c];
#pragma unroll
      for (int i = 0; i < kBC / 4; ++i) {
        const int t = 4 * i + sub;
        if (t > s) {
          const float cts = (sdM[t * kBP + s] * sK[t * ldk + c] + sdP[t * kBP + s] * sQ[t * ldk + c]) * ks;
          inner[i] = fmaf(al, inner[i], cts);
        }
      }
    }
  }
  __syncthreads();
  for (int r = tid; r < nrows; r += kGThreads) {
    const size_t row = (size_t)(row0 + r) * H + h;
    p.gb[row] = sdBeta[r] * dbeta_db(p.b[row], p.signed_gate);
    if (per_head) p.ga[row] = sDaRow[r] * dalpha_da(to_f32(a[row]), p.signed_gate);
  }
}

size_t prep_smem(int dk) {
  const int ldk = dk + 1, ldz = dk + 4;
  return sizeof(float) * ((size_t)3 * kBC * ldk + 3 * kBC * kBC + 3 * kBC + 2 * dk) +
         (size_t)kBC * ldz + sizeof(int) * dk + 64;
}
size_t state_fwd_smem(int dk, int dvs) {
  return sizeof(float) * (2 * (size_t)rec_layout(dk).qr + (size_t)dk * dvs + 2 * kBC * dvs) + 16;
}
size_t state_rev_smem(int dk, int dvs) {
  return sizeof(float) * (2 * (size_t)rec_layout(dk).m + (size_t)dk * dvs + 3 * kBC * dvs) + 16;
}
size_t grad_smem(int dk) {
  const int ldk = dk + 8, ldz = dk + 4;
  return sizeof(float) * ((size_t)8 * kBC * ldk + 6 * kBC * kBP + 2 * dk * kJP + 5 * kBC * kJP +
                          2 * kBC + 3 * dk + 3 * kBC) +
         (size_t)kBC * ldz + sizeof(int) * dk + 64;
}

template <typename K>
bool allow_smem(K kern, size_t bytes) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) ==
         cudaSuccess;
}

template <typename TIn, typename TG>
int launch_typed(const BwdArgs &g, cudaStream_t stream) {
  BwdParams p;
  p.q = g.q; p.k = g.k; p.v = g.v; p.a = g.a; p.dO = g.dO; p.b = g.b; p.S0 = g.S0;
  p.dS_T = g.dS_T; p.cu = g.cu_seqlens;
  p.gq = g.gq; p.gk = g.gk; p.gv = g.gv; p.ga = g.ga; p.gb = g.gb; p.gS0 = g.gS0;
  p.S_in = g.S_chunks; p.dS_out = g.dS_chunks; p.rec = g.rec; p.status = g.status;
  p.n_seqs = g.n_seqs; p.T = g.T; p.H = g.H; p.dk = g.dk; p.dv = g.dv;
  p.dvs = g.dv % 32 == 0 ? 32 : 16;   // dv is a multiple of 16
  p.signed_gate = g.signed_gate; p.n_slots = g.n_slots;
  const size_t s1 = prep_smem(g.dk), s2 = state_fwd_smem(g.dk, p.dvs),
               s3 = state_rev_smem(g.dk, p.dvs), s4 = grad_smem(g.dk);
  auto k1 = bwd_prep_kernel<TIn>;
  auto k2 = bwd_state_fwd_kernel<TIn>;
  auto k3 = bwd_state_rev_kernel<TIn, TG>;
  auto k4 = bwd_grad_kernel<TIn, TG>;
  if (!allow_smem(k1, s1) || !allow_smem(k2, s2) || !allow_smem(k3, s3) || !allow_smem(k4, s4))
    return CKDA_ERR_CUDA;
  const dim3 chunks((unsigned)g.n_slots, (unsigned)g.H);
  const dim3 walks((unsigned)(g.n_seqs * g.H), (unsigned)(g.dv / p.dvs));
  if (g.n_slots > 0) k1<<<chunks, kGThreads, s1, stream>>>(p);
  k2<<<walks, kBThreads, s2, stream>>>(p);
  k3<<<walks, kBThreads, s3, stream>>>(p);
  if (g.n_slots > 0) k4<<<chunks, kGThreads, s4, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? CKDA_OK : CKDA_ERR_CUDA;
}

}  // namespace

int bwd_chunk_rows() { return kBC; }

int launch_chunk_bwd(const BwdArgs &g, cudaStream_t s) {
  if (g.n_seqs * g.H == 0) return CKDA_OK;
  const bool in_bf = g.io_dtype == CKDA_BF16, do_bf = g.do_dtype == CKDA_BF16;
  if (in_bf && do_bf) return launch_typed<__nv_bfloat16, __nv_bfloat16>(g, s);
  if (in_bf) return launch_typed<__nv_bfloat16, float>(g, s);
  if (do_bf) return launch_typed<float, __nv_bfloat16>(g, s);
  return launch_typed<float, float>(g, s);
}

}  // namespace ckda

// chunk_tc.cu -- tensor-core chunkwise (WY / UT-transform) forward for
// dk = dv = 128, chunk 64, bf16 q/k/v/a, on sm_100a (tcgen05 + TMEM + TMA).
//
// Chunk algebra (the CKDA review: the DPR1 transition keeps WY chunk-wise
// parallelism, section "Diagonal-plus-rank-one (DPR1) transition").  For a
// chunk with incoming state S (dk x dv), rows t = 0..63, per-channel
// cumulative gate product G_t = prod_{s<=t} alpha_s (signed), and
//   Kr = K * G,  Qr = Q * G,  Kc = K / G    (row-wise, per channel)
//   A  = tril(Diag(beta) Kr Kc^T, -1)       P = tril(Qr Kc^T)
//   Tm = (I + A)^{-1} Diag(beta)
//   W  = Tm Kr,   U = Tm V - W S
//   O  = Qr S + P U
//   S' = Diag(G_63) (S + Kc^T U)
// Everything is computed transposed so that every product has M = 128 on the
// tensor core: the state lives in TMEM as S^T (lane = value channel j,
// column = key channel i) and is the A operand of the state products.
//   (1) [A;P]   = [Kr;Qr] Kc^T          M=128 (64 Kr rows + 64 Qr rows), N=64, K=128
//   (2) W^T     = Kr^T Tm^T              A = Kr^T in TMEM (lane = key channel), K=64
//   (3) U^T     = V^T Tm^T               A = V^T in TMEM (lane = value channel), K=64
//   (4) U^T    -= S^T W^T                A = S^T in TMEM, K=128
//   (5) O^T     = S^T Qr^T + U^T P^T     A from TMEM
//   (6) S^T    += U^T Kc,  then columns scaled by G_63 (threads, in TMEM)
// All MMAs are kind::tf32 with fp32 accumulation and K-major operands; smem
// operands and the TMEM copies of Kr^T are rounded to tf32 (round-to-nearest)
// when written; the state and U are read from TMEM directly.  The gate products are the signed cumulative products in
// fp32 (the sign bit carries the gate-sign parity).  A chunk whose product
// falls outside [2^-100, 2^100] in some channel (an exact zero gate, or
// extreme decay) cannot use the factorisation Kr Kc^T; it is run token by
// token, exactly, on the same TMEM-resident state (slow path).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace ckda {
namespace {

using namespace sm100;

constexpr int kC = 64;      // chunk rows
constexpr int kD = 128;     // dk = dv
constexpr int kThreads = 256;

// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_KQ = 0;          // [Kr;Qr] 128 rows x 128 fp32, 4 column blocks of 16 KB;
                                        // rows 0..63 hold W once (1) has consumed Kr
constexpr uint32_t OFF_KC = 65536;      // Kc 64 rows x 128 fp32, 4 column blocks of 8 KB;
                                        // then the solve's A and X (plain 64 x 64 fp32 each)
constexpr uint32_t OFF_KCT = 98304;     // Kc^T 128 rows x 64 fp32, 2 column blocks of 16 KB
constexpr uint32_t OFF_T = 131072;      // Tm 64 x 64 fp32, 2 column blocks of 8 KB (the solve's
                                        // block scratch before that); T and P together
constexpr uint32_t OFF_P = 147456;      // P  64 x 64 fp32 (2 blocks); T+P stage O for its TMA store
constexpr uint32_t OFF_STG = 163840;    // TMA staging: q, k, v, a bf16 64 x 128 (16 KB each)
constexpr uint32_t OFF_MISC = 229376;   // beta[64], gC[128], xch[128], barriers, tmem slot
constexpr uint32_t kSmemUsed = OFF_MISC + 2048;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;  // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory budget");

// TMEM columns (all 512 allocated)
constexpr uint32_t COL_S = 0, COL_AP = 128, COL_W = 192, COL_U = 256, COL_O = 320, COL_KRT = 384,
                   COL_VT = 448;

constexpr uint32_t IDESC_N64 = idesc_tf32(128, 64, false, false);        // (1), (2), (3), (5)
constexpr uint32_t IDESC_U = idesc_tf32(128, 64, false, false, true);    // (4), B negated
constexpr uint32_t IDESC_S = idesc_tf32(128, 128, false, false);         // (6)

constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s bound on any single wait

struct TcParams {
  const float *b;
  const float *S0;
  const int32_t *cu;
  void *o;
  float *S_T;
  int *status;
  int n_seqs, T, H, signed_gate;
};

// byte offset of fp32 element (r, c) in a 128-byte-swizzled tile of R rows
__device__ __forceinline__ uint32_t sw32(int R, int r, int c) {
  return (uint32_t)((c >> 5) * (R * 128) + r * 128 + ((((c & 31) >> 2) ^ (r & 7)) << 4) +
                    ((c & 3) << 2));
}
// byte offset of bf16 element (r, c) in a staged 64 x 128 tile (two TMA boxes of 64 columns)
__device__ __forceinline__ uint32_t swbf(int r, int c) {
  return (uint32_t)((c >> 6) * 8192 + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) +
                    ((c & 7) << 1));
}
__device__ __forceinline__ float ldbf(const uint8_t *tile, int r, int c) {
  return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(tile + swbf(r, c)));
}
__device__ __forceinline__ void st_tf32(uint8_t *tile, uint32_t off, float x) {
  *reinterpret_cast<uint32_t *>(tile + off) = to_tf32(x);
}

// Gates for the bf16 path, from their definitions with fast exponentials
// (relative error ~1e-6, far inside the bf16-input tolerance):
//   sigma(a) = 1 / (1 + e^{-a});  2 sigma(a) - 1 = tanh(a/2) = (1 - e^{-|a|}) / (1 + e^{-|a|})
// with the odd Taylor series tanh(y) = y - y^3/3 + 2 y^5/15 for |a| < 0.1
// (truncation below 2e-10 relative there), so small gates keep full precision.
template <int SG>
__device__ __forceinline__ float fast_alpha(float a) {
  if (SG == 0) return __fdividef(1.f, 1.f + __expf(-a));
  if (SG == 1) {
    const float x = fabsf(a);
    float t;
    if (x < 0.1f) {
      const float y = 0.5f * x, y2 = y * y;
      t = y * fmaf(y2, fmaf(y2, 2.f / 15.f, -1.f / 3.f), 1.f);
    } else {
      const float e = __expf(-x);
      t = __fdividef(1.f - e, 1.f + e);
    }
    return copysignf(t, a);
  }
  return a;
}
template <int SG>
__device__ __forceinline__ float fast_beta(float b) {
  if (SG == 0) return __fdividef(1.f, 1.f + __expf(-b));
  if (SG == 1) return __fdividef(2.f, 1.f + __expf(-b));
  return b;
}

// plain 64 x 64 fp32 scratch, columns XOR-swizzled by row so that a warp
// touching one column of 32 consecutive rows hits 32 banks
__device__ __forceinline__ int pidx(int r, int c) { return r * 64 + (c ^ (r & 31)); }

// X = (I + A)^{-1} for a 64 x 64 strictly lower A (plain, pidx layout):
// 16 x 16 diagonal blocks by forward substitution (one warp each), then the
// block rows in order, X_ij = -X_ii sum_{k=j}^{i-1} A_ik X_kj, with four
// partial sums per dot product.
__device__ void unit_lower_inverse(const float *A, float *X, float *Y, int tid) {
  const int warp = tid >> 5, lane = tid & 31;
  if (warp < 4 && lane < 16) {
    const int o = 16 * warp, m = lane;
    float x[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      float a0 = 0.f, a1 = 0.f;
#pragma unroll
      for (int l = 0; l < r; ++l) {
        if (l & 1) a1 = fmaf(-A[pidx(o + r, o + l)], x[l], a1);
        else a0 = fmaf(-A[pidx(o + r, o + l)], x[l], a0);
      }
      x[r] = (r == m) ? 1.f : a0 + a1;
    }
#pragma unroll
    for (int r = 0; r < 16; ++r) X[pidx(o + r, o + m)] = x[r];
  }
  __syncthreads();
  const int r = tid >> 4, m = tid & 15;
#pragma unroll
  for (int i = 1; i < 4; ++i) {
    // Y_j = sum_{k=j}^{i-1} A_ik X_kj for every block j < i
#pragma unroll
    for (int j = 0; j < i; ++j) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int k = j; k < i; ++k) {
#pragma unroll
        for (int l = 0; l < 16; ++l)
          acc[l & 3] = fmaf(A[pidx(16 * i + r, 16 * k + l)], X[pidx(16 * k + l, 16 * j + m)], acc[l & 3]);
      }
      Y[(j * 16 + r) * 17 + m] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
    }
    __syncthreads();
    // X_ij = -X_ii Y_j
#pragma unroll
    for (int j = 0; j < i; ++j) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int l = 0; l < 16; ++l)
        acc[l & 3] = fmaf(-X[pidx(16 * i + r, 16 * i + l)], Y[(j * 16 + l) * 17 + m], acc[l & 3]);
      X[pidx(16 * i + r, 16 * j + m)] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
    }
    __syncthreads();
  }
}

template <typename TOut, int SG>
__global__ void __launch_bounds__(kThreads, 1)
    chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_a,
                    const __grid_constant__ CUtensorMap tm_o, TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sKQ = sm + OFF_KQ, *sKC = sm + OFF_KC, *sKCT = sm + OFF_KCT, *sT = sm + OFF_T,
          *sP = sm + OFF_P, *sStg = sm + OFF_STG;
  float *sBeta = reinterpret_cast<float *>(sm + OFF_MISC);
  float *sGC = sBeta + 64;
  float *sXch = sGC + 128;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_MISC + 1280);
  uint64_t *tma_bar = bars, *mma_bar = bars + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_MISC + 1296);
  const uint32_t sbase = smem_u32(sm);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = p.H;
  const int unit = blockIdx.x, n = unit / H, h = unit % H;
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
  const size_t sofs = ((size_t)n * H + h) * kD * kD;
  TOut *o = static_cast<TOut *>(p.o);

  if (tid == 0) {
    mbar_init(tma_bar, 1);
    mbar_init(mma_bar, 1);
    mbar_fence_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int q4 = warp & 3, half = warp >> 2;
  const uint32_t lane_addr = tmem + ((uint32_t)(32 * q4) << 16);
  const int jrow = 32 * q4 + lane;  // TMEM lane owned by this thread

  uint32_t tma_phase = 0, mma_phase = 0;
  bool tma_pending = false, mma_pending = false, failed = false;

  // one warp polls an mbarrier phase; the block then agrees on the outcome
  auto block_wait = [&](uint64_t *bar, uint32_t parity) -> bool {
    bool ok = true;
    if (warp == 0) ok = mbar_wait(bar, parity, kWaitNs);
    return __syncthreads_and(ok) != 0;
  };
  auto issue_tma = [&](long cs) {
    mbar_arrive_expect_tx(tma_bar, 4 * 2 * 8192);
    const int row = (int)(bofs + cs);
    const CUtensorMap *maps[4] = {&tm_q, &tm_k, &tm_v, &tm_a};
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int bx = 0; bx < 2; ++bx)
        tma_load_3d(sStg + x * 16384 + bx * 8192, maps[x], tma_bar, bx * 64, h, row);
  };

  // ---- initial state into TMEM: thread (lane j, half) holds S^T[j][64*half .. +64) = S0[i][j]
  {
#pragma unroll
    for (int cb = 0; cb < 2; ++cb) {
      uint32_t r[32];
      const int i0 = 64 * half + 32 * cb;
#pragma unroll
      for (int x = 0; x < 32; ++x)
        r[x] = __float_as_uint(p.S0 ? p.S0[sofs + (size_t)(i0 + x) * kD + jrow] : 0.f);
      tmem_st32(lane_addr + COL_S + i0, r);
    }
    tmem_wait_st();
  }
  if (tid == 0 && t1 > t0) {
    issue_tma(t0);
  }
  tma_pending = t1 > t0;
  tc_fence_before();
  __syncthreads();

  const uint8_t *stq = sStg, *stk = sStg + 16384, *stv = sStg + 32768, *sta = sStg + 49152;
  // strengths are loaded one chunk ahead (threads 0..63, one row each)
  float b_next = 0.f;
  if (tid < kC && t0 + tid < t1) b_next = p.b[(size_t)(bofs + t0 + tid) * H + h];
  bool store_pending = false;

  for (long cs = t0; cs < t1; cs += kC) {
    const int nrows = (int)(t1 - cs < kC ? t1 - cs : kC);
    const bool has_next = cs + kC < t1;
    const float b_cur = b_next;
    if (tid < kC && cs + kC + tid < t1) b_next = p.b[(size_t)(bofs + cs + kC + tid) * H + h];
    // ---------------------------------------------------------------- A: gates and operands
    if (!block_wait(tma_bar, tma_phase)) { failed = true; break; }
    tma_phase ^= 1;
    tma_pending = false;
    const int c = tid & 127, hf = tid >> 7;
    float g[32];
    {
      float run = 1.f;
#pragma unroll
      for (int rr = 0; rr < 32; ++rr) {
        const int r = 32 * hf + rr;
        const float al = fast_alpha<SG>(ldbf(sta, r, c));
        run *= r < nrows ? al : 1.f;
        g[rr] = run;
      }
      if (hf == 0) sXch[c] = run;
    }
    if (tid < kC) sBeta[tid] = tid < nrows ? fast_beta<SG>(b_cur) : 0.f;
    __syncthreads();
    bool bad = false;
    {
      const float mult = hf ? sXch[c] : 1.f;
#pragma unroll
      for (int grp = 0; grp < 2; ++grp) {
        uint32_t krt[16], vt[16];
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          const int rr = 16 * grp + x, r = 32 * hf + rr;
          const float gam = g[rr] * mult;
          const float ag = fabsf(gam);
          bad |= !(ag >= 0x1p-100f && ag <= 0x1p100f);
          const float inv = __fdividef(1.f, gam);
          // rows past the sequence end hold another sequence's tokens or TMA fill: masked
          const bool valid = r < nrows;
          const float q_raw = ldbf(stq, r, c), k_raw = ldbf(stk, r, c), v_raw = ldbf(stv, r, c);
          const float qv = valid ? q_raw : 0.f, kv = valid ? k_raw : 0.f, vv = valid ? v_raw : 0.f;
          const uint32_t kr = to_tf32(kv * gam), kc = to_tf32(kv * inv);
          *reinterpret_cast<uint32_t *>(sKQ + sw32(128, r, c)) = kr;
          st_tf32(sKQ, sw32(128, 64 + r, c), qv * gam);
          *reinterpret_cast<uint32_t *>(sKC + sw32(64, r, c)) = kc;
          *reinterpret_cast<uint32_t *>(sKCT + sw32(128, c, r)) = kc;
          krt[x] = kr;
          vt[x] = __float_as_uint(vv);
          if (rr == 31 && hf == 1) sGC[c] = gam;
        }
        // lane c of TMEM holds Kr^T[c][.] and V^T[c][.] (A operands of (2) and (3))
        tmem_st16(lane_addr + COL_KRT + 32 * hf + 16 * grp, krt);
        tmem_st16(lane_addr + COL_VT + 32 * hf + 16 * grp, vt);
      }
      tmem_wait_st();
    }
    tc_fence_before();
    fence_proxy_async();
    const bool slow = __syncthreads_or(bad);

    if (slow) {
      // ------------------------------------------------------------ exact token-by-token path
      float *sAl = reinterpret_cast<float *>(sKQ);  // plain [64][128] gates
#pragma unroll 4
      for (int rr = 0; rr < 32; ++rr) {
        const int r = 32 * hf + rr;
        sAl[r * kD + c] = r < nrows ? gate_alpha(ldbf(sta, r, c), SG) : 1.f;
      }
      __syncthreads();
      {
        // thread (value channel jrow, key half): s[x] = S^T[jrow][64*half + x]
        float *sRed = sAl + kC * kD;  // [2][2][128] partial dot products
        float s[64];
#pragma unroll
        for (int cb = 0; cb < 2; ++cb) {
          uint32_t r[32];
          tmem_ld32(lane_addr + COL_S + 64 * half + 32 * cb, r);
          tmem_wait_ld();
#pragma unroll
          for (int x = 0; x < 32; ++x) s[32 * cb + x] = __uint_as_float(r[x]);
        }
        for (int t = 0; t < nrows; ++t) {
          float pk = 0.f;
#pragma unroll
          for (int x = 0; x < 64; ++x) {
            const int i = 64 * half + x;
            s[x] *= sAl[t * kD + i];
            pk = fmaf(ldbf(stk, t, i), s[x], pk);
          }
          sRed[half * 128 + jrow] = pk;
          __syncthreads();
          const float u = sBeta[t] * (ldbf(stv, t, jrow) - (sRed[jrow] + sRed[128 + jrow]));
          float acc = 0.f;
#pragma unroll
          for (int x = 0; x < 64; ++x) {
            const int i = 64 * half + x;
            s[x] = fmaf(ldbf(stk, t, i), u, s[x]);
            acc = fmaf(ldbf(stq, t, i), s[x], acc);
          }
          sRed[256 + half * 128 + jrow] = acc;
          __syncthreads();
          if (half == 0 && o)
            o[((size_t)(bofs + cs + t) * H + h) * kD + jrow] =
                from_f32<TOut>(sRed[256 + jrow] + sRed[384 + jrow]);
        }
#pragma unroll
        for (int cb = 0; cb < 2; ++cb) {
          uint32_t r[32];
#pragma unroll
          for (int x = 0; x < 32; ++x) r[x] = __float_as_uint(s[32 * cb + x]);
          tmem_st32(lane_addr + COL_S + 64 * half + 32 * cb, r);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      __syncthreads();
      if (tid == 0 && has_next) issue_tma(cs + kC);
      tma_pending = has_next;
      continue;
    }

    // ---------------------------------------------------------------- (1) [A;P] = [Kr;Qr] Kc^T
    if (tid == 0) {
      if (has_next) issue_tma(cs + kC);   // staging is free: prep has consumed it
      tc_fence_after();
#pragma unroll
      for (int s = 0; s < 16; ++s) {
        const uint64_t a = smem_desc_sw128(sbase + OFF_KQ + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024);
        const uint64_t b = smem_desc_sw128(sbase + OFF_KC + (s >> 2) * 8192 + (s & 3) * 32, 16, 1024);
        mma_ss(tmem + COL_AP, a, b, IDESC_N64, s > 0);
      }
      mma_commit(mma_bar);
      if (store_pending) bulk_wait_read();  // previous O tile (over T and P) has left smem
    }
    tma_pending = has_next;
    store_pending = false;
    mma_pending = true;
    if (!block_wait(mma_bar, mma_phase)) { failed = true; break; }
    mma_phase ^= 1;
    mma_pending = false;
    tc_fence_after();
    // ---------------------------------------------------------------- A and P out of TMEM
    float *sA = reinterpret_cast<float *>(sKC);           // plain [64][64], pidx layout
    float *sX = sA + 64 * 64;                              // plain [64][64], pidx layout
    float *sY = reinterpret_cast<float *>(sT);             // [3*16][17] block scratch
    {
      uint32_t r[32];
      tmem_ld32(lane_addr + COL_AP + 32 * half, r);
      tmem_wait_ld();
      if (jrow < 64) {
        const int t = jrow;
        const float bt = sBeta[t];
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          const int j = 32 * half + x;
          sA[pidx(t, j)] = j < t ? __uint_as_float(r[x]) * bt : 0.f;
        }
      } else {
        const int t = jrow - 64;
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          const int j = 32 * half + x;
          st_tf32(sP, sw32(64, t, j), j <= t ? __uint_as_float(r[x]) : 0.f);
        }
      }
    }
    __syncthreads();
    // ---------------------------------------------------------------- Tm = (I + A)^{-1} Diag(beta)
    unit_lower_inverse(sA, sX, sY, tid);
    for (int e = tid; e < kC * kC; e += kThreads) {
      const int t = e >> 6, s = e & 63;
      st_tf32(sT, sw32(64, t, s), s <= t ? sX[pidx(t, s)] * sBeta[s] : 0.f);
    }
    fence_proxy_async();
    __syncthreads();
    // ---------------------------------------------------------------- (2) W^T, (3) U^T
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const uint64_t bt = smem_desc_sw128(sbase + OFF_T + (s >> 2) * 8192 + (s & 3) * 32, 16, 1024);
        mma_ts(tmem + COL_W, tmem + COL_KRT + 8 * s, bt, IDESC_N64, s > 0);
        mma_ts(tmem + COL_U, tmem + COL_VT + 8 * s, bt, IDESC_N64, s > 0);
      }
      mma_commit(mma_bar);
    }
    mma_pending = true;
    if (!block_wait(mma_bar, mma_phase)) { failed = true; break; }
    mma_phase ^= 1;
    mma_pending = false;
    tc_fence_after();
    // ---------------------------------------------------------------- W (rows t, key channels) over Kr
    {
      uint32_t r[32];
      tmem_ld32(lane_addr + COL_W + 32 * half, r);
      tmem_wait_ld();
      const int i = jrow;
#pragma unroll
      for (int x = 0; x < 32; ++x) st_tf32(sKQ, sw32(128, 32 * half + x, i), __uint_as_float(r[x]));
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    // ---------------------------------------------------------------- (4) U^T -= S^T W^T, (5a) O^T = S^T Qr^T
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int s = 0; s < 16; ++s) {
        const uint64_t bw = smem_desc_sw128(sbase + OFF_KQ + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024);
        mma_ts(tmem + COL_U, tmem + COL_S + 8 * s, bw, IDESC_U, 1);
      }
#pragma unroll
      for (int s = 0; s < 16; ++s) {
        const uint64_t bq =
            smem_desc_sw128(sbase + OFF_KQ + 8192 + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024);
        mma_ts(tmem + COL_O, tmem + COL_S + 8 * s, bq, IDESC_N64, s > 0);
      }
      mma_commit(mma_bar);
    }
    mma_pending = true;
    if (!block_wait(mma_bar, mma_phase)) { failed = true; break; }
    mma_phase ^= 1;
    mma_pending = false;
    // ---------------------------------------------------------------- (5b) O^T += U^T P^T, (6) S^T += U^T Kc
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const uint64_t bp = smem_desc_sw128(sbase + OFF_P + (s >> 2) * 8192 + (s & 3) * 32, 16, 1024);
        mma_ts(tmem + COL_O, tmem + COL_U + 8 * s, bp, IDESC_N64, 1);
      }
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const uint64_t bk = smem_desc_sw128(sbase + OFF_KCT + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024);
        mma_ts(tmem + COL_S, tmem + COL_U + 8 * s, bk, IDESC_S, 1);
      }
      mma_commit(mma_bar);
    }
    mma_pending = true;
    if (!block_wait(mma_bar, mma_phase)) { failed = true; break; }
    mma_phase ^= 1;
    mma_pending = false;
    tc_fence_after();
    // ---------------------------------------------------------------- O out; S^T columns scaled by G_63
    {
      uint32_t r[32];
      tmem_ld32(lane_addr + COL_O + 32 * half, r);
      tmem_wait_ld();
      if (o && nrows == kC) {
        // full chunk: O [t][j] staged over T and P, written by one TMA store
        TOut *sO = reinterpret_cast<TOut *>(sT);
#pragma unroll
        for (int x = 0; x < 32; ++x)
          sO[(32 * half + x) * kD + jrow] = from_f32<TOut>(__uint_as_float(r[x]));
        fence_proxy_async();
      } else if (o) {
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          const int t = 32 * half + x;
          if (t < nrows)
            o[((size_t)(bofs + cs + t) * H + h) * kD + jrow] = from_f32<TOut>(__uint_as_float(r[x]));
        }
      }
#pragma unroll
      for (int cb = 0; cb < 2; ++cb) {
        const int i0 = 64 * half + 32 * cb;
        tmem_ld32(lane_addr + COL_S + i0, r);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x) r[x] = __float_as_uint(__uint_as_float(r[x]) * sGC[i0 + x]);
        tmem_st32(lane_addr + COL_S + i0, r);
      }
      tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && o && nrows == kC) {
      tma_store_3d(&tm_o, sT, 0, h, (int)(bofs + cs));
      bulk_commit();
      store_pending = true;
    }
  }
  if (tid == 0) bulk_wait_all();

  if (failed) {
    if (tid == 0) set_status(p.status, CKDA_ERR_TIMEOUT);
    // let in-flight copies and MMAs drain (bounded) before giving TMEM back
    if (tma_pending) mbar_wait(tma_bar, tma_phase, kWaitNs);
    if (mma_pending) mbar_wait(mma_bar, mma_phase, kWaitNs);
  } else if (p.S_T) {
    tc_fence_after();
#pragma unroll
    for (int cb = 0; cb < 2; ++cb) {
      uint32_t r[32];
      const int i0 = 64 * half + 32 * cb;
      tmem_ld32(lane_addr + COL_S + i0, r);
      tmem_wait_ld();
#pragma unroll
      for (int x = 0; x < 32; ++x) p.S_T[sofs + (size_t)(i0 + x) * kD + jrow] = __uint_as_float(r[x]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// [rows, H, 128] bf16 viewed as a 3-D tensor (channel, head, token); box 64 x 1 x 64,
// 128-byte swizzle (the staging layout the gate threads read).
bool make_map(CUtensorMap *map, const void *base, int H, long rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)H * kD * 2};
  cuuint32_t box[3] = {64, 1, 64};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// o [rows, H, 128] (bf16 or fp32) for whole-chunk stores: box 128 x 1 x 64, no swizzle.
bool make_out_map(CUtensorMap *map, void *base, int H, long rows, bool bf16) {
  auto enc = get_encode();
  if (!enc) return false;
  const cuuint64_t es = bf16 ? 2 : 4;
  cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)kD * es, (cuuint64_t)H * kD * es};
  cuuint32_t box[3] = {kD, 1, kC};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base,
             dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename TOut, int SG>
int launch_typed(const ChunkArgs &g, cudaStream_t stream) {
  const long rows = (long)g.B * g.T;
  if (rows == 0) {
    // no tokens: S_T = S0 (or zero) is still produced by the kernel below
  }
  CUtensorMap mq, mk, mv, ma, mo;
  const long map_rows = rows > 0 ? rows : 1;
  if (!make_map(&mq, g.q, g.H, map_rows) || !make_map(&mk, g.k, g.H, map_rows) ||
      !make_map(&mv, g.v, g.H, map_rows) || !make_map(&ma, g.a, g.H, map_rows))
    return CKDA_ERR_CUDA;
  memset(&mo, 0, sizeof(mo));
  if (g.o && !make_out_map(&mo, g.o, g.H, map_rows, g.o_dtype == CKDA_BF16)) return CKDA_ERR_CUDA;
  TcParams p;
  p.b = g.b; p.S0 = g.S0; p.cu = g.cu_seqlens; p.o = g.o; p.S_T = g.S_T; p.status = g.status;
  p.n_seqs = g.n_seqs; p.T = g.T; p.H = g.H; p.signed_gate = g.signed_gate;
  auto kern = chunk_tc_kernel<TOut, SG>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes) !=
      cudaSuccess)
    return CKDA_ERR_CUDA;
  kern<<<g.n_seqs * g.H, kThreads, kSmemBytes, stream>>>(mq, mk, mv, ma, mo, p);
  return cudaGetLastError() == cudaSuccess ? CKDA_OK : CKDA_ERR_CUDA;
}

}  // namespace

bool chunk_tc_supported(const ChunkArgs &g) {
  return g.dk == kD && g.dv == kD && g.chunk == kC && g.io_dtype == CKDA_BF16 && g.B * (long)g.T > 0;
}

int launch_chunk_tc(const ChunkArgs &g, cudaStream_t s) {
  if (g.n_seqs * g.H == 0) return CKDA_OK;
  const bool bf = g.o_dtype == CKDA_BF16;
  switch (g.signed_gate) {
    case 0: return bf ? launch_typed<__nv_bfloat16, 0>(g, s) : launch_typed<float, 0>(g, s);
    case 1: return bf ? launch_typed<__nv_bfloat16, 1>(g, s) : launch_typed<float, 1>(g, s);
    default: return bf ? launch_typed<__nv_bfloat16, 2>(g, s) : launch_typed<float, 2>(g, s);
  }
}

}  // namespace ckda

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
constexpr uint32_t OFF_MISC = 229376;   // beta[64], gC[2][128], xch[128], barriers, tmem slot
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

// T = (I + A)^{-1} Diag(beta) for a 64 x 64 strictly lower A (pidx layout),
// written as tf32 into the K-major T tile.  X (plain, stride 64) receives the
// inverse, Y (4 KB) is scratch.  Recursive doubling on the block structure:
//   stage 0: the eight 8 x 8 diagonal blocks by forward substitution (warp w,
//            lane m = column m of block w);
//   stage s = 1, 2, 3: every diagonal block of size 2b = 8 << s is finished
//            from its two halves, X_10 = -X_11 (A_10 X_00), all such blocks at
//            once; each product is spread over all 256 threads.
// The strictly upper part of T is written as zeros at stage 0.
__device__ void solve_T(const float *A, float *X, float *Y, uint8_t *sT, const float *beta, int tid) {
  const int warp = tid >> 5, lane = tid & 31;
  {
    // stage 0 (lanes 0..7 of every warp) and T's upper zeros (all threads)
    if (lane < 8) {
      const int o = 8 * warp, m = lane;
      float x[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        float acc = 0.f;
#pragma unroll
        for (int l = 0; l < r; ++l) acc = fmaf(-A[pidx(o + r, o + l)], x[l], acc);
        x[r] = (r == m) ? 1.f : acc;
      }
      const float bm = beta[o + m];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        X[(o + r) * 64 + o + m] = x[r];
        st_tf32(sT, sw32(64, o + r, o + m), r >= m ? x[r] * bm : 0.f);
      }
    }
    // zeros above the 8 x 8 diagonal blocks, in T and in X (the merges read X's
    // diagonal blocks whole)
    for (int e = tid; e < 64 * 64; e += 256) {
      const int t = e >> 6, s = e & 63;
      if (s >= ((t >> 3) + 1) * 8) {
        st_tf32(sT, sw32(64, t, s), 0.f);
        X[t * 64 + s] = 0.f;
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int st = 1; st <= 3; ++st) {
    const int b = 4 << st;                // half size of the blocks finished here: 8, 16, 32
    const int tpb = (b / 2) * (b / 2);    // 2 x 2 output tiles per block
    const int ntiles = (64 / (2 * b)) * tpb;
    const int blk = tid / tpb, w = tid % tpb, r0 = 2 * (w / (b / 2)), c0 = 2 * (w % (b / 2));
    const int o = blk * 2 * b;
    float *Yb = Y + blk * b * b;
    // phase 1: Y = A_10 X_00 (A_10: rows o+b.., columns o..; X_00: the upper diagonal block)
    if (tid < ntiles) {
      float y00 = 0.f, y01 = 0.f, y10 = 0.f, y11 = 0.f;
#pragma unroll 8
      for (int l = 0; l < b; ++l) {
        const float a0 = A[pidx(o + b + r0, o + l)], a1 = A[pidx(o + b + r0 + 1, o + l)];
        const float2 xv = *reinterpret_cast<const float2 *>(X + (o + l) * 64 + o + c0);
        y00 = fmaf(a0, xv.x, y00); y01 = fmaf(a0, xv.y, y01);
        y10 = fmaf(a1, xv.x, y10); y11 = fmaf(a1, xv.y, y11);
      }
      *reinterpret_cast<float2 *>(Yb + r0 * b + c0) = make_float2(y00, y01);
      *reinterpret_cast<float2 *>(Yb + (r0 + 1) * b + c0) = make_float2(y10, y11);
    }
    __syncthreads();
    // phase 2: X_10 = -X_11 Y (X_11: the lower diagonal block, finished earlier)
    if (tid < ntiles) {
      float z00 = 0.f, z01 = 0.f, z10 = 0.f, z11 = 0.f;
#pragma unroll 8
      for (int l = 0; l < b; ++l) {
        const float x0 = X[(o + b + r0) * 64 + o + b + l], x1 = X[(o + b + r0 + 1) * 64 + o + b + l];
        const float2 yv = *reinterpret_cast<const float2 *>(Yb + l * b + c0);
        z00 = fmaf(-x0, yv.x, z00); z01 = fmaf(-x0, yv.y, z01);
        z10 = fmaf(-x1, yv.x, z10); z11 = fmaf(-x1, yv.y, z11);
      }
      float *X0 = X + (o + b + r0) * 64 + o + c0;
      *reinterpret_cast<float2 *>(X0) = make_float2(z00, z01);
      *reinterpret_cast<float2 *>(X0 + 64) = make_float2(z10, z11);
      const float b0 = beta[o + c0], b1 = beta[o + c0 + 1];
      st_tf32(sT, sw32(64, o + b + r0, o + c0), z00 * b0);
      st_tf32(sT, sw32(64, o + b + r0, o + c0 + 1), z01 * b1);
      st_tf32(sT, sw32(64, o + b + r0 + 1, o + c0), z10 * b0);
      st_tf32(sT, sw32(64, o + b + r0 + 1, o + c0 + 1), z11 * b1);
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
  float *sBeta = reinterpret_cast<float *>(sm + OFF_MISC);     // [64]
  float *sGC = sBeta + 64;                                       // [2][128] G_63, double-buffered
  float *sXch = sGC + 256;                                       // [128]
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_MISC + 1792);
  uint64_t *tma_bar = bars, *mma_bar = bars + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_MISC + 1808);
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
  // TMEM lane of this thread and which half of a row it handles; the gate pass
  // uses the same mapping (channel c = jrow, rows 32*half .. 32*half + 31).
  const int half = warp >> 2;
  const int jrow = 32 * (warp & 3) + lane;
  const int c = jrow, hf = half;
  const uint32_t lane_addr = tmem + ((uint32_t)(32 * (warp & 3)) << 16);

  uint32_t tma_phase = 0, mma_phase = 0;
  bool tma_pending = false, mma_pending = false, failed = false, store_pending = false;

  // descriptors of the fixed operand tiles (K-major, 128-byte swizzle)
  const uint64_t dKQ = smem_desc_sw128(sbase + OFF_KQ, 16, 1024);
  const uint64_t dKC = smem_desc_sw128(sbase + OFF_KC, 16, 1024);
  const uint64_t dKCT = smem_desc_sw128(sbase + OFF_KCT, 16, 1024);
  const uint64_t dT = smem_desc_sw128(sbase + OFF_T, 16, 1024);
  const uint64_t dP = smem_desc_sw128(sbase + OFF_P, 16, 1024);
  auto dadd = [](uint64_t d, uint32_t bytes) -> uint64_t { return d + (bytes >> 4); };

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

  const uint8_t *stq = sStg, *stk = sStg + 16384, *stv = sStg + 32768, *sta = sStg + 49152;

  // ---- gate pass: staging (q, k, v, a of one chunk) -> Kr, Qr, Kc, Kc^T tiles, Kr^T and V^T
  // in TMEM, beta, G_63.  Kc^T is left in kc[] for the caller to store (its tile may still be
  // read by the previous chunk's last MMA group).  Returns whether the chunk is out of range.
  float b_next = 0.f;
  if (tid < kC && t0 + tid < t1) b_next = p.b[(size_t)(bofs + t0 + tid) * H + h];
  float kc[32];
  auto gate_pass = [&](long cs, int nrows, float *gc_out) -> bool {
    const float b_cur = b_next;
    if (tid < kC && cs + kC + tid < t1) b_next = p.b[(size_t)(bofs + cs + kC + tid) * H + h];
    float g[32];
    float run = 1.f;
#pragma unroll
    for (int rr = 0; rr < 32; ++rr) {
      const int r = 32 * hf + rr;
      const float al = fast_alpha<SG>(ldbf(sta, r, c));
      run *= r < nrows ? al : 1.f;
      g[rr] = run;
    }
    if (hf == 0) sXch[c] = run;
    if (tid < kC) sBeta[tid] = tid < nrows ? fast_beta<SG>(b_cur) : 0.f;
    __syncthreads();
    bool bad = false;
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
        const uint32_t kr = to_tf32(kv * gam);
        const uint32_t kcb = to_tf32(kv * inv);
        *reinterpret_cast<uint32_t *>(sKQ + sw32(128, r, c)) = kr;
        st_tf32(sKQ, sw32(128, 64 + r, c), qv * gam);
        *reinterpret_cast<uint32_t *>(sKC + sw32(64, r, c)) = kcb;
        kc[rr] = __uint_as_float(kcb);
        krt[x] = kr;
        vt[x] = __float_as_uint(vv);
        if (rr == 31 && hf == 1) gc_out[c] = gam;
      }
      // lane c of TMEM holds Kr^T[c][.] and V^T[c][.] (A operands of (2) and (3))
      tmem_st16(lane_addr + COL_KRT + 32 * hf + 16 * grp, krt);
      tmem_st16(lane_addr + COL_VT + 32 * hf + 16 * grp, vt);
    }
    tmem_wait_st();
    return bad;
  };
  auto store_kct = [&]() {  // four consecutive t per 16-byte store
#pragma unroll
    for (int rr = 0; rr < 32; rr += 4)
      *reinterpret_cast<float4 *>(sKCT + sw32(128, c, 32 * hf + rr)) =
          make_float4(kc[rr], kc[rr + 1], kc[rr + 2], kc[rr + 3]);
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
  if (tid == 0 && t1 > t0) issue_tma(t0);
  tma_pending = t1 > t0;
  tc_fence_before();
  __syncthreads();

  // gate pass of the first chunk
  int gsel = 0;              // sGC buffer of the chunk being processed
  bool slow = false;
  if (t1 > t0) {
    if (!block_wait(tma_bar, tma_phase)) failed = true;
    tma_phase ^= 1;
    tma_pending = false;
    if (!failed) {
      const bool bad = gate_pass(t0, (int)(t1 - t0 < kC ? t1 - t0 : kC), sGC);
      store_kct();
      fence_proxy_async();
      tc_fence_before();
      slow = __syncthreads_or(bad) != 0;
    }
  }

  for (long cs = t0; cs < t1 && !failed; cs += kC) {
    const int nrows = (int)(t1 - cs < kC ? t1 - cs : kC);
    const bool has_next = cs + kC < t1;
    const int nrows_next = has_next ? (int)(t1 - cs - kC < kC ? t1 - cs - kC : kC) : 0;
    float *gc_cur = sGC + 128 * gsel, *gc_next = sGC + 128 * (gsel ^ 1);

    if (slow) {
      // ------------------------------------------------------------ exact token-by-token path
      // state S[i][j] in smem over Kr/Qr, gates over Kc, partial sums over Kc^T
      float *sS = reinterpret_cast<float *>(sKQ);
      float *sAl = reinterpret_cast<float *>(sKC);
      float *sRed = reinterpret_cast<float *>(sKCT);
#pragma unroll 4
      for (int rr = 0; rr < 32; ++rr) {
        const int r = 32 * hf + rr;
        sAl[r * kD + c] = r < nrows ? gate_alpha(ldbf(sta, r, c), SG) : 1.f;
      }
      tc_fence_after();
#pragma unroll
      for (int cb = 0; cb < 2; ++cb) {
        uint32_t r[32];
        const int i0 = 64 * half + 32 * cb;
        tmem_ld32(lane_addr + COL_S + i0, r);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x) sS[(i0 + x) * kD + jrow] = __uint_as_float(r[x]);
      }
      __syncthreads();
      for (int t = 0; t < nrows; ++t) {
        float pk = 0.f;
        for (int x = 0; x < 64; ++x) {
          const int i = 64 * half + x;
          const float sv = sS[i * kD + jrow] * sAl[t * kD + i];
          sS[i * kD + jrow] = sv;
          pk = fmaf(ldbf(stk, t, i), sv, pk);
        }
        sRed[half * 128 + jrow] = pk;
        __syncthreads();
        const float u = sBeta[t] * (ldbf(stv, t, jrow) - (sRed[jrow] + sRed[128 + jrow]));
        float acc = 0.f;
        for (int x = 0; x < 64; ++x) {
          const int i = 64 * half + x;
          const float sv = fmaf(ldbf(stk, t, i), u, sS[i * kD + jrow]);
          sS[i * kD + jrow] = sv;
          acc = fmaf(ldbf(stq, t, i), sv, acc);
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
        const int i0 = 64 * half + 32 * cb;
#pragma unroll
        for (int x = 0; x < 32; ++x) r[x] = __float_as_uint(sS[(i0 + x) * kD + jrow]);
        tmem_st32(lane_addr + COL_S + i0, r);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncthreads();
      if (has_next) {
        if (tid == 0) issue_tma(cs + kC);
        tma_pending = true;
        if (!block_wait(tma_bar, tma_phase)) { failed = true; break; }
        tma_phase ^= 1;
        tma_pending = false;
        const bool bad = gate_pass(cs + kC, nrows_next, gc_next);
        store_kct();
        fence_proxy_async();
        tc_fence_before();
        slow = __syncthreads_or(bad) != 0;
        gsel ^= 1;
      }
      continue;
    }

    // ---------------------------------------------------------------- (1) [A;P] = [Kr;Qr] Kc^T
    if (tid == 0) {
      if (has_next) issue_tma(cs + kC);   // staging is free: the gate pass has consumed it
      tc_fence_after();
#pragma unroll
      for (int s = 0; s < 16; ++s) {
        const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
        mma_ss(tmem + COL_AP, dadd(dKQ, off), dadd(dKC, (s >> 2) * 8192 + (s & 3) * 32), IDESC_N64,
               s > 0);
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
    float *sX = sA + 64 * 64;                              // plain [64][64]
    float *sY = reinterpret_cast<float *>(sKQ);           // [3][16][16] over the consumed Kr rows
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
    solve_T(sA, sX, sY, sT, sBeta, tid);
    fence_proxy_async();
    __syncthreads();
    // ---------------------------------------------------------------- (2) W^T, (3) U^T
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const uint64_t bt = dadd(dT, (s >> 2) * 8192 + (s & 3) * 32);
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
        const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
        mma_ts(tmem + COL_U, tmem + COL_S + 8 * s, dadd(dKQ, off), IDESC_U, 1);
      }
#pragma unroll
      for (int s = 0; s < 16; ++s) {
        const uint32_t off = 8192 + (s >> 2) * 16384 + (s & 3) * 32;
        mma_ts(tmem + COL_O, tmem + COL_S + 8 * s, dadd(dKQ, off), IDESC_N64, s > 0);
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
      for (int s = 0; s < 8; ++s)
        mma_ts(tmem + COL_O, tmem + COL_U + 8 * s, dadd(dP, (s >> 2) * 8192 + (s & 3) * 32),
               IDESC_N64, 1);
#pragma unroll
      for (int s = 0; s < 8; ++s)
        mma_ts(tmem + COL_S, tmem + COL_U + 8 * s, dadd(dKCT, (s >> 2) * 16384 + (s & 3) * 32),
               IDESC_S, 1);
      mma_commit(mma_bar);
    }
    mma_pending = true;
    // ---------------------------------------------------------------- next chunk's gate pass,
    // overlapping (5b)/(6): Kr, Qr and Kc are free, Kc^T is not (kept in registers)
    bool bad_next = false;
    if (has_next) {
      if (!block_wait(tma_bar, tma_phase)) { failed = true; break; }
      tma_phase ^= 1;
      tma_pending = false;
      bad_next = gate_pass(cs + kC, nrows_next, gc_next);
    }
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
        for (int x = 0; x < 32; ++x) r[x] = __float_as_uint(__uint_as_float(r[x]) * gc_cur[i0 + x]);
        tmem_st32(lane_addr + COL_S + i0, r);
      }
      tmem_wait_st();
    }
    if (has_next) store_kct();
    fence_proxy_async();
    tc_fence_before();
    slow = __syncthreads_or(bad_next) != 0;
    if (tid == 0 && o && nrows == kC) {
      tma_store_3d(&tm_o, sT, 0, h, (int)(bofs + cs));
      bulk_commit();
      store_pending = true;
    }
    gsel ^= 1;
  }
  if (tid == 0) bulk_wait_all();

  if (failed) {
    if (tid == 0) set_status(p.status, CKDA_ERR_TIMEOUT);
    // let in-flight copies and MMAs drain (bounded) before giving TMEM back
    if (warp == 0) {
      if (tma_pending) mbar_wait(tma_bar, tma_phase, kWaitNs);
      if (mma_pending) mbar_wait(mma_bar, mma_phase, kWaitNs);
    }
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

extern "C" int ckda_timed_solve(unsigned long long *out) {
}

extern "C" int ckda_timed_phases(unsigned long long *out) {
}

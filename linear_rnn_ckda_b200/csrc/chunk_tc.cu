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
//   U  = Tm (V - Kr S)          (the WY form U = Tm V - (Tm Kr) S, regrouped)
//   O  = Qr S + P U
//   S' = Diag(G_63) (S + Kc^T U)
// Everything is computed transposed so that every product has M = 128 on the
// tensor core: the state lives in TMEM as S^T (lane = value channel j,
// column = key channel i) and is the A operand of the state products.
//   (1) [A;P]   = [Kr;Qr] Kc^T          M=128 (64 Kr rows + 64 Qr rows), N=64, K=128
//   (a) [X^T|O^T] = S^T [Kr;Qr]^T       N=128 (X = Kr S, and O's first term), K=128
//   (b) V' = V - X in fp32 (threads), kept in TMEM as tf32 hi + lo parts
//   (c) U^T     = V'^T Tm^T              A = V'^T in TMEM (hi and lo), K=64, then three corrections
//   (d) [O^T|S^T] += U^T [P;Kc^T]^T     N=192, then S^T columns scaled by G_63 (threads)
// (1) and (a) need only the chunk's inputs and S, so they are issued together
// when the chunk starts, and (b) overlaps the solve.  All MMAs are kind::tf32
// with fp32 accumulation and K-major operands; smem operands are rounded to
// tf32 (round-to-nearest) when written.  TMEM operands (S, U) are read as tf32
// directly (the low mantissa bits ignored); V' is split so that none of it is
// lost.  The gate products are the signed cumulative products in fp32
// (the sign bit carries the gate-sign parity).
//
// Range of the factorisation.  Kr Kc^T needs G_t and 1/G_t in fp32 for every row.
// A channel whose chunk product stays above 2^-100 uses them as they are.  A
// faster-decaying channel i carries a power-of-two reference R_i = 2^e_i, with e_i
// half the channel's exponent sum over the chunk (exponents summed exactly, so no
// product underflows on the way): Kr, Qr use G / R and Kc uses R / G, which leaves
// A and P unchanged and keeps both factors within 2^+-110 for a chunk decay down
// to 2^-220.  The state is then kept scaled, S^ = Diag(R) S, so that (a) and (d)
// stay the same products:
//   X = (Kr/R) S^,  O = (Qr/R) S^ + P U,  S^' = Diag(R') Diag(G_63 / R) (S^ + (Kc R)^T U)
// with R' the next chunk's reference, applied after G_63 / R (their product can fall below
// fp32's range while S' itself does not).  A
// chunk that decays further in some channel is cut after its last row group of 8
// that fits (the next chunk starts there); a chunk whose first 8 rows already do
// not fit (an exact zero gate, a NaN, decay beyond 2^-126 in 8 rows) runs those
// rows token by token, exactly, on the same TMEM-resident state (slow path).
// Raw gates (which may exceed 1) keep the reference 1 and send a chunk outside
// [2^-100, 2^100] to the slow path whole.
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
constexpr int kCompute = 512;               // 16 compute warps: 4 per scheduler
constexpr int kThreads = kCompute + 32;     // + one warp that issues TMA loads and MMAs
constexpr int kBarC = 1;                    // named barrier of the compute warps

// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_KQ = 0;          // [Kr;Qr] 128 rows x 128 fp32, 4 column blocks of 16 KB
constexpr uint32_t OFF_KC = 65536;      // Kc 64 rows x 128 fp32, 4 column blocks of 8 KB;
                                        // then the solve's A (64 x kAS) (or the gate pass's
                                        // exchange) and the R tiles
constexpr uint32_t OFF_R2 = OFF_KC + 18432;    // [M10; M20; M30]: 48 rows, K = 16 of 32
constexpr uint32_t OFF_R34 = OFF_KC + 24576;   // [M21; M31; M32]: 48 rows, K = 16 of 32
constexpr uint32_t OFF_PK = 98304;      // [P; Kc^T]: 64 + 128 rows x 64 fp32, the B operand of
                                        // (d); each 32-column block holds P's 64 rows and then
                                        // Kc^T's 128 rows (24 KB)
constexpr uint32_t OFF_T = 147456;      // Tm 64 x 64 fp32, 2 column blocks of 8 KB; bf16 O staging
constexpr uint32_t OFF_STG = 163840;    // TMA staging: q, k, v, a bf16 64 x 128 (16 KB each)
constexpr uint32_t OFF_MISC = 229376;   // beta[64], gC[2][128], barriers, tmem slot, abort flag
constexpr uint32_t kSmemUsed = OFF_MISC + 2048;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;  // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory budget");

// TMEM columns (all 512 allocated)
// [A;P] and, once read out, the lo part of V'; X, O and S adjacent so that (a) writes
// [X|O] and (d) writes [O|S] as single products; V^T (then the hi part of V') of two
// chunks in COL_VT0 and COL_VT1
constexpr uint32_t COL_U = 0, COL_VT0 = 64, COL_AP = 128, COL_LO = 128, COL_X = 192, COL_O = 256,
                   COL_S = 320, COL_VT1 = 448;

constexpr uint32_t IDESC_N64 = idesc_tf32(128, 64, false, false);         // (1), (c), O += U P^T
constexpr uint32_t IDESC_N48_NEG = idesc_tf32(128, 48, false, false, true);  // (c) correction 1
constexpr uint32_t IDESC_N32_NEG = idesc_tf32(128, 32, false, false, true);  // (c) correction 2
constexpr uint32_t IDESC_N16_NEG = idesc_tf32(128, 16, false, false, true);  // (c) correction 3
constexpr uint32_t IDESC_N128 = idesc_tf32(128, 128, false, false);       // (a)
constexpr uint32_t IDESC_N192 = idesc_tf32(128, 192, false, false);       // (d)

constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s bound on any single wait
// bound on the waits that drain in-flight copies and products before a unit gives up (these
// always finish; the bound only keeps a broken invariant from hanging the GPU)
constexpr uint64_t kDrainNs = 2000000000ull;

struct TcParams {
  const float *b;
  const float *S0;
  const int32_t *cu;
  void *o;
  float *S_T;
  int *status;
  int n_seqs, T, H, signed_gate;
  int inject_chunk;         // test hook: chunk index of the never-completing wait (-1: off)
  uint64_t inject_wait_ns;  // its bound
  const __nv_bfloat16 *a_head;  // per-head gate logits [rows, H] (CKDA_GATE_PER_HEAD), else NULL
  // Hand-off of units whose gates decay past the plain kernel's range to the kernel with
  // per-channel references (NULL: none, such chunks run token by token).  The plain kernel
  // appends (sequence, head, first row, 0) to queue and the state at that row to saved_S
  // ([entry][dk][dv]); the kernel with references takes entry blockIdx.x.
  int *queue_count;
  int4 *queue;
  float *saved_S;
  // Unit list of a planned launch (NULL: unit = (sequence, head) in length order): CTA x runs
  // entry x / H for head x % H when x / H < *plan_count.  slots holds the cut sequences' states.
  const SegDesc *plan;
  const int *plan_count;
  float *slots;
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
// byte offset of fp32 element (r, c) of the [P; Kc^T] tile (r < 64: P, else Kc^T row r - 64)
__device__ __forceinline__ uint32_t swpk(int r, int c) {
  return (uint32_t)((c >> 5) * 24576 + r * 128 + ((((c & 31) >> 2) ^ (r & 7)) << 4) +
                    ((c & 3) << 2));
}
__device__ __forceinline__ void st_tf32(uint8_t *tile, uint32_t off, float x) {
  *reinterpret_cast<uint32_t *>(tile + off) = to_tf32(x);
}

// beta for the bf16 path from its definition with a fast exponential (relative error ~1e-6,
// far inside the bf16-input tolerance): sigma(b) (KDA), 2 sigma(b) (CKDA), b (raw)
__device__ __forceinline__ float fast_beta(float b, int form) {
  if (form == 0) return __fdividef(1.f, 1.f + __expf(-b));
  if (form == 1) return __fdividef(2.f, 1.f + __expf(-b));
  return b;
}

// 2^n as an fp32 number, built from its exponent field (n clamped to the normal range)
__device__ __forceinline__ float exp2i(int n) {
  n = n < -126 ? -126 : (n > 127 ? 127 : n);
  return __uint_as_float((uint32_t)(n + 127) << 23);
}

// Bound on |log2| of the scaled gate factors G/R and R/G of a chunk (the reference R sits
// halfway): a channel may decay by up to 2^-2kRefRange over one chunk.  The margin to fp32's
// 2^-126 keeps a key component down to 2^-16 times a factor a normal number.
constexpr int kRefRange = 110;

// The gate products of one chunk are exchanged between the gate-pass threads as
// xp[(x * 128 + ch) * 2 + {0, 1}]: the product of the gates of row group x (rows 8x .. 8x + 7) in
// channel ch, and the product of their inverses.
//
// The reference exponent of a channel whose product over a chunk has the exponent sum etot
// (summed exactly from its group products): none while the product stays above 2^-100, else
// half the sum (toward zero), which centres G / R and R / G.
__device__ __forceinline__ int ref_exponent(int etot) { return etot >= -100 ? 0 : -((-etot) >> 1); }

// The references (e0, e1) of channels ch0, ch0 + 1 from the products of row groups 0 .. ng-1;
// false if one of them, or its inverse, is not a normal number or a channel decays below
// 2^-2kRefRange over those groups (no reference brings its factors within 2^+-kRefRange).
__device__ __forceinline__ bool chunk_refs(const float *xp, int ch0, int ng, int &e0, int &e1) {
  int es0 = 0, es1 = 0;
  bool ok = true;
#pragma unroll 1
  for (int x = 0; x < ng; ++x) {
    const float4 v = *reinterpret_cast<const float4 *>(xp + (x * 128 + ch0) * 2);
    const int f0 = (int)((__float_as_uint(v.x) >> 23) & 255u);
    const int i0 = (int)((__float_as_uint(v.y) >> 23) & 255u);
    const int f1 = (int)((__float_as_uint(v.z) >> 23) & 255u);
    const int i1 = (int)((__float_as_uint(v.w) >> 23) & 255u);
    ok &= f0 >= 1 && f0 <= 254 && i0 >= 1 && i0 <= 254 && f1 >= 1 && f1 <= 254 && i1 >= 1 &&
          i1 <= 254;
    es0 += f0 - 127;
    es1 += f1 - 127;
  }
  e0 = ref_exponent(es0);
  e1 = ref_exponent(es1);
  return ok && es0 >= -2 * kRefRange && es1 >= -2 * kRefRange;
}

// The first row group (8 if none) of channels ch0, ch0 + 1 whose product, or its inverse, is not
// a normal number, or past which the chunk's exponent sum drops below -2kRefRange.
__device__ __forceinline__ int first_failing_group(const float *xp, int ch0) {
  int es0 = 0, es1 = 0;
#pragma unroll 1
  for (int x = 0; x < 8; ++x) {
    const float4 v = *reinterpret_cast<const float4 *>(xp + (x * 128 + ch0) * 2);
    const int e0 = (int)((__float_as_uint(v.x) >> 23) & 255u);
    const int i0 = (int)((__float_as_uint(v.y) >> 23) & 255u);
    const int e1 = (int)((__float_as_uint(v.z) >> 23) & 255u);
    const int i1 = (int)((__float_as_uint(v.w) >> 23) & 255u);
    es0 += e0 - 127;
    es1 += e1 - 127;
    const bool normal = e0 >= 1 && e0 <= 254 && i0 >= 1 && i0 <= 254 && e1 >= 1 && e1 <= 254 &&
                        i1 >= 1 && i1 <= 254;
    if (!normal || es0 < -2 * kRefRange || es1 < -2 * kRefRange) return x;
  }
  return 8;
}

// ---------------------------------------------------------------- the gate pass proper
// Run by the 512 compute threads of a CTA on the chunk in the staging tiles: V^T into TMEM
// (columns vcol..vcol+63), the Kr, Qr tile, Kc (returned in kc, stored later by the caller)
// and G_63 / R (gc_out).  Thread (pair pc = tid % 64, row group rg = tid / 64) takes channels
// 2pc, 2pc + 1 of rows 8rg .. 8rg + 7, reading bf16 pairs and writing 8-byte pairs; V^T keeps
// the one-channel-per-lane mapping TMEM needs.  Returns whether a channel of this thread leaves
// the range with the references e0, e1 it was given (R = 2^e for channels 2pc, 2pc + 1; 0: none).
// (Everything is inline: an out-of-line call anywhere in the kernel costs the common path about
// 15 %.)
// the gate and (KDA, CKDA) its inverse, so that the second part needs no reciprocal:
//   KDA   sigma(a) = 1 / (1 + e^{-a}), inverse 1 + e^{-a}
//   CKDA  2 sigma(a) - 1 = tanh(a/2) = sign(a) (1 - e^{-|a|}) / (1 + e^{-|a|}), inverse the
//         ratio upside down; both from one reciprocal r = 1 / (num den) (num r = 1 / den,
//         den r = 1 / num).  Small |a|: 1 - e^{-|a|} cancels, an error at fp32 rounding level
//         in absolute terms.  a = 0 gives 0 or NaN (0 inf): either fails the range check.
template <int SG>
__device__ __forceinline__ void gate_pair(float a, float &al, float &ial) {
  if (SG == 0) {
    const float e = __expf(-a);
    ial = 1.f + e;
    al = __fdividef(1.f, ial);
  } else if (SG == 1) {
    const float e = __expf(-fabsf(a));
    const float num = 1.f - e, den = 1.f + e;
    const float r = __fdividef(1.f, num * den);
    al = copysignf(num * (num * r), a);
    ial = copysignf(den * (den * r), a);
  } else {
    ial = 1.f;
    al = a;
  }
}

template <int SG, int FL, bool REFS>
__device__ __forceinline__ bool gate_pass_body(uint8_t *sm, uint32_t tmem, int signed_gate,
                                               int nrows, float b_this, __nv_bfloat16 a_this,
                                               float *gc_out, uint32_t vcol, float (&kc)[16],
                                               int e0, int e1) {
  constexpr bool per_head = (FL & 1) != 0;
  constexpr bool l2 = (FL & 2) != 0;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qg = warp >> 2, c = 32 * (warp & 3) + lane;
  const uint32_t lane_addr = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
  const int pc = tid & 63, rg = tid >> 6, ch0 = 2 * pc;
  uint8_t *sStg = sm + OFF_STG;
  const uint8_t *stq = sStg, *stk = stq + 16384, *stv = stq + 32768, *sta = stq + 49152;
  uint8_t *sKQ = sm + OFF_KQ;
  float *sXp = reinterpret_cast<float *>(sm + OFF_KC);
  float *sBeta = reinterpret_cast<float *>(sm + OFF_MISC);
  __nv_bfloat16 *sAh = reinterpret_cast<__nv_bfloat16 *>(sm + OFF_MISC + 1408);
  float *sInvQ = reinterpret_cast<float *>(sm + OFF_MISC + 1536), *sInvK = sInvQ + kC;
  if (tid < kC) sBeta[tid] = tid < nrows ? fast_beta(b_this, beta_form(signed_gate)) : 0.f;
  if (per_head && tid < kC) {
    // the chunk's per-head gate logits (rows past the end: a gate of exactly 1)
    sAh[tid] = tid < nrows ? a_this : __float2bfloat16_rn(SG == 2 ? 1.f : 100.f);
  }
  if (nrows < kC) {
    // Rows past the sequence end (or a cut) hold other tokens or TMA fill.  They are
    // overwritten in the staging copy with q = k = v = 0 and a gate of exactly 1
    // (a = 100 gives sigma(a) = 2 sigma(a) - 1 = 1 in fp32; raw gates take a = 1), so
    // the pass needs no per-row masking.
    const uint32_t afill = SG == 2 ? 0x3F803F80u : 0x42C842C8u;   // bf16 pairs 1.0, 100.0
    const int nt = (kC - nrows) * 16;   // 16-byte pieces of one array: 8 per row and box
    for (int e = tid; e < 4 * nt; e += kCompute) {
      const int x = e / nt, rem = e - x * nt;
      const int row = nrows + (rem >> 4), piece = rem & 15;
      const uint32_t f = x == 3 ? afill : 0u;
      *reinterpret_cast<uint4 *>(sStg + x * 16384 + (piece >> 3) * 8192 + row * 128 +
                                 (piece & 7) * 16) = make_uint4(f, f, f, f);
    }
    bar_sync(kBarC, kCompute);
  } else if (per_head || l2) {
    bar_sync(kBarC, kCompute);
  }
  if (l2) {
    // 1 / ||q_r|| and 1 / ||k_r|| over the key channels: warp w takes rows w, w + 16, ...
    // of q and of k, four channels per lane (8 bytes inside one 16-byte chunk); they are
    // read after the exchange barrier below
    for (int it = warp; it < 2 * kC; it += kCompute / 32) {
      const int r = it % kC;
      const uint8_t *tile = it < kC ? stq : stk;
      const uint2 u = *reinterpret_cast<const uint2 *>(tile + swbf(r, 4 * lane));
      const float x0 = __uint_as_float(u.x << 16), x1 = __uint_as_float(u.x & 0xFFFF0000u);
      const float x2 = __uint_as_float(u.y << 16), x3 = __uint_as_float(u.y & 0xFFFF0000u);
      float ss = fmaf(x0, x0, fmaf(x1, x1, fmaf(x2, x2, x3 * x3)));
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      if (lane == 0) (it < kC ? sInvQ : sInvK)[r] = inv_norm(ss);
    }
  }
  auto ldbf2 = [&](const uint8_t *tile, int r, float &x0, float &x1) {
    const uint32_t u = *reinterpret_cast<const uint32_t *>(tile + swbf(r, ch0));
    x0 = __uint_as_float(u << 16);
    x1 = __uint_as_float(u & 0xFFFF0000u);
  };
  {
    // lane c of TMEM holds V^T[c][.] (V' = V - X is formed in place before (c))
    uint32_t vt[16];
#pragma unroll
    for (int rr = 0; rr < 16; ++rr) vt[rr] = __float_as_uint(ldbf(stv, 16 * qg + rr, c));
    tmem_st16(lane_addr + vcol + 16 * qg, vt);
  }
  // [row][channel of the pair]: the running products of the gates and of their inverses within
  // the row group (the inverse factors need no reciprocal: the gate pass is sensitive to the
  // special-function unit's throughput)
  float g[16], ig[16];
  float run0 = 1.f, run1 = 1.f, irun0 = 1.f, irun1 = 1.f;
#pragma unroll
  for (int rr = 0; rr < 8; ++rr) {
    float a0, a1, al0, al1, ial0, ial1;
    if (per_head) {
      a0 = a1 = __bfloat162float(sAh[8 * rg + rr]);
    } else {
      ldbf2(sta, 8 * rg + rr, a0, a1);
    }
    if (SG == 1) {
      // the pair's CKDA ratios in packed fp32 pairs (same arithmetic as gate_pair)
      const uint64_t one = f2pk(1.f, 1.f);
      const uint64_t e = f2pk(__expf(-fabsf(a0)), __expf(-fabsf(a1)));
      const uint64_t num = f2sub(one, e), den = f2add(one, e);
      float p0, p1;
      f2up(f2mul(num, den), p0, p1);
      // the gate's sign rides on the shared reciprocal: num^2 r and den^2 r take it
      const uint64_t rr2 = f2pk(copysignf(__fdividef(1.f, p0), a0),
                                copysignf(__fdividef(1.f, p1), a1));
      f2up(f2mul(num, f2mul(num, rr2)), al0, al1);
      f2up(f2mul(den, f2mul(den, rr2)), ial0, ial1);
    } else {
      gate_pair<SG>(a0, al0, ial0);
      gate_pair<SG>(a1, al1, ial1);
    }
    run0 *= al0;
    run1 *= al1;
    g[2 * rr] = run0;
    g[2 * rr + 1] = run1;
    if (SG != 2) {
      irun0 *= ial0;
      irun1 *= ial1;
      ig[2 * rr] = irun0;
      ig[2 * rr + 1] = irun1;
    }
  }
  *reinterpret_cast<float4 *>(sXp + (rg * 128 + ch0) * 2) = make_float4(run0, irun0, run1, irun1);
  bar_sync(kBarC, kCompute);
  // the row group's prefix factors G/R and R/G: products of the earlier row groups (of the
  // gates and of their inverses), started at 1/R and R so that no partial product leaves fp32's
  // range (G_t / R lies between 2^-e and G_63 / R)
  float mult0 = exp2i(-e0), mult1 = exp2i(-e1), imult0 = exp2i(e0), imult1 = exp2i(e1);
#pragma unroll
  for (int x = 0; x < 7; ++x)
    if (x < rg) {
      const float4 v = *reinterpret_cast<const float4 *>(sXp + (x * 128 + ch0) * 2);
      mult0 *= v.x;
      imult0 *= v.y;
      mult1 *= v.z;
      imult1 *= v.w;
    }
  // each group's own product a normal number (below 2^-126 the running products lose bits)
  bool bad = SG != 2 && !(fabsf(run0) >= 0x1p-126f && fabsf(run1) >= 0x1p-126f);
#pragma unroll
  for (int rr = 0; rr < 8; ++rr) {
    const int r = 8 * rg + rr;
    const float gam0 = g[2 * rr] * mult0, gam1 = g[2 * rr + 1] * mult1;
    if (SG == 2) {
      const float ag0 = fabsf(gam0), ag1 = fabsf(gam1);
      bad |= !(ag0 >= 0x1p-100f && ag0 <= 0x1p100f && ag1 >= 0x1p-100f && ag1 <= 0x1p100f);
    }
    // R / G_t: the earlier groups' inverse product times this group's inverse running product
    float inv0, inv1;
    if constexpr (SG == 2) {
      inv0 = __fdividef(1.f, gam0);
      inv1 = __fdividef(1.f, gam1);
    } else {
      inv0 = ig[2 * rr] * imult0;
      inv1 = ig[2 * rr + 1] * imult1;
    }
    if (SG != 2 && rr == 7 && rg == 7) {
      // |alpha| <= 1: G/R falls and R/G grows along the chunk, so the last row decides (a NaN
      // gate reaches it too)
      const float ag0 = fabsf(gam0), ag1 = fabsf(gam1), ai0 = fabsf(inv0), ai1 = fabsf(inv1);
      bad |= !(ag0 >= 0x1p-110f && ag1 >= 0x1p-110f && ai0 <= 0x1p110f && ai1 <= 0x1p110f);
    }
    float q0, q1, k0, k1;
    ldbf2(stq, r, q0, q1);
    ldbf2(stk, r, k0, k1);
    if (l2) {
      const float iq = sInvQ[r], ik = sInvK[r];
      q0 *= iq;
      q1 *= iq;
      k0 *= ik;
      k1 *= ik;
    }
    *reinterpret_cast<uint2 *>(sKQ + sw32(128, r, ch0)) =
        make_uint2(to_tf32(k0 * gam0), to_tf32(k1 * gam1));
    *reinterpret_cast<uint2 *>(sKQ + sw32(128, 64 + r, ch0)) =
        make_uint2(to_tf32(q0 * gam0), to_tf32(q1 * gam1));
    kc[2 * rr] = __uint_as_float(to_tf32(k0 * inv0));
    kc[2 * rr + 1] = __uint_as_float(to_tf32(k1 * inv1));
    if (rr == 7 && rg == 7) *reinterpret_cast<float2 *>(gc_out + ch0) = make_float2(gam0, gam1);
  }
  tmem_wait_st();
  return bad;
}


// Row stride (floats) of the plain A array: consecutive rows start 16 bytes
// apart modulo 128, so 32 threads writing 16 bytes of 32 different rows hit
// every bank once per wavefront.
constexpr int kAS = 68;

// Tm = (I + A)^{-1} Diag(beta) for the 64 x 64 strictly lower A (plain, row stride kAS,
// zeros on and above the diagonal), in 16 x 16 blocks i, j = 0..3 with diagonal blocks
// D_i = I + A_ii.  Block forward substitution of (I + A) U = Diag(beta) V' gives
//   U_i = Ub_i - sum_{j<i} M_ij U_j,   Ub = Tb V',  Tb = blockdiag(X_i) Diag(beta),
//   X_i = D_i^{-1},  M_ij = X_i A_ij,
// so the solve needs only ten independent 16-row forward substitutions: X_0..X_3 (right-hand
// sides the identity) and the six M_ij (right-hand sides the columns of A_ij).  Half a warp
// takes one of them (lane = column, kept in registers, rows finished in order, each row of
// D_i read as a broadcast; all fp32), two per warp over warps w0..w0+4.  Written as tf32:
// Tb into the T tile (its zero blocks by solve_T_zeros), [M10; M20; M30] and [M21; M31; M32]
// into two 48-row tiles (K = 16 of each 32-wide row used).  MMA corrections then apply the
// M_ij as each U_j becomes final.
__device__ __forceinline__ void solve_T(const float *A, uint8_t *sT, uint8_t *sR2, uint8_t *sR34,
                                        const float *beta, int task2, int lane) {
  // task: 0..3 X_i;  4..9 M_ij in the order (1,0) (2,0) (3,0) (2,1) (3,1) (3,2)
  const int task = 2 * task2 + (lane >> 4), jj = lane & 15;
  constexpr int kI[10] = {0, 1, 2, 3, 1, 2, 3, 2, 3, 3};
  constexpr int kJ[10] = {0, 1, 2, 3, 0, 0, 0, 1, 1, 2};
  int bi = 0, bj = 0;
#pragma unroll
  for (int x = 0; x < 10; ++x)
    if (x == task) {
      bi = kI[x];
      bj = kJ[x];
    }
  const bool is_x = task < 4;
  const int o = 16 * bi;
  // right-hand sides up front (column jj of I or of A_ij); each row of D_i is fetched one
  // step ahead of its use, so the loads stay off the dependent chain
  float rhs[16];
#pragma unroll
  for (int r = 0; r < 16; ++r) rhs[r] = is_x ? (r == jj ? 1.f : 0.f) : A[(o + r) * kAS + 16 * bj + jj];
  float xv[16];
  float4 nx[4];
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    float4 cur[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) cur[q] = nx[q];
    if (r + 1 < 16) {
      const float *row1 = A + (o + r + 1) * kAS + o;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (4 * q < r + 1) nx[q] = *reinterpret_cast<const float4 *>(row1 + 4 * q);
    }
    float acc0 = rhs[r], acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
#pragma unroll
    for (int l4 = 0; l4 < r; l4 += 4) {
      const float4 a = cur[l4 >> 2];
      acc0 = fmaf(-a.x, xv[l4], acc0);
      if (l4 + 1 < r) acc1 = fmaf(-a.y, xv[l4 + 1], acc1);
      if (l4 + 2 < r) acc2 = fmaf(-a.z, xv[l4 + 2], acc2);
      if (l4 + 3 < r) acc3 = fmaf(-a.w, xv[l4 + 3], acc3);
    }
    xv[r] = (acc0 + acc1) + (acc2 + acc3);
  }
  if (is_x) {
    // column o + jj of Tb's diagonal block (the zero blocks: solve_T_zeros)
    const float bj_ = beta[o + jj];
#pragma unroll
    for (int r = 0; r < 16; ++r) st_tf32(sT, sw32(64, o + r, o + jj), xv[r] * bj_);
  } else {
    // row n of R2 = rows of U updated by U_0 (blocks 1..3); R34 = blocks 2, 3 by U_1, 3 by U_2
    uint8_t *tile = bj == 0 ? sR2 : sR34;
    const int base = bj == 0 ? 16 * (bi - 1) : (bj == 1 ? 16 * (bi - 2) : 32);
#pragma unroll
    for (int r = 0; r < 16; ++r) st_tf32(tile, sw32(48, base + r, jj), xv[r]);
  }
}

// The twelve off-diagonal 16 x 16 blocks of Tb are zero: 768 16-byte pieces, six per thread
// of a 128-thread group (t = 0..127), written while other warps run the substitutions.
__device__ __forceinline__ void solve_T_zeros(uint8_t *sT, int t) {
#pragma unroll
  for (int k = 0; k < 6; ++k) {
    const int e = t + 128 * k, r = e / 12, q = e - 12 * (e / 12), rb = r >> 4;
    const int c4 = q < 4 * rb ? q : q + 4;   // 4-column piece, skipping the diagonal block
    *reinterpret_cast<uint4 *>(sT + sw32(64, r, 4 * c4)) = make_uint4(0u, 0u, 0u, 0u);
  }
}

// Packed batches are processed longest first: the sequence whose rank in descending length
// order (ties: lower index first) is `rank`.  Every thread of the block calls this; s_cu is
// shared scratch of n_seqs + 2 ints.  Past kMaxRanked sequences the order is left as given
// (the ranking is O(n^2) per block).  Offsets are only read here; each block checks its own
// sequence's offsets afterwards.
constexpr int kMaxRanked = 1024;
__device__ __forceinline__ int seq_of_length_rank(const int32_t *cu, int n_seqs, int rank,
                                                  int *s_cu) {
  if (n_seqs > kMaxRanked) return rank;
  for (int x = threadIdx.x; x <= n_seqs; x += blockDim.x) s_cu[x] = cu[x];
  if (threadIdx.x == 0) s_cu[n_seqs + 1] = rank;   // (the ranks are a permutation: replaced)
  __syncthreads();
  for (int sq = threadIdx.x; sq < n_seqs; sq += blockDim.x) {
    const long len = (long)s_cu[sq + 1] - s_cu[sq];
    int r = 0;
    for (int x = 0; x < n_seqs; ++x) {
      const long lx = (long)s_cu[x + 1] - s_cu[x];
      r += (lx > len) || (lx == len && x < sq);
    }
    if (r == rank) s_cu[n_seqs + 1] = sq;
  }
  __syncthreads();
  const int sel = s_cu[n_seqs + 1];
  __syncthreads();   // the scratch is reused afterwards
  return sel;
}

// FL: bit 0 per-head gates (CKDA_GATE_PER_HEAD), bit 1 in-kernel q/k normalisation.
// REFS: the kernel that carries per-channel references (launched on the units the plain one
// hands off); the plain kernel keeps every factor relative to the chunk start.
template <typename TOut, int SG, int FL, bool REFS>
__global__ void __launch_bounds__(kThreads, 1)
    chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_a,
                    const __grid_constant__ CUtensorMap tm_o, TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sKQ = sm + OFF_KQ, *sKC = sm + OFF_KC, *sPK = sm + OFF_PK, *sT = sm + OFF_T,
          *sStg = sm + OFF_STG;
  float *sBeta = reinterpret_cast<float *>(sm + OFF_MISC);     // [64]
  float *sGC = sBeta + 64;                                       // [2][128] G_63, double-buffered
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_MISC + 1280);
  // completion (TMA or tcgen05.commit): staging, (1), (a), the steps of (c), (d), all MMAs
  uint64_t *bar_tma = bars, *bar_mma1 = bars + 1, *bar_a = bars + 2, *bar_r = bars + 3,
           *bar_d = bars + 4, *bar_fin = bars + 5;
  // compute warps -> issuer (one arrival per compute warp): a chunk's tiles are ready and
  // it takes the fast path (rdy1) or the token-by-token path (rdy_slow); S is final and
  // TMEM O is free (rdy2); Tm, M, P and V' are ready (rdy3)
  uint64_t *rdy1 = bars + 6, *rdy_slow = bars + 7, *rdy2 = bars + 8, *rdy3 = bars + 9;
  // issuer -> compute warps: a token-by-token announcement has been consumed (so the next
  // announcement cannot be mistaken for it)
  uint64_t *bar_ack = bars + 10;
  // the last correction of (c) is done: the R tiles in Kc's area have been read
  uint64_t *bar_r4 = bars + 11;
  // test hook: a barrier nothing ever arrives on (ckda_debug_wait_injection)
  uint64_t *bar_never = bars + 12;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_MISC + 1392);
  volatile int *sAbort = reinterpret_cast<volatile int *>(sm + OFF_MISC + 1396);
  // staging loads issued so far (by the issuer or compute thread 0); the compute warps count
  // the ones they consumed, so a unit that gives up knows whether one is still in flight
  unsigned int *sTmaIssued = reinterpret_cast<unsigned int *>(sm + OFF_MISC + 1400);
  // length of the chunk being announced (compute warps -> issuer; chunks are cut short where
  // a channel's gate product leaves the factorisation's range)
  volatile int *sLen = reinterpret_cast<volatile int *>(sm + OFF_MISC + 1404);
  // per-head gate logits of the chunk in the gate pass (bf16, CKDA_GATE_PER_HEAD), and
  // 1 / ||q_r||, 1 / ||k_r|| of its rows (CKDA_QK_L2NORM)
  __nv_bfloat16 *sAh = reinterpret_cast<__nv_bfloat16 *>(sm + OFF_MISC + 1408);
  float *sInvQ = reinterpret_cast<float *>(sm + OFF_MISC + 1536);
  float *sInvK = sInvQ + kC;
  constexpr bool per_head = (FL & 1) != 0;
  constexpr bool l2 = (FL & 2) != 0;
  const uint32_t sbase = smem_u32(sm);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = p.H;
  const int unit = blockIdx.x;
  int n, h, mode = 0;
  long t0, t1, bofs;
  const float *s_init = nullptr;   // the state the unit starts from ([dk][dv]; NULL: zero)
  int out_slot = 0;
  auto slot_state = [&](int slot) { return p.slots + ((size_t)slot * H + h) * kD * kD; };
  if constexpr (REFS) {
    // a unit the plain kernel handed off: from its first row on, from the state it saved (this
    // grid may start before the plain one has finished: wait for it, and for its writes)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (unit >= *p.queue_count) return;
    const int4 e = p.queue[unit];
    n = e.x;
    h = e.y;
    t0 = e.z;
    if (p.plan && e.w >= 0) {
      const SegDesc d = p.plan[e.w];
      t1 = d.t1;
      mode = d.mode & ~(kSegInZero | kSegInIdent | kSegInSlot);
      out_slot = d.out_slot;
    } else {
      t1 = p.cu ? p.cu[n + 1] : p.T;
    }
    s_init = p.saved_S + (size_t)unit * kD * kD;
  } else if (p.plan) {
    // an entry of the unit list (offsets were checked by the planner)
    const int di = unit / H;
    if (di >= *p.plan_count) return;
    const SegDesc d = p.plan[di];
    h = unit - di * H;
    n = d.n;
    t0 = d.t0;
    t1 = d.t1;
    mode = d.mode;
    out_slot = d.out_slot;
    if (mode & kSegInSlot) s_init = slot_state(d.in_slot);
    else if (!(mode & (kSegInZero | kSegInIdent)) && p.S0)
      s_init = p.S0 + ((size_t)n * H + h) * kD * kD;
  } else {
    h = unit % H;
    // CTAs start in blockIdx order: in a packed batch the longest sequences go first, so that
    // the units with the longest serial chunk walk do not start last (ranking in the staging
    // buffer, which no load has reached yet)
    n = p.cu ? seq_of_length_rank(p.cu, p.n_seqs, unit / H, reinterpret_cast<int *>(sStg))
             : unit / H;
    if (p.cu) {
      t0 = p.cu[n];
      t1 = p.cu[n + 1];
      if (t0 < 0 || t1 < t0 || t1 > p.T || (n == 0 && t0 != 0) ||
          (n == p.n_seqs - 1 && t1 != p.T)) {
        if (tid == 0) set_status(p.status, CKDA_ERR_SEQLENS);
        return;
      }
    } else {
      t0 = 0;
      t1 = p.T;
    }
    if (p.S0) s_init = p.S0 + ((size_t)n * H + h) * kD * kD;
  }
  bofs = p.cu ? 0 : (long)n * p.T;
  // where the end state goes (NULL: nowhere)
  float *const s_out = (mode & kSegOutSlot) ? slot_state(out_slot)
                       : (!(mode & kSegOutNone) && p.S_T) ? p.S_T + ((size_t)n * H + h) * kD * kD
                                                          : nullptr;
  const bool vzero = (mode & kSegVZero) != 0;   // v = 0 (the v tile is not loaded)
  TOut *o = (mode & kSegNoO) ? nullptr : static_cast<TOut *>(p.o);

  if (tid == 0) {
    for (int x = 0; x < 6; ++x) mbar_init(bars + x, 1);
    for (int x = 6; x < 10; ++x) mbar_init(bars + x, kCompute / 32);
    mbar_init(bar_ack, 1);
    mbar_init(bar_r4, 1);
    mbar_init(bar_never, 1);
    *sAbort = 0;
    *sTmaIssued = 0;
    mbar_fence_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // descriptors of the fixed operand tiles (K-major, 128-byte swizzle)
  const uint64_t dKQ = smem_desc_sw128(sbase + OFF_KQ, 16, 1024);
  const uint64_t dKC = smem_desc_sw128(sbase + OFF_KC, 16, 1024);
  const uint64_t dPK = smem_desc_sw128(sbase + OFF_PK, 16, 1024);
  const uint64_t dT = smem_desc_sw128(sbase + OFF_T, 16, 1024);
  const uint64_t dR2 = smem_desc_sw128(sbase + OFF_R2, 16, 1024);
  const uint64_t dR34 = smem_desc_sw128(sbase + OFF_R34, 16, 1024);
  auto dadd = [](uint64_t d, uint32_t bytes) -> uint64_t { return d + (bytes >> 4); };

  auto issue_tma = [&](long cs) {   // q, k, v and (per-channel gates) a of one chunk
    atomicAdd(sTmaIssued, 1u);
    const int ntens = per_head ? 3 : 4;
    mbar_arrive_expect_tx(bar_tma, (ntens - (vzero ? 1 : 0)) * 2 * 8192);
    const int row = (int)(bofs + cs);
    const CUtensorMap *maps[4] = {&tm_q, &tm_k, &tm_v, &tm_a};
#pragma unroll
    for (int x = 0; x < 4; ++x)
      if (x < ntens && !(x == 2 && vzero)) {
#pragma unroll
        for (int bx = 0; bx < 2; ++bx)
          tma_load_3d(sStg + x * 16384 + bx * 8192, maps[x], bar_tma, bx * 64, h, row);
      }
  };

  // the compute side's staging-load bookkeeping, for the drain at the end
  uint32_t tma_ph_out = 0;
  unsigned int tma_consumed_out = 0;

  if (warp == kCompute / 32) {
    // ================================================================ issuer (one thread)
    // Walks the chunks in order and issues each fast chunk's products as soon as their
    // operands are announced, so that no compute warp ever waits in an MMA issue queue.
    if (lane == 0) {
      uint32_t ph1 = 0, phs = 0, ph2 = 0, ph3 = 0, phr = 0;
      bool ok = true;
      long cs = t0;
      for (int ci = 0; cs < t1 && ok; ++ci) {
        // which path does this chunk take, and how long is it?
        bool fast = false;
        int len = 0;
        {
          const uint64_t w0 = globaltimer();
          for (;;) {
            if (mbar_try_wait_sleep(rdy1, ph1, 2000)) {
              fast = true;
              ph1 ^= 1;
              len = *sLen;
              break;
            }
            if (mbar_try_wait(rdy_slow, phs)) {
              phs ^= 1;
              len = *sLen;   // read before the acknowledgement frees the slot
              mbar_arrive(bar_ack);
              break;
            }
            if (*sAbort || globaltimer() - w0 > kWaitNs) { ok = false; break; }
          }
        }
        if (!ok || len < 0) break;   // len < 0: the unit is handed off
        cs += len;
        if (!fast) continue;
        // (1) [A;P] = [Kr;Qr] Kc^T, and the staging load of the next chunk (staging is
        // free: this chunk's gate pass has consumed it)
        if (cs < t1) issue_tma(cs);
        tc_fence_after();
#pragma unroll
        for (int s = 0; s < 16; ++s) {
          const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
          mma_ss(tmem + COL_AP, dadd(dKQ, off), dadd(dKC, (s >> 2) * 8192 + (s & 3) * 32),
                 IDESC_N64, s > 0);
        }
        mma_commit(bar_mma1);
        // (a) [X^T|O^T] = S^T [Kr;Qr]^T
        if (!(ok = mbar_wait_or_abort(rdy2, ph2, kWaitNs, sAbort))) break;
        ph2 ^= 1;
        tc_fence_after();
#pragma unroll
        for (int s = 0; s < 16; ++s) {
          const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
          mma_ts(tmem + COL_X, tmem + COL_S + 8 * s, dadd(dKQ, off), IDESC_N128, s > 0);
        }
        mma_commit(bar_a);
        // (c) first step: U^T = V'^T Tb^T, hi and lo parts of V'
        if (!(ok = mbar_wait_or_abort(rdy3, ph3, kWaitNs, sAbort))) break;
        ph3 ^= 1;
        const uint32_t vt_cur = (ci & 1) ? COL_VT1 : COL_VT0;
        tc_fence_after();
#pragma unroll
        for (int s = 0; s < 8; ++s)
          mma_ts(tmem + COL_U, tmem + vt_cur + 8 * s, dadd(dT, (s >> 2) * 8192 + (s & 3) * 32),
                 IDESC_N64, s > 0);
#pragma unroll
        for (int s = 0; s < 8; ++s)
          mma_ts(tmem + COL_U, tmem + COL_LO + 8 * s, dadd(dT, (s >> 2) * 8192 + (s & 3) * 32),
                 IDESC_N64, 1);
        mma_commit(bar_r);
        // corrections: U_i -= M_ij U_j for the blocks j = 0, 1, 2 as each becomes final
        // (U_j^T read from TMEM, K = 16)
        if (!(ok = mbar_wait_or_abort(bar_r, phr, kWaitNs, sAbort))) break;
        phr ^= 1;
        tc_fence_after();
#pragma unroll
        for (int s = 0; s < 2; ++s)
          mma_ts(tmem + COL_U + 16, tmem + COL_U + 8 * s, dadd(dR2, s * 32), IDESC_N48_NEG, 1);
        mma_commit(bar_r);
        if (!(ok = mbar_wait_or_abort(bar_r, phr, kWaitNs, sAbort))) break;
        phr ^= 1;
        tc_fence_after();
#pragma unroll
        for (int s = 0; s < 2; ++s)
          mma_ts(tmem + COL_U + 32, tmem + COL_U + 16 + 8 * s, dadd(dR34, s * 32), IDESC_N32_NEG,
                 1);
        mma_commit(bar_r);
        if (!(ok = mbar_wait_or_abort(bar_r, phr, kWaitNs, sAbort))) break;
        phr ^= 1;
        tc_fence_after();
#pragma unroll
        for (int s = 0; s < 2; ++s)
          mma_ts(tmem + COL_U + 48, tmem + COL_U + 32 + 8 * s, dadd(dR34, 4096 + s * 32),
                 IDESC_N16_NEG, 1);
        mma_commit(bar_r);
        mma_commit(bar_r4);
        // (d) [O^T|S^T] += U^T [P;Kc^T]^T
        if (!(ok = mbar_wait_or_abort(bar_r, phr, kWaitNs, sAbort))) break;
        phr ^= 1;
        tc_fence_after();
#pragma unroll
        for (int s = 0; s < 8; ++s)
          mma_ts(tmem + COL_O, tmem + COL_U + 8 * s, dadd(dPK, (s >> 2) * 24576 + (s & 3) * 32),
                 IDESC_N192, 1);
        mma_commit(bar_d);
      }
      if (!ok) *sAbort = 1;
      // every MMA issued above has finished before TMEM is released
      mma_commit(bar_fin);
      mbar_wait(bar_fin, 0, kDrainNs);
    }
    __syncwarp();
  } else {
    // ================================================================ compute warps 0..15
    // Warp w reaches TMEM lanes 32*(w%4)..+31 (jrow); the four warps sharing a lane
    // quarter split each TMEM row's columns (qg = w/4).  The gate pass uses the same
    // mapping: channel c = jrow, rows 16*qg .. 16*qg + 15.
    const int qg = warp >> 2;
    const int jrow = 32 * (warp & 3) + lane;
    const int c = jrow;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
    // phase bits of the barriers the compute warps wait on, packed (registers are the limit)
    enum : int { PH_TMA = 0, PH_MMA1, PH_A, PH_D, PH_ACK, PH_R4, PH_NEVER };
    uint32_t phs = 0;
    unsigned int tma_consumed = 0;   // staging loads whose completion the compute warps saw
    // bf16 O (16 KB per chunk) is staged in T's tile and written by one TMA store;
    // fp32 O is written directly from registers
    constexpr bool kTmaStoreO = sizeof(TOut) == 2;
    bool failed = false, store_pending = false;

    auto csync = [&]() { bar_sync(kBarC, kCompute); };
    // warp 0 polls a completion barrier; the compute warps then agree on the outcome
    // (the phase advances only on success, so after a failure it still names the phase that
    // did not complete)
    auto cwait_for = [&](uint64_t *bar, int bit, uint64_t limit_ns) -> bool {
      bool ok = true;
      if (warp == 0) ok = mbar_wait_or_abort(bar, (phs >> bit) & 1u, limit_ns, sAbort);
      ok = bar_and(kBarC, kCompute, ok);
      if (ok) {
        phs ^= 1u << bit;
        if (bit == PH_TMA) ++tma_consumed;
      }
      return ok;
    };
    auto cwait = [&](uint64_t *bar, int bit) -> bool { return cwait_for(bar, bit, kWaitNs); };
    // one arrival per warp, after the whole warp's writes (each thread fenced its own)
    auto announce = [&](uint64_t *bar) {
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
    };

    const uint8_t *stq = sStg, *stk = sStg + 16384, *stv = sStg + 32768, *sta = sStg + 49152;

    // ---- gate pass: staging (q, k, v, a of one chunk) -> Kr, Qr tiles, V^T in TMEM
    // (columns vcol..vcol+63), beta, G_63.  Kc stays in kc[] until store_kc() writes the Kc
    // and Kc^T tiles, whose previous contents the running chunk may still be reading.
    // Returns whether the chunk is out of range.  Range: for KDA and CKDA every |alpha| <= 1,
    // so |G_t| never grows within the chunk and the last row decides (a NaN gate propagates
    // to it); raw gates are checked at every row.
    float b_next = 0.f;
    if (tid < kC && t0 + tid < t1) b_next = p.b[(size_t)(bofs + t0 + tid) * H + h];
    __nv_bfloat16 a_next = __float2bfloat16_rn(0.f);   // per-head gate logit, a chunk ahead
    if (per_head && tid < kC && t0 + tid < t1) a_next = p.a_head[(size_t)(bofs + t0 + tid) * H + h];
    float kc[16];
    // The gate pass proper works on channel pairs: thread (pair pc = tid % 64, row group
    // rg = tid / 64) takes channels 2pc, 2pc + 1 of rows 8rg .. 8rg + 7, reading bf16 pairs
    // and writing 8-byte pairs.  V^T keeps the one-channel-per-lane mapping TMEM needs.
    const int pc = tid & 63, rg = tid >> 6, ch0 = 2 * pc;
    float *sXp = reinterpret_cast<float *>(sKC);   // [8][128][2] row-group products of the gates
                                                   // and of their inverses (the solve's A is
                                                   // dead whenever a gate pass runs)
    // reference exponents of this thread's two channels in the last decided chunk (0: none)
    int eref0 = 0, eref1 = 0;
    auto gate_pass = [&](int nrows, float *gc_out, uint32_t vcol, float b_this,
                         __nv_bfloat16 a_this, int e0, int e1) -> bool {
      return gate_pass_body<SG, FL, REFS>(sm, tmem, p.signed_gate, nrows, b_this, a_this, gc_out,
                                          vcol, kc, e0, e1);
    };
    // The gate pass of the chunk starting at cs (at most nmax rows) and the chunk's length and
    // path.  The pass first takes each channel's reference from the chunk before (gc_prev,
    // its G_63 / R, and its references; NULL: none), the decay of a channel being much the
    // same from chunk to chunk.  If a channel leaves the range, the references are taken from
    // the chunk's own products and the pass runs again; if a channel decays too fast for any
    // reference, the chunk is cut after its last row group of 8 that fits and the pass runs
    // again on the shorter chunk (rows past the cut become padding); if not even the first
    // group fits, the chunk is its first min(8, rows) rows on the token-by-token path.  Raw
    // gates take no references and send an out-of-range chunk to that path whole.
    int *sTrunc = reinterpret_cast<int *>(sKC + 8192);   // beside the exchange, in the dead A
    // Chunk lengths follow the decay (kernel with references): the fastest channel's decay over
    // the last chunk, in bits (sDecay[parity], a block-wide max), sets the next length to the
    // largest multiple of 8 rows expected to decay by at most kTargetBits, so that a stationary
    // decay needs neither a second pass nor a cut.
    constexpr int kTargetBits = 190;
    int *sDecay = reinterpret_cast<int *>(sm + OFF_MISC + 1384);   // [2]
    int last_rows = kC, dpar = 0;
    auto decide_chunk = [&](long cs, int nmax, float *gc_out, uint32_t vcol, const float *gc_prev,
                            bool &slow_out) -> int {
      const float b_this = b_next;
      const __nv_bfloat16 a_this = a_next;
      if (tid < kC && cs + kC + tid < t1) b_next = p.b[(size_t)(bofs + cs + kC + tid) * H + h];
      if (per_head && tid < kC && cs + kC + tid < t1)
        a_next = p.a_head[(size_t)(bofs + cs + kC + tid) * H + h];
      int rows = nmax;
      bool slow;
      if constexpr (!REFS) {
        slow = bar_or(kBarC, kCompute, gate_pass(rows, gc_out, vcol, b_this, a_this, 0, 0));
      } else {
        // the length from the last chunk's decay, and each channel's reference from its own
        // decay over the last chunk, scaled to the new length
        rows = nmax;
        int e0 = 0, e1 = 0;
        if (gc_prev) {
          const int dmax = sDecay[dpar ^ 1];
          if (dmax > kTargetBits * last_rows / kC) {
            int want = (kTargetBits * last_rows / dmax) & ~7;
            want = want < 8 ? 8 : (want > kC ? kC : want);
            rows = rows < want ? rows : want;
          }
          const float2 gp = *reinterpret_cast<const float2 *>(gc_prev + ch0);
          const int E0 = (int)((__float_as_uint(gp.x) >> 23) & 255u) - 127 + eref0;
          const int E1 = (int)((__float_as_uint(gp.y) >> 23) & 255u) - 127 + eref1;
          e0 = ref_exponent(E0 * rows / last_rows);
          e1 = ref_exponent(E1 * rows / last_rows);
        }
        if (tid == 0) sDecay[dpar] = 0;   // this chunk's slot (read a chunk ago)
        bool cut = false, retried = false;
        if (tid == 0) *sTrunc = kC;   // ordered before any update by the pass's exchange barrier
#pragma unroll 1
        for (;;) {
          slow = bar_or(kBarC, kCompute, gate_pass(rows, gc_out, vcol, b_this, a_this, e0, e1));
          if (!slow || SG == 2) break;
          if (!retried) {
            // references from the chunk's own products; a chunk they do not fit gets cut
            retried = true;
            if (bar_and(kBarC, kCompute, chunk_refs(sXp, ch0, (rows + 7) >> 3, e0, e1))) continue;
          }
          if (cut) break;   // the cut chunk failed again: token by token
          const int fail = first_failing_group(sXp, ch0);
          if (fail < 8) atomicMin(sTrunc, 8 * fail);
          csync();
          const int r = *sTrunc;   // read once per chunk (at most one cut)
          if (r == 0) rows = rows < 8 ? rows : 8;   // the token-by-token path for these rows
          if (r == 0 || r >= rows) break;
          rows = r;   // the cut chunk: its references from its groups, and the pass again
          cut = true;
          chunk_refs(sXp, ch0, r >> 3, e0, e1);
        }
        eref0 = e0;
        eref1 = e1;
        if (!slow && rg == 7) {
          // the decay of this thread's channels over the chunk: the exponent of G_63 / R plus e
          const float2 g = *reinterpret_cast<const float2 *>(gc_out + ch0);
          const int d0 = 127 - (int)((__float_as_uint(g.x) >> 23) & 255u) - e0;
          const int d1 = 127 - (int)((__float_as_uint(g.y) >> 23) & 255u) - e1;
          atomicMax(&sDecay[dpar], d0 > d1 ? d0 : d1);
        }
        last_rows = rows;
        dpar ^= 1;
      }
      if (rows < nmax) {
        // the next chunk starts at the cut: its logits replace the ones fetched a chunk ahead
        if (tid < kC) b_next = cs + rows + tid < t1 ? p.b[(size_t)(bofs + cs + rows + tid) * H + h] : 0.f;
        if (per_head && tid < kC && cs + rows + tid < t1)
          a_next = p.a_head[(size_t)(bofs + cs + rows + tid) * H + h];
      }
      slow_out = slow;
      return rows;
    };
    // The reference R of the chunk just decided (a fast one), per key channel, for the threads
    // that scale the state by it.  Over the 1 / ||q||, 1 / ||k|| factors, which a fast chunk's
    // gate pass has consumed by the time this is written (decide_chunk ends on a barrier) and
    // which are next written by the following chunk's gate pass, after the scaling.  R is
    // applied as a factor of its own: multiplied into G_63 / R of the chunk before, it would
    // fall below fp32's range for a channel decaying by more than about 2^-150 over the two.
    float *sRn = sInvQ;   // [128] (sInvQ and sInvK)
    auto publish_ref = [&]() {
      if (rg == 7) *reinterpret_cast<float2 *>(sRn + ch0) = make_float2(exp2i(eref0), exp2i(eref1));
    };
    auto store_kc_tile = [&]() {  // Kc (row t, channel pair)
#pragma unroll
      for (int rr = 0; rr < 8; ++rr)
        *reinterpret_cast<float2 *>(sKC + sw32(64, 8 * rg + rr, ch0)) =
            make_float2(kc[2 * rr], kc[2 * rr + 1]);
    };
    auto store_kct_tile = [&]() {  // Kc^T (rows 2pc and 2pc + 1, four t per 16-byte store)
      // the first store of a lane takes row 2pc + ((pc >> 2) & 1), the second the other one,
      // so the 32 rows of one store instruction fall on all eight 16-byte bank groups
      const int e0 = (pc >> 2) & 1;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int e = e0 ^ k;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const float x0 = e ? kc[8 * hf + 1] : kc[8 * hf], x1 = e ? kc[8 * hf + 3] : kc[8 * hf + 2];
          const float x2 = e ? kc[8 * hf + 5] : kc[8 * hf + 4], x3 = e ? kc[8 * hf + 7] : kc[8 * hf + 6];
          *reinterpret_cast<float4 *>(sPK + swpk(64 + ch0 + e, 8 * rg + 4 * hf)) =
              make_float4(x0, x1, x2, x3);
        }
      }
    };
    auto store_kc = [&]() {
      store_kc_tile();
      store_kct_tile();
    };
    // tiles of the next chunk written: tell the issuer which path it takes
    auto announce_chunk = [&](bool is_slow) {
      fence_proxy_async();
      tc_fence_before();
      announce(is_slow ? rdy_slow : rdy1);
    };

    // The plain kernel hands a unit whose chunk leaves its range (gates not raw) to the kernel
    // with references, when the caller's workspace has room: the chunk is announced with
    // length -1 (the issuer stops) and the unit saves its state and queues its first row.
    const bool handoff = !REFS && SG != 2 && p.saved_S != nullptr;
    bool handed_off = false;
    auto len_word = [&](int len, bool slow_chunk) { return handoff && slow_chunk ? -1 : len; };

    // ---- initial state into TMEM: thread (lane j, qg) holds S^T[j][32*qg .. +32) = S0[i][j]
    {
      uint32_t r[32];
      const int i0 = 32 * qg;
      const bool ident = (mode & kSegInIdent) != 0;
#pragma unroll
      for (int x = 0; x < 32; ++x)
        r[x] = __float_as_uint(ident    ? (i0 + x == jrow ? 1.f : 0.f)
                               : s_init ? s_init[(size_t)(i0 + x) * kD + jrow]
                                        : 0.f);
      tmem_st32(lane_addr + COL_S + i0, r);
      tmem_wait_st();
    }
    if (vzero) {
      // the v tile is never loaded: zero once (rows past a chunk's end are zeroed anyway)
      for (int e = tid; e < 1024; e += kCompute)
        reinterpret_cast<uint4 *>(sStg + 32768)[e] = make_uint4(0u, 0u, 0u, 0u);
    }
    if (tid == 0 && t1 > t0) issue_tma(t0);
    csync();

    // S^ = Diag(R) S in TMEM for the fast chunk just decided
    auto scale_state_by_ref = [&]() {
      publish_ref();
      csync();
      tc_fence_after();
      uint32_t r[32];
      const int i0 = 32 * qg;
      tmem_ld32(lane_addr + COL_S + i0, r);
      tmem_wait_ld();
#pragma unroll
      for (int x = 0; x < 32; ++x) r[x] = __float_as_uint(__uint_as_float(r[x]) * sRn[i0 + x]);
      tmem_st32(lane_addr + COL_S + i0, r);
      tmem_wait_st();
    };

    // gate pass of the first chunk
    int gsel = 0;              // sGC / V^T buffer of the chunk being processed
    bool slow = false;
    int len = 0;               // rows of the chunk being processed, then of the next one
    if (t1 > t0) {
      if (!cwait(bar_tma, PH_TMA)) {
        failed = true;
      } else {
        len = decide_chunk(t0, (int)(t1 - t0 < kC ? t1 - t0 : kC), sGC, COL_VT0, nullptr, slow);
        store_kc();
        if (REFS && !slow) scale_state_by_ref();
        if (tid == 0) *sLen = len_word(len, slow);
        announce_chunk(slow);
        if (!slow) announce(rdy2);
      }
    }

    long cs = t0, cs_next = t0;
    int len_next = 0;
    for (int ci = 0; cs < t1 && !failed; ++ci, cs = cs_next, len = len_next) {
      const int nrows = len;
      cs_next = cs + nrows;
      const bool has_next = cs_next < t1;
      const int nmax_next = has_next ? (int)(t1 - cs_next < kC ? t1 - cs_next : kC) : 0;
      len_next = 0;
      float *gc_cur = sGC + 128 * gsel, *gc_next = sGC + 128 * (gsel ^ 1);
      const uint32_t vt_cur = gsel ? COL_VT1 : COL_VT0, vt_next = gsel ? COL_VT0 : COL_VT1;

      if (p.inject_chunk >= 0 && ci == p.inject_chunk) {
        // test hook: a wait that runs out (nothing arrives on bar_never)
        if (!cwait_for(bar_never, PH_NEVER, p.inject_wait_ns ? p.inject_wait_ns : kWaitNs)) {
          failed = true;
          break;
        }
      }

      if (slow && handoff) {
        // ------------------------------------------------------------ hand-off: the state (TMEM
        // holds S itself: the plain kernel's factors are relative to the chunk start) and the
        // row the kernel with references resumes at
        int *sSlot = reinterpret_cast<int *>(sKC + 8192);
        if (tid == 0) {
          const int slot = atomicAdd(p.queue_count, 1);
          *sSlot = slot;
          p.queue[slot] = make_int4(n, h, (int)cs, p.plan ? (int)(blockIdx.x / H) : -1);
        }
        csync();
        const int slot = *sSlot;
        tc_fence_after();
        uint32_t r[32];
        const int i0 = 32 * qg;
        tmem_ld32(lane_addr + COL_S + i0, r);
        tmem_wait_ld();
        float *dst = p.saved_S + (size_t)slot * kD * kD;
#pragma unroll
        for (int x = 0; x < 32; ++x) dst[(size_t)(i0 + x) * kD + jrow] = __uint_as_float(r[x]);
        handed_off = true;
        break;
      }
      if (slow) {
        // ------------------------------------------------------------ exact token-by-token path
        // state S[i][j] in smem over Kr/Qr, gates over Kc, partial sums over [P;Kc^T]; thread
        // (value channel jrow, key quarter qg) owns S[32*qg .. +32][jrow]
        float *sS = reinterpret_cast<float *>(sKQ);
        float *sAl = reinterpret_cast<float *>(sKC);
        float *sRed = reinterpret_cast<float *>(sPK);    // [2][4][128]
        if (tid == 0 && store_pending) bulk_wait_read();  // T may still feed an O store
        store_pending = false;
#pragma unroll 4
        for (int rr = 0; rr < 16; ++rr) {
          const int r = 16 * qg + rr;
          sAl[r * kD + c] =
              r < nrows ? gate_alpha(per_head ? __bfloat162float(sAh[r]) : ldbf(sta, r, c), SG)
                        : 1.f;
        }
        tc_fence_after();
        {
          uint32_t r[32];
          const int i0 = 32 * qg;
          tmem_ld32(lane_addr + COL_S + i0, r);
          tmem_wait_ld();
#pragma unroll
          for (int x = 0; x < 32; ++x) sS[(i0 + x) * kD + jrow] = __uint_as_float(r[x]);
        }
        csync();
        for (int t = 0; t < nrows; ++t) {
          const float iqt = l2 ? sInvQ[t] : 1.f, ikt = l2 ? sInvK[t] : 1.f;
          float pk = 0.f;
          for (int x = 0; x < 32; ++x) {
            const int i = 32 * qg + x;
            const float sv = sS[i * kD + jrow] * sAl[t * kD + i];
            sS[i * kD + jrow] = sv;
            pk = fmaf(ldbf(stk, t, i) * ikt, sv, pk);
          }
          sRed[qg * 128 + jrow] = pk;
          csync();
          const float ptot =
              (sRed[jrow] + sRed[128 + jrow]) + (sRed[256 + jrow] + sRed[384 + jrow]);
          const float u = sBeta[t] * (ldbf(stv, t, jrow) - ptot);
          float acc = 0.f;
          for (int x = 0; x < 32; ++x) {
            const int i = 32 * qg + x;
            const float sv = fmaf(ldbf(stk, t, i) * ikt, u, sS[i * kD + jrow]);
            sS[i * kD + jrow] = sv;
            acc = fmaf(ldbf(stq, t, i) * iqt, sv, acc);
          }
          sRed[512 + qg * 128 + jrow] = acc;
          csync();
          if (qg == 0 && o)
            o[((size_t)(bofs + cs + t) * H + h) * kD + jrow] = from_f32<TOut>(
                (sRed[512 + jrow] + sRed[640 + jrow]) + (sRed[768 + jrow] + sRed[896 + jrow]));
        }
        {
          uint32_t r[32];
          const int i0 = 32 * qg;
#pragma unroll
          for (int x = 0; x < 32; ++x) r[x] = __float_as_uint(sS[(i0 + x) * kD + jrow]);
          tmem_st32(lane_addr + COL_S + i0, r);
          tmem_wait_st();
        }
        tc_fence_before();
        csync();
        if (has_next) {
          if (tid == 0) issue_tma(cs_next);
          if (!cwait(bar_tma, PH_TMA)) { failed = true; break; }
          len_next = decide_chunk(cs_next, nmax_next, gc_next, vt_next, nullptr, slow);
          store_kc();
          if (REFS && !slow) scale_state_by_ref();   // this chunk left S unscaled
          if (!cwait(bar_ack, PH_ACK)) { failed = true; break; }   // this chunk's announcement seen
          if (tid == 0) *sLen = len_word(len_next, slow);
          announce_chunk(slow);
          if (!slow) announce(rdy2);
          gsel ^= 1;
        }
        continue;
      }

      // ---------------------------------------------------------------- (1)
      // issued by the issuer once this chunk was announced
      if (tid == 0 && store_pending) bulk_wait_read();  // previous O tile (over T) has left
      store_pending = false;
      if (!cwait(bar_mma1, PH_MMA1)) { failed = true; break; }
      tc_fence_after();
      // ---------------------------------------------------------------- A and P out of TMEM
      float *sA = reinterpret_cast<float *>(sKC);           // plain [64][kAS]
      {
        uint32_t r[16];
        tmem_ld16(lane_addr + COL_AP + 16 * qg, r);
        tmem_wait_ld();
        if (jrow < 64) {
          const int t = jrow;
          const float bt = sBeta[t];
          float av[16];
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            const int j = 16 * qg + x;
            av[x] = j < t ? __uint_as_float(r[x]) * bt : 0.f;
          }
#pragma unroll
          for (int y = 0; y < 4; ++y)
            *reinterpret_cast<float4 *>(sA + t * kAS + 16 * qg + 4 * y) =
                make_float4(av[4 * y], av[4 * y + 1], av[4 * y + 2], av[4 * y + 3]);
        } else {
          // four consecutive columns of row t per 16-byte store (one store per row and
          // 16-byte piece keeps the 32 rows of a warp on distinct bank groups)
          const int t = jrow - 64;
#pragma unroll
          for (int y = 0; y < 4; ++y) {
            uint32_t w4[4];
#pragma unroll
            for (int z = 0; z < 4; ++z) {
              const int x = 4 * y + z, j = 16 * qg + x;
              w4[z] = to_tf32(j <= t ? __uint_as_float(r[x]) : 0.f);
            }
            *reinterpret_cast<uint4 *>(sPK + swpk(t, 16 * qg + 4 * y)) =
                make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
      }
      tc_fence_before();
      csync();
      // ---------------------------------------------------------------- Tm = (I + A)^{-1} Diag(beta)
      // warps 8..12 solve; meanwhile warps 4..7 form (b) V' = V - X once (a) is done, as a
      // round-to-nearest tf32 hi part (over V^T) and the fp32 remainder (over [A;P])
      bool ok = true;
      if (warp >= 4 && warp < 8) {
        ok = mbar_wait_or_abort(bar_a, (phs >> PH_A) & 1u, kWaitNs, sAbort);
        tc_fence_after();
        if (ok) {
#pragma unroll 1
          for (int qt = 0; qt < 4; ++qt) {
            uint32_t xv[16], vv[16];
            tmem_ld16(lane_addr + COL_X + 16 * qt, xv);
            tmem_ld16(lane_addr + vt_cur + 16 * qt, vv);
            tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 16; ++x) {
              const float vp = __uint_as_float(vv[x]) - __uint_as_float(xv[x]);
              const uint32_t hi = to_tf32(vp);
              vv[x] = hi;
              xv[x] = __float_as_uint(vp - __uint_as_float(hi));
            }
            tmem_st16(lane_addr + vt_cur + 16 * qt, vv);
            tmem_st16(lane_addr + COL_LO + 16 * qt, xv);
          }
          tmem_wait_st();
        }
      } else {
        if (warp >= 8 && warp < 13) solve_T(sA, sT, sm + OFF_R2, sm + OFF_R34, sBeta, warp - 8, lane);
        if (warp < 4) solve_T_zeros(sT, tid);
      }
      phs ^= 1u << PH_A;
      fence_proxy_async();
      tc_fence_before();
      if (!bar_and(kBarC, kCompute, ok)) { failed = true; break; }
      announce(rdy3);
      // ---------------------------------------------------------------- next chunk's gate pass,
      // overlapping (c) and (d): Kr, Qr are free ((a) is done); Kc and Kc^T are stored
      // after (d)
      if (has_next) {
        if (!cwait(bar_tma, PH_TMA)) { failed = true; break; }
        len_next = decide_chunk(cs_next, nmax_next, gc_next, vt_next, gc_cur, slow);
        if (REFS && !slow) publish_ref();   // for this chunk's end-of-chunk scaling
      }
      // the next chunk's Kc tile once (c) is done with the R tiles; then (1) of the next
      // chunk can run under this chunk's (d) and read-out.  Kc^T waits for (d).
      if (!cwait(bar_r4, PH_R4)) { failed = true; break; }
      if (has_next) {
        store_kc_tile();
        if (tid == 0) *sLen = len_word(len_next, slow);
        announce_chunk(slow);
      }
      if (!cwait(bar_d, PH_D)) { failed = true; break; }
      tc_fence_after();
      if (has_next) store_kct_tile();
      // ---------------------------------------------------------------- O out; S^T columns scaled by G_63
      {
        uint32_t r[32];
        tmem_ld16(lane_addr + COL_O + 16 * qg, *reinterpret_cast<uint32_t(*)[16]>(r));
        tmem_wait_ld();
        if (kTmaStoreO && o && nrows == kC) {
          // full chunk: O [t][j] staged over T, written by one TMA store
          TOut *sO = reinterpret_cast<TOut *>(sT);
#pragma unroll
          for (int x = 0; x < 16; ++x)
            sO[(16 * qg + x) * kD + jrow] = from_f32<TOut>(__uint_as_float(r[x]));
        } else if (o) {
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            const int t = 16 * qg + x;
            if (t < nrows)
              o[((size_t)(bofs + cs + t) * H + h) * kD + jrow] =
                  from_f32<TOut>(__uint_as_float(r[x]));
          }
        }
        const int i0 = 32 * qg;
        tmem_ld32(lane_addr + COL_S + i0, r);
        tmem_wait_ld();
        // S' = (G_63 / R) S^, then S^ for the next chunk = R' S' (R' = 1 if it is token by
        // token or there is none)
        const bool rnext = REFS && has_next && !slow;
#pragma unroll
        for (int x = 0; x < 32; x += 4) {
          const float4 gv = *reinterpret_cast<const float4 *>(gc_cur + i0 + x);
          float4 rv = make_float4(1.f, 1.f, 1.f, 1.f);
          if (rnext) rv = *reinterpret_cast<const float4 *>(sRn + i0 + x);
          r[x] = __float_as_uint(__uint_as_float(r[x]) * gv.x * rv.x);
          r[x + 1] = __float_as_uint(__uint_as_float(r[x + 1]) * gv.y * rv.y);
          r[x + 2] = __float_as_uint(__uint_as_float(r[x + 2]) * gv.z * rv.z);
          r[x + 3] = __float_as_uint(__uint_as_float(r[x + 3]) * gv.w * rv.w);
        }
        tmem_st32(lane_addr + COL_S + i0, r);
        tmem_wait_st();
      }
      fence_proxy_async();
      tc_fence_before();
      if (has_next && !slow) announce(rdy2);   // S final, TMEM O free: (a) may run
      csync();
      if (kTmaStoreO && tid == 0 && o && nrows == kC) {
        tma_store_3d(&tm_o, sT, 0, h, (int)(bofs + cs));
        bulk_commit();
        store_pending = true;
      }
      gsel ^= 1;
    }
    if (tid == 0) bulk_wait_all();

    tma_ph_out = phs & 1u;
    tma_consumed_out = tma_consumed;
    if (failed) {
      if (tid == 0) {
        set_status(p.status, CKDA_ERR_TIMEOUT);
        *sAbort = 1;   // the issuer leaves its loop at its next wait
      }
    } else if (s_out && !handed_off) {
      tc_fence_after();
      uint32_t r[32];
      const int i0 = 32 * qg;
      tmem_ld32(lane_addr + COL_S + i0, r);
      tmem_wait_ld();
#pragma unroll
      for (int x = 0; x < 32; ++x) s_out[(size_t)(i0 + x) * kD + jrow] = __uint_as_float(r[x]);
    }
  }
  tc_fence_before();
  __syncthreads();
  // Both sides have left their loops, so no further staging load can be issued.  A load the
  // compute warps did not consume (a unit that gave up) must land before the CTA's shared
  // memory is released; at most one is ever in flight, on the phase tma_ph names.  The issuer
  // has already waited for its last products (bar_fin).
  if (tid == 0 && *sTmaIssued != tma_consumed_out) mbar_wait(bar_tma, tma_ph_out, kDrainNs);
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  // the plain kernel's work is done: the launch of the kernel with references (programmatic
  // dependent launch) may start once every CTA got here; it waits for this grid's completion
  // before it reads the queue
  if constexpr (!REFS) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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

// The workspace (tc_workspace_layout): the 256-byte header (status word; at byte 64 the count
// of handed-off units; at kSegHeaderOffset the plan's header), the hand-off queue and saved
// states, and for a planned call the two unit lists and the cut sequences' state slots.
constexpr size_t kQueueCountOffset = 64;

int sm_count() {
  int dev = 0, P = kSegAssumedSMs;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&P, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || P <= 0)
    P = kSegAssumedSMs;
  return P;
}

template <typename TOut, int SG, int FL>
int launch_typed(const ChunkArgs &g, cudaStream_t stream) {
  const long rows = (long)g.B * g.T;
  CUtensorMap mq, mk, mv, ma, mo;
  const long map_rows = rows > 0 ? rows : 1;
  const bool per_head = per_head_gate(g.signed_gate);   // a is [rows, H]: no tile map
  memset(&ma, 0, sizeof(ma));
  if (!make_map(&mq, g.q, g.H, map_rows) || !make_map(&mk, g.k, g.H, map_rows) ||
      !make_map(&mv, g.v, g.H, map_rows) || (!per_head && !make_map(&ma, g.a, g.H, map_rows)))
    return CKDA_ERR_CUDA;
  memset(&mo, 0, sizeof(mo));
  if (g.o && !make_out_map(&mo, g.o, g.H, map_rows, g.o_dtype == CKDA_BF16)) return CKDA_ERR_CUDA;
  TcParams p;
  p.b = g.b; p.S0 = g.S0; p.cu = g.cu_seqlens; p.o = g.o; p.S_T = g.S_T; p.status = g.status;
  p.n_seqs = g.n_seqs; p.T = g.T; p.H = g.H; p.signed_gate = g.signed_gate;
  p.inject_chunk = g.inject_chunk;
  p.inject_wait_ns = g.inject_wait_ns;
  p.a_head = per_head ? static_cast<const __nv_bfloat16 *>(g.a) : nullptr;
  p.plan = nullptr;
  p.plan_count = nullptr;
  p.slots = nullptr;

  // plan (cut the longest sequences) when the cost model may gain and the workspace has room
  const bool packed = g.cu_seqlens != nullptr;
  const int P = sm_count();
  const bool want_plan = g.n_seqs <= kSegMaxSeqs &&
                         (g.force_split > 0 ? packed : tc_plans(packed, g.B, g.T, g.H, g.n_seqs, P));
  TcWorkspace L = tc_workspace_layout(g.n_seqs, g.H, true);
  const bool plan = want_plan && g.workspace && g.workspace_bytes >= L.total;
  if (!plan) L = tc_workspace_layout(g.n_seqs, g.H, false);
  const bool handoff = SG != 2 && g.workspace && g.workspace_bytes >= L.total;
  uint8_t *ws = static_cast<uint8_t *>(g.workspace);
  p.queue_count = handoff ? reinterpret_cast<int *>(ws + kQueueCountOffset) : nullptr;
  p.queue = handoff ? reinterpret_cast<int4 *>(ws + L.queue_off) : nullptr;
  p.saved_S = handoff ? reinterpret_cast<float *>(ws + L.saved_off) : nullptr;

  auto kern = chunk_tc_kernel<TOut, SG, FL, false>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes) !=
      cudaSuccess)
    return CKDA_ERR_CUDA;
  // one launch of the plain kernel over `units` CTAs, then (hand-off) the kernel with references
  // on the units it queued
  auto run = [&](long units) -> int {
    kern<<<(unsigned)units, kThreads, kSmemBytes, stream>>>(mq, mk, mv, ma, mo, p);
    if (cudaGetLastError() != cudaSuccess) return CKDA_ERR_CUDA;
    if constexpr (SG != 2) {
      if (handoff) {
        // CTAs past the queue's count return at once
        auto kern_r = chunk_tc_kernel<TOut, SG, FL, true>;
        if (cudaFuncSetAttribute(kern_r, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kSmemBytes) != cudaSuccess)
          return CKDA_ERR_CUDA;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)units);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = kSmemBytes;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // launch early
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, kern_r, mq, mk, mv, ma, mo, p) != cudaSuccess)
          return CKDA_ERR_CUDA;
      }
    }
    return CKDA_OK;
  };
  if (!plan) return run((long)g.n_seqs * g.H);

  SegHeader *hdr = reinterpret_cast<SegHeader *>(ws + kSegHeaderOffset);
  SegDesc *d1 = reinterpret_cast<SegDesc *>(ws + L.desc_off), *d3 = d1 + L.max_desc;
  p.slots = reinterpret_cast<float *>(ws + L.slot_off);
  int rc = launch_seg_plan(g.cu_seqlens, g.n_seqs, g.T, g.H, P, g.force_split, g.force_nseg, hdr,
                           d1, d3, g.status, stream);
  if (rc != CKDA_OK) return rc;
  p.plan = d1;
  p.plan_count = &hdr->n1;
  if ((rc = run((long)L.max_desc * g.H)) != CKDA_OK) return rc;
  if ((rc = launch_seg_combine(hdr, p.slots, p.queue_count, g.H, stream)) != CKDA_OK) return rc;
  p.plan = d3;
  p.plan_count = &hdr->n3;
  return run((long)L.max_desc * g.H);
}

}  // namespace

bool chunk_tc_supported(const ChunkArgs &g) {
  return g.dk == kD && g.dv == kD && g.chunk == kC && g.io_dtype == CKDA_BF16 &&
         g.B * (long)g.T > 0 && !delta_product2(g.signed_gate);
}

int launch_chunk_tc(const ChunkArgs &g, cudaStream_t s) {
  if (g.n_seqs * g.H == 0) return CKDA_OK;
  const bool bf = g.o_dtype == CKDA_BF16;
  // the kernel is specialised on the gate's form and the flags; the strength's form is read
  // at run time
  const int fl = (per_head_gate(g.signed_gate) ? 1 : 0) | (qk_l2norm(g.signed_gate) ? 2 : 0);
  switch (alpha_form(g.signed_gate) * 4 + fl) {
#define CKDA_TC_CASE(SGV, FLV)                                                     \
  case SGV * 4 + FLV:                                                             \
    return bf ? launch_typed<__nv_bfloat16, SGV, FLV>(g, s) : launch_typed<float, SGV, FLV>(g, s);
    CKDA_TC_CASE(0, 0) CKDA_TC_CASE(0, 1) CKDA_TC_CASE(0, 2) CKDA_TC_CASE(0, 3)
    CKDA_TC_CASE(1, 0) CKDA_TC_CASE(1, 1) CKDA_TC_CASE(1, 2) CKDA_TC_CASE(1, 3)
    CKDA_TC_CASE(2, 0) CKDA_TC_CASE(2, 1) CKDA_TC_CASE(2, 2) CKDA_TC_CASE(2, 3)
#undef CKDA_TC_CASE
  }
  return CKDA_ERR_DTYPE;
}

}  // namespace ckda

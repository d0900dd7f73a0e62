// segments.cu -- the unit plan of the tensor-core prefill: cutting the longest sequences of a
// batch into segments that run in two launches, and the state combination between them.
//
// The recurrence (CKDA review, section "Diagonal-plus-rank-one (DPR1) transition")
//   S_t = (I - b_t k_t k_t^T) Diag(alpha_t) S_{t-1} + b_t k_t v_t^T
// is affine in S, so over a segment S_end = A S_in + B with A the ordered product of the
// segment's transitions and B the end state from S_in = 0.  A is the end state of the same
// walk from S_in = I with every v_t = 0, so both come out of the ordinary chunk kernel.  The
// plan (internal.h) runs the cut sequences' segments from 0 and from I in the first launch, the
// chain X_s <- Y_s X_{s-1} + X_s here, and the segments again from their true starting states
// in the second launch; the other sequences fill the two launches.
#include "common.cuh"
#include "internal.h"

namespace ckda {
namespace {

constexpr int kD = 128;                 // dk = dv of the tensor-core path
constexpr int kRows = 64;               // rows per chunk
constexpr int kPlanThreads = 1024;      // = kSegMaxSeqs: one thread per sequence
static_assert(kPlanThreads >= kSegMaxSeqs, "one planner thread per sequence");

size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }

// One CTA.  Thread x owns sequence x: its offsets are checked (a bad sequence records
// CKDA_ERR_SEQLENS and gets no unit), it is ranked by length (descending, ties by index), and it
// writes its own unit list entry.  The first kSegCandidates threads evaluate one candidate cut
// each; thread 0 picks one and writes the cut sequences' entries and the header.
__global__ void __launch_bounds__(kPlanThreads, 1)
    seg_plan_kernel(const int32_t *cu, int n_seqs, int T, int H, int P, int force_k, int force_m,
                    SegHeader *hdr, SegDesc *d1, SegDesc *d3, int *status) {
  __shared__ int s_len[kSegMaxSeqs];     // by sequence; -1: bad offsets
  __shared__ int s_t0[kSegMaxSeqs];      // by sequence
  __shared__ int s_seq[kSegMaxSeqs];     // by rank
  __shared__ int s_ch[kSegMaxSeqs];      // chunks, by rank
  __shared__ unsigned long long s_W;
  __shared__ int s_nv, s_n1short;
  __shared__ SegChoice s_c, s_cand[kSegCandidates];
  __shared__ bool s_valid[kSegCandidates];
  __shared__ long long s_cap1;
  const int tid = threadIdx.x;
  const bool packed = cu != nullptr;
  if (tid == 0) {
    s_W = 0;
    s_nv = 0;
    s_n1short = 0;
  }
  int len = -1, t0 = 0;
  if (tid < n_seqs) {
    if (packed) {
      const int a = cu[tid], b = cu[tid + 1];
      const bool bad = a < 0 || b < a || b > T || (tid == 0 && a != 0) ||
                       (tid == n_seqs - 1 && b != T);
      if (bad) set_status(status, CKDA_ERR_SEQLENS);
      else len = b - a;
      t0 = a;
    } else {
      len = T;
    }
    s_len[tid] = len;
    s_t0[tid] = t0;
  }
  __syncthreads();
  int rank = -1, ch = 0;
  if (tid < n_seqs && len >= 0) {
    int r = 0;
    for (int x = 0; x < n_seqs; ++x) {
      const int lx = s_len[x];
      r += (lx > len) || (lx == len && x < tid);
    }
    rank = r;
    ch = (len + kRows - 1) / kRows;
    s_seq[r] = tid;
    s_ch[r] = ch;
    atomicAdd(&s_nv, 1);
    atomicAdd(&s_W, (unsigned long long)ch * (unsigned long long)H);
  }
  __syncthreads();
  // the cost model's candidates, one per thread
  {
    const int nv = s_nv;
    int top[kSegMaxSplit + 1];
    for (int i = 0; i <= kSegMaxSplit; ++i) top[i] = i < nv ? s_ch[i] : 0;
    if (tid < kSegCandidates) {
      const long est0 = seg_est0(top, nv, (long)s_W, P);
      const bool forced = force_k > 0;
      int k, nseg;
      seg_candidate_of(tid, k, nseg);
      SegChoice c = {};
      s_valid[tid] = k <= nv && (!forced || (k == force_k && nseg == force_m)) &&
                     seg_candidate(top, nv, (long)s_W, H, P, k, nseg, forced, est0, c);
      s_cand[tid] = c;
    }
  }
  __syncthreads();
  if (tid == 0) {
    const int nv = s_nv;
    int top[kSegMaxSplit + 1];
    for (int i = 0; i <= kSegMaxSplit; ++i) top[i] = i < nv ? s_ch[i] : 0;
    const SegChoice c = seg_pick(s_cand, s_valid, seg_est0(top, nv, (long)s_W, P), force_k > 0);
    // the first launch's spare capacity (chunk times x SMs) for the uncut sequences: the two
    // launches split the estimated walk in proportion to the cut sequences' waves in each
    long long cap1 = 0x7FFFFFFFFFFFFFFFLL;
    if (c.k > 0) {
      long long load1 = 0;
      for (int i = 0; i < c.k; ++i) load1 += (long long)H * c.seg[i] * (2 * c.m[i] - 3);
      const long long chain = (long long)c.seg[0] * (c.w1 + c.w3);
      const long long t1 = (long long)c.seg[0] * c.w1 + (c.est > chain ? (c.est - chain) / 2 : 0);
      cap1 = (long long)P * t1 - load1;
      if (cap1 < 0) cap1 = 0;
    }
    s_c = c;
    s_cap1 = cap1;
  }
  __syncthreads();
  const SegChoice c = s_c;
  const int nv = s_nv;
  // cut sequences' entries: first launch X_0, X_s, Y_s; second launch segments 1 .. m-1
  int nxy = 0, nsg = 0;
  for (int i = 0; i < c.k; ++i) {
    nxy += 2 * c.m[i] - 3;
    nsg += c.m[i] - 1;
  }
  // uncut sequences in rank order: a prefix of them (by cumulative work) to the first launch
  bool first = false;
  if (rank >= c.k) {
    long long pre = 0;
    for (int x = c.k; x <= rank; ++x) pre += (long long)H * s_ch[x];
    first = pre <= s_cap1;
    if (first) atomicAdd(&s_n1short, 1);
  }
  __syncthreads();
  const int n1short = s_n1short;
  if (rank >= c.k) {
    SegDesc d;
    d.t0 = packed ? s_t0[tid] : 0;
    d.t1 = d.t0 + len;
    d.n = tid;
    d.mode = 0;
    d.in_slot = d.out_slot = d.pad0 = d.pad1 = 0;
    if (first) d1[nxy + (rank - c.k)] = d;
    else d3[nsg + (rank - c.k - n1short)] = d;
  }
  if (tid == 0) {
    int e1 = 0, e3 = 0;
    for (int i = 0; i < c.k; ++i) {
      const int n = s_seq[i];
      const int a = packed ? s_t0[n] : 0, b = a + s_len[n];
      const int m = c.m[i], rows = c.seg[i] * kRows, base = i * kSegSlotsPerSplit;
      SegDesc d;
      d.n = n;
      d.in_slot = d.out_slot = d.pad0 = d.pad1 = 0;
      // X_0: the true walk of segment 0 (o written), its end state to slot 0
      d.t0 = a;
      d.t1 = a + rows;
      d.mode = kSegOutSlot;
      d.out_slot = base;
      d1[e1++] = d;
      for (int s = 1; s <= m - 2; ++s) {
        d.t0 = a + s * rows;
        d.t1 = d.t0 + rows;
        d.mode = kSegInZero | kSegOutSlot | kSegNoO;   // X_s = B_s
        d.out_slot = base + s;
        d1[e1++] = d;
        d.mode = kSegInIdent | kSegVZero | kSegOutSlot | kSegNoO;   // Y_s = A_s
        d.out_slot = base + (m - 1) + (s - 1);
        d1[e1++] = d;
      }
      // the second launch: segment s from X_{s-1}; the last one writes S_T
      d.out_slot = 0;
      for (int s = 1; s <= m - 1; ++s) {
        d.t0 = a + s * rows;
        d.t1 = s == m - 1 ? b : d.t0 + rows;
        d.mode = kSegInSlot | (s == m - 1 ? 0 : kSegOutNone);
        d.in_slot = base + s - 1;
        d3[e3++] = d;
      }
      hdr->split[i].m = m;
      hdr->split[i].seg_rows = rows;
      hdr->split[i].slot_base = base;
      hdr->split[i].pad = 0;
    }
    hdr->n1 = nxy + n1short;
    hdr->n3 = nsg + (nv - c.k - n1short);
    hdr->nsplit = c.k;
    hdr->pad = 0;
  }
}

// The chain between the launches: X_s <- Y_s X_{s-1} + X_s for s = 1 .. m-2 in fp32 (states
// [dk][dv] row-major; Y_s is [dk][dk]).  Column blocks of X are independent through the whole
// chain, so CTA (cut sequence i, head h, block cb) owns the 32 columns 32 cb .. 32 cb + 31 of
// every X_s; thread (ty, tx) owns the 4 x 4 block at rows 4 ty, columns 4 tx of it.  CTA 0 also
// clears the hand-off queue's count for the second launch (the first launch's units with
// references have finished).
constexpr int kCombThreads = 256;
constexpr int kCombCols = 32;                 // columns of X per CTA
constexpr int kCombBlocks = kD / kCombCols;   // CTAs per (cut sequence, head)
constexpr int kATStride = kD + 4;             // floats per row of A^T in shared memory
constexpr size_t kCombSmem = (size_t)(kD * kATStride + kD * kCombCols) * sizeof(float);

__global__ void __launch_bounds__(kCombThreads, 1)
    seg_combine_kernel(const SegHeader *hdr, float *slots, int *queue_count, int H) {
  extern __shared__ float4 comb_smem4[];
  float *sAT = reinterpret_cast<float *>(comb_smem4);   // [k][i] = A[i][k]
  float *sS = sAT + kD * kATStride;                      // [k][j] = S_in[k][32 cb + j]
  if (blockIdx.x == 0 && threadIdx.x == 0 && queue_count) *queue_count = 0;
  const int cb = blockIdx.x % kCombBlocks, ih = blockIdx.x / kCombBlocks;
  const int i = ih / H, h = ih - (ih / H) * H;
  if (i >= hdr->nsplit) return;
  const SegSplit sp = hdr->split[i];
  const int tid = threadIdx.x, ty = tid >> 3, tx = tid & 7;
  auto slot = [&](int j) { return slots + ((size_t)(sp.slot_base + j) * H + h) * kD * kD; };
  for (int s = 1; s <= sp.m - 2; ++s) {
    const float *A = slot(sp.m - 1 + s - 1);
    const float *Sin = slot(s - 1) + kCombCols * cb;
    float *X = slot(s) + kCombCols * cb;
    for (int e = tid; e < kD * kD; e += kCombThreads) {
      const int r = e >> 7, cc = e & (kD - 1);
      sAT[cc * kATStride + r] = A[e];
    }
    for (int e = tid; e < kD * kCombCols; e += kCombThreads) {
      const int r = e / kCombCols, cc = e % kCombCols;
      sS[e] = Sin[(size_t)r * kD + cc];
    }
    __syncthreads();
    float acc[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[r][q] = 0.f;
#pragma unroll 4
    for (int kk = 0; kk < kD; ++kk) {
      const float4 a = *reinterpret_cast<const float4 *>(sAT + kk * kATStride + 4 * ty);
      const float4 b = *reinterpret_cast<const float4 *>(sS + kk * kCombCols + 4 * tx);
      const float av[4] = {a.x, a.y, a.z, a.w};
      const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[r][q] = fmaf(av[r], bv[q], acc[r][q]);
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      float4 *row = reinterpret_cast<float4 *>(X + (size_t)(4 * ty + r) * kD + 4 * tx);
      float4 x = *row;
      x.x += acc[r][0];
      x.y += acc[r][1];
      x.z += acc[r][2];
      x.w += acc[r][3];
      *row = x;
    }
    __syncthreads();   // this block of X_s is the next step's S_in block; the tiles are restaged
  }
}

}  // namespace

TcWorkspace tc_workspace_layout(int n_seqs, int H, bool plan) {
  TcWorkspace w;
  w.max_desc = plan ? n_seqs + kSegMaxSplit * kSegSlotsPerSplit : 0;
  w.units = (long)(plan ? w.max_desc : n_seqs) * H;
  const size_t state = (size_t)kD * kD * sizeof(float);
  w.queue_off = kWorkspaceHeader;
  w.saved_off = w.queue_off + round256((size_t)w.units * 16);
  w.desc_off = w.saved_off + (size_t)w.units * state;
  w.slot_off = w.desc_off + round256((size_t)2 * w.max_desc * sizeof(SegDesc));
  w.total = plan ? w.slot_off + (size_t)kSegMaxSplit * kSegSlotsPerSplit * H * state : w.desc_off;
  return w;
}

bool tc_plans(bool packed, int B, int T, int H, int n_seqs, int P) {
  if (packed) return n_seqs > 0 && n_seqs <= kSegMaxSeqs;
  if (B <= 0 || B > kSegMaxSeqs || T <= 0) return false;
  const int c = (T + kRows - 1) / kRows;
  int top[kSegMaxSplit + 1];
  for (int i = 0; i <= kSegMaxSplit; ++i) top[i] = i < B ? c : 0;
  return seg_choose(top, B, (long)B * H * c, H, P, 0, 0).k > 0;
}

int launch_seg_plan(const int32_t *cu, int n_seqs, int T, int H, int P, int force_k, int force_m,
                    SegHeader *hdr, SegDesc *d1, SegDesc *d3, int *status, cudaStream_t s) {
  if (n_seqs <= 0 || n_seqs > kSegMaxSeqs) return CKDA_ERR_DIM;
  seg_plan_kernel<<<1, kPlanThreads, 0, s>>>(cu, n_seqs, T, H, P, force_k, force_m, hdr, d1, d3,
                                             status);
  return cudaGetLastError() == cudaSuccess ? CKDA_OK : CKDA_ERR_CUDA;
}

int launch_seg_combine(const SegHeader *hdr, float *slots, int *queue_count, int H,
                       cudaStream_t s) {
  if (cudaFuncSetAttribute(seg_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kCombSmem) != cudaSuccess)
    return CKDA_ERR_CUDA;
  seg_combine_kernel<<<kSegMaxSplit * H * kCombBlocks, kCombThreads, kCombSmem, s>>>(
      hdr, slots, queue_count, H);
  return cudaGetLastError() == cudaSuccess ? CKDA_OK : CKDA_ERR_CUDA;
}

}  // namespace ckda

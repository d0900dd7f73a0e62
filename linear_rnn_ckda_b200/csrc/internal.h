// internal.h -- launch interface between the C ABI (ckda_abi.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <math.h>
#include <stddef.h>
#include <stdint.h>

namespace ckda {

struct ChunkArgs {
  const void *q, *k, *v, *a;
  const float *b;
  const float *S0;
  const int32_t *cu_seqlens;  // device, or NULL
  void *o;                    // may be NULL
  float *S_T;                 // may be NULL
  int n_seqs;                 // N (sequences)
  int B, T, H, dk, dv, chunk, signed_gate, io_dtype, o_dtype;
  int *status;                // device status word (workspace)
  void *workspace;            // whole workspace (status word first)
  size_t workspace_bytes;
  // test hook (ckda_debug_wait_injection): chunk index at which every unit of the
  // tensor-core kernel waits on a barrier nothing arrives on (-1: off), and that wait's bound
  int inject_chunk;
  unsigned long long inject_wait_ns;
  // test hook (ckda_debug_segment_split): cut the force_split longest sequences into
  // force_nseg segments whatever the cost model says (0: the cost model decides)
  int force_split, force_nseg;
};

// ---------------------------------------------------------------- segment plan (tensor-core path)
// A sequence's chunk walk is serial, so a batch whose longest sequence holds far more chunks than
// the batch's work per SM is bound by that one walk.  The state map of a segment of the
// recurrence is affine in the state it starts from: S_end = A S_in + B, A the product of the
// segment's transitions (the end state from S_in = I with v = 0) and B the end state from
// S_in = 0.  A long sequence cut into segments 0 .. m-1 then runs in two launches:
//   first:   X_0 = segment 0 from the caller's S0 (o written); for s = 1 .. m-2 X_s from 0 and
//            Y_s from I with v = 0 (o not written);
//   combine: X_s <- Y_s X_{s-1} + X_s for s = 1 .. m-2 (X_s: the state entering segment s + 1);
//   second:  segments 1 .. m-1 from X_{s-1}, o written, the last one writes S_T.
// Every other sequence runs whole in one of the two launches, chosen to balance them.
constexpr int kSegMaxSplit = 2;                       // sequences cut at most
constexpr int kSegMaxSeg = 8;                         // segments per cut sequence at most
constexpr int kSegSlotsPerSplit = 2 * kSegMaxSeg - 3; // X_0 .. X_{m-2}, Y_1 .. Y_{m-2}
constexpr int kSegMinChunks = 48;                     // shorter sequences are never cut
constexpr int kSegMaxSeqs = 1024;                     // larger packed batches are not planned
constexpr int kSegAssumedSMs = 148;                   // SM count the workspace size assumes

// one unit list entry: rows [t0, t1) of sequence n (packed rows, or rows of batch row n), run
// for every head; states in slots are [slot][H][dk][dv]
struct SegDesc {
  int t0, t1, n, mode, in_slot, out_slot, pad0, pad1;
};
enum : int {
  kSegInZero = 1,    // start from S = 0 (else the caller's S0)
  kSegInIdent = 2,   // start from S = I
  kSegInSlot = 4,    // start from slot in_slot
  kSegOutSlot = 8,   // end state to slot out_slot (else the caller's S_T)
  kSegOutNone = 16,  // end state not written
  kSegVZero = 32,    // v = 0
  kSegNoO = 64,      // o not written
};
struct SegSplit {
  int m, seg_rows, slot_base, pad;
};
// in the workspace header at byte kSegHeaderOffset
struct SegHeader {
  int n1, n3, nsplit, pad;
  SegSplit split[kSegMaxSplit];
};
constexpr size_t kSegHeaderOffset = 128;

// The cost model: given the chunk counts of the longest sequences (top[0] >= top[1] >= ...,
// min(nv, kSegMaxSplit + 1) of them), the batch's total chunk count over all heads W, H and
// the SM count P, how many sequences to cut (k, 0: none) and into how many segments each (m[i]
// of seg[i] chunks), and the estimated walk (in chunk times) with and without the cut.
struct SegChoice {
  int k;
  int m[kSegMaxSplit], seg[kSegMaxSplit];
  long est, est0;
  int w1, w3;   // waves of the cut sequences' units in the first and second launch
};
// Divisions by the SM count go through fp32 (an estimate; the same IEEE operations on the host
// and the device, so both take the same decision) and chunk counts are 32-bit: 64-bit integer
// division is a long software sequence on the device.
__host__ __device__ inline long seg_per_sm(long work, int P) {
  return (long)ceilf((float)work / (float)P);
}
// the estimated walk without a cut
__host__ __device__ inline long seg_est0(const int *top, int nv, long W, int P) {
  if (nv <= 0) return 0;
  const long w = seg_per_sm(W, P);
  return top[0] > w ? (long)top[0] : w;
}
// One candidate: the k longest sequences each cut into (up to) nseg segments.  Returns whether
// it is possible (forced: whatever the length, but every cut sequence needs three segments).
__host__ __device__ inline bool seg_candidate(const int *top, int nv, long W, int H, int P, int k,
                                              int nseg, bool forced, long est0, SegChoice &c) {
  c.k = k;
  c.est0 = est0;
  int U1 = 0, U3 = 0;
  long extra = 0;
  for (int i = 0; i < k; ++i) {
    const int ch = top[i];
    if (!forced && ch < kSegMinChunks) return false;
    const int L = ch > 0 ? (ch + nseg - 1) / nseg : 1;
    const int mm = (ch + L - 1) / L;
    if (mm < 3) return false;
    c.m[i] = mm;
    c.seg[i] = L;
    U1 += H * (2 * mm - 3);
    U3 += H * (mm - 1);
    extra += (long)H * L * (2 * mm - 4);
  }
  const long L0 = c.seg[0];
  c.w1 = (U1 + P - 1) / P;
  c.w3 = (U3 + P - 1) / P;
  long chain = L0 * (c.w1 + c.w3);
  if (k < nv) {
    const long wsmall = c.w1 < c.w3 ? c.w1 : c.w3;
    const long alt = L0 * wsmall + (long)top[k];
    if (alt > chain) chain = alt;
  }
  const long work = seg_per_sm(W + extra, P);
  c.est = chain > work ? chain : work;
  return true;
}
constexpr int kSegCandidates = kSegMaxSplit * (kSegMaxSeg - 2);   // (k, nseg) pairs
__host__ __device__ inline void seg_candidate_of(int idx, int &k, int &nseg) {
  k = 1 + idx / (kSegMaxSeg - 2);
  nseg = 3 + idx % (kSegMaxSeg - 2);
}
// The choice among evaluated candidates (valid[x]: candidate x is possible), in candidate order
// (k, then nseg, ascending; the first of equal estimates): a cut costs two more launches and up
// to twice the work of the cut sequences, so it is taken only for a clear gain (or when forced).
__host__ __device__ inline SegChoice seg_pick(const SegChoice *cand, const bool *valid, long est0,
                                              bool forced) {
  SegChoice best;
  best.k = 0;
  best.w1 = best.w3 = 0;
  best.est = best.est0 = est0;
  for (int x = 0; x < kSegCandidates; ++x)
    if (valid[x] && (forced || cand[x].est < best.est)) best = cand[x];
  if (!forced && best.k > 0 && best.est * 10 > est0 * 9) best.k = 0;
  return best;
}
// The whole cost model, one candidate after the other (the planner kernel evaluates them in
// parallel).
__host__ __device__ inline SegChoice seg_choose(const int *top, int nv, long W, int H, int P,
                                                int force_k, int force_m) {
  const long est0 = seg_est0(top, nv, W, P);
  const bool forced = force_k > 0;
  SegChoice cand[kSegCandidates];
  bool valid[kSegCandidates];
  for (int x = 0; x < kSegCandidates; ++x) {
    int k, nseg;
    seg_candidate_of(x, k, nseg);
    valid[x] = k <= nv && (!forced || (k == force_k && nseg == force_m)) &&
               seg_candidate(top, nv, W, H, P, k, nseg, forced, est0, cand[x]);
  }
  return seg_pick(cand, valid, est0, forced);
}

// Workspace of the tensor-core path: the header, the hand-off queue and saved states for
// `units` units, and (plan) the unit lists and the cut sequences' state slots.
struct TcWorkspace {
  size_t queue_off, saved_off, desc_off, slot_off, total;
  long units;      // hand-off capacity (units of one launch)
  int max_desc;    // entries of each unit list
};
TcWorkspace tc_workspace_layout(int n_seqs, int H, bool plan);
// Whether the tensor-core path plans a batch of these sizes (packed: always, up to kSegMaxSeqs
// sequences; otherwise when the cost model cuts at kSegAssumedSMs SMs) and the workspace bytes
// it then uses.
bool tc_plans(bool packed, int B, int T, int H, int n_seqs, int P);
// The unit planner (one CTA) and the state combination between the two launches.
int launch_seg_plan(const int32_t *cu, int n_seqs, int T, int H, int P, int force_k, int force_m,
                    SegHeader *hdr, SegDesc *d1, SegDesc *d3, int *status, cudaStream_t s);
int launch_seg_combine(const SegHeader *hdr, float *slots, int *queue_count, int H,
                       cudaStream_t s);

struct DecodeArgs {
  const void *q, *k, *v, *a;
  const float *b;
  float *S;
  void *o;
  int B, H, dk, dv, signed_gate, io_dtype, o_dtype;
};

// Argument checks of ckda_chunk_fwd that need no device (everything but the workspace):
// CKDA_OK or the CKDA_ERR_* code the call returns.
int check_chunk_args(const void *q, const void *k, const void *v, const void *a, const float *b,
                     const float *S0, const int32_t *cu_seqlens, int n_seqs, int B, int T, int H,
                     int dk, int dv, int chunk, int signed_gate, int io_dtype, int o_dtype,
                     const void *o, const float *S_T);

// Exact fp32 SIMT chunkwise forward (any dk, dv, chunk).  Returns a CKDA_* code.
int launch_chunk_simt(const ChunkArgs &args, cudaStream_t stream);

// Tensor-core chunkwise forward (tcgen05, dk = dv = 128, chunk 64, bf16 io).
bool chunk_tc_supported(const ChunkArgs &args);
int launch_chunk_tc(const ChunkArgs &args, cudaStream_t stream);

// First chunk slot of sequence n when chunks of C tokens of every sequence are numbered in one
// array (the backward's saved states): cu[n] / C + n for a packed batch (consecutive sequences
// never overlap: the next base is at least ceil(len / C) further), n * ceil(T / C) otherwise.
__host__ __device__ __forceinline__ long chunk_slot_base(const int32_t *cu, int n, long T, int C) {
  return cu ? (long)cu[n] / C + n : (long)n * ((T + C - 1) / C);
}
// Number of chunk slots per head: an upper bound of the last base plus its chunks.
__host__ __device__ __forceinline__ long chunk_slots(bool packed, int B, long T, int N, int C) {
  return packed ? T / C + N + 1 : (long)B * ((T + C - 1) / C);
}

// Chunkwise backward (exact fp32, CUDA cores): gradients of sum dO . o + sum dS_T . S_T.
struct BwdArgs {
  const void *q, *k, *v, *a;
  const float *b, *S0, *dS_T;
  const int32_t *cu_seqlens;
  const void *dO;             // may be NULL (zero)
  float *gq, *gk, *gv, *ga, *gb, *gS0;   // gS0 may be NULL
  float *S_chunks, *dS_chunks;           // workspace: [n_slots][H][dk][dv] each
  float *rec;                            // workspace: [n_slots][H][bwd_record_floats]
  int *status;
  int n_seqs, B, T, H, dk, dv, signed_gate, io_dtype, do_dtype;
  long n_slots;
};
int launch_chunk_bwd(const BwdArgs &args, cudaStream_t stream);
// Floats of one (chunk slot, head) record of the backward: the chunk's state-independent
// factors Kr, Kd, Qr ([C][dk] each), Li, P, M ([C][C] each), beta [C] and g [dk], rounded up
// to 16 bytes.
__host__ __device__ __forceinline__ long bwd_record_floats(int C, int dk) {
  return (3L * C * dk + 3L * C * C + C + dk + 3) & ~3L;
}
int bwd_chunk_rows();   // the backward's chunk size (its saved states are every this many rows)

// One decode step.  Returns a CKDA_* code.
int launch_decode(const DecodeArgs &args, cudaStream_t stream);

// Bytes of the workspace header (status word and counters).
constexpr size_t kWorkspaceHeader = 256;

}  // namespace ckda

// internal.h -- launch interface between the C ABI (ckda_abi.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
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
};

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
// Workspace bytes that let the tensor-core kernel hand units whose gates decay past its range to
// its variant with per-channel references (the header, a queue and one saved state per unit);
// with less, such chunks run token by token.
size_t chunk_tc_handoff_bytes(int n_seqs, int H);
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

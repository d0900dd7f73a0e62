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
int launch_chunk_tc(const ChunkArgs &args, cudaStream_t stream);

// One decode step.  Returns a CKDA_* code.
int launch_decode(const DecodeArgs &args, cudaStream_t stream);

// Bytes of the workspace header (status word and counters).
constexpr size_t kWorkspaceHeader = 256;

}  // namespace ckda

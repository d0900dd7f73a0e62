// noalloc.cu -- ckda_chunk_fwd for callers that cannot allocate device memory.
//
// ckda_chunk_fwd asks its caller for a small device workspace (the status
// word and counters the kernels use).  Some callers have no way to provide
// one: a serving runtime that plans every byte of device memory when it starts
// and refuses any allocation afterwards, or plain C code that links only this
// library and has no device allocator of its own.  This entry point serves
// them from a fixed scratch array that lives in the library's own device
// image, so neither the caller nor the library calls cudaMalloc.
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/ckda.h"
#include "internal.h"

namespace {

// Upper bound of the scratch this entry point can offer.  Every GPU that
// loads the library keeps this array resident until the process exits.
constexpr size_t kNoAllocScratchBytes = 4096;
static_assert(kNoAllocScratchBytes >= ckda::kWorkspaceHeader, "scratch smaller than the header");

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array on the current device.  Looked up on every call: the
// lookup is cheap once the library's module is loaded on the device, and a cached address
// would go stale if the module were unloaded and loaded again (after cudaDeviceReset, for
// example).  The host-side name of the array is only a stand-in, not a device address.
int scratch_for_current_device(void **out) {
  void *ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return CKDA_ERR_CUDA;
  *out = ptr;
  return CKDA_OK;
}

}  // namespace

extern "C" int ckda_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const void *a,
                                      const float *b, const float *S0, const int32_t *cu_seqlens,
                                      int n_seqs, int B, int T, int H, int dk, int dv, int chunk,
                                      int signed_gate, int io_dtype, int o_dtype, void *o,
                                      float *S_T, void *stream) {
  // the arguments are checked before any CUDA call, as ckda_chunk_fwd does
  const int arg_rc = ckda::check_chunk_args(q, k, v, a, b, S0, cu_seqlens, n_seqs, B, T, H, dk, dv,
                                            chunk, signed_gate, io_dtype, o_dtype, o, S_T);
  if (arg_rc != CKDA_OK) return arg_rc;
  void *scratch = nullptr;
  const int rc = scratch_for_current_device(&scratch);
  if (rc != CKDA_OK) return rc;
  // ckda_chunk_fwd clears the status header of the scratch on `stream` before
  // its kernels run, so nothing a previous call left behind leaks into this one.
  return ckda_chunk_fwd(q, k, v, a, b, S0, cu_seqlens, n_seqs, B, T, H, dk, dv, chunk, signed_gate,
                        io_dtype, o_dtype, o, S_T, scratch, kNoAllocScratchBytes, stream);
}

extern "C" int ckda_noalloc_status(int *status, void *stream) {
  if (!status) return CKDA_ERR_NULL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int host = 0;
  // offset 0 of the scratch is the status word the kernels write (the workspace header)
  if (cudaMemcpyFromSymbolAsync(&host, g_noalloc_scratch, sizeof(int), 0, cudaMemcpyDeviceToHost,
                                s) != cudaSuccess)
    return CKDA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return CKDA_ERR_CUDA;
  *status = host;
  return CKDA_OK;
}

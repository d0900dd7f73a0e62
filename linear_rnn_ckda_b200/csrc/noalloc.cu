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
#include <mutex>

#include "../../include/ckda.h"
#include "internal.h"

namespace {

// Upper bound of the scratch this entry point can offer.  Every GPU that
// loads the library keeps this array resident until the process exits.
constexpr size_t kNoAllocScratchBytes = 4096;
static_assert(kNoAllocScratchBytes >= ckda::kWorkspaceHeader, "scratch smaller than the header");

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once
// per device; the host-side name of the array is not a device address).
int scratch_for_current_device(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CKDA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev]) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return CKDA_ERR_CUDA;
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return CKDA_OK;
}

}  // namespace

extern "C" int ckda_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const void *a,
                                      const float *b, const float *S0, const int32_t *cu_seqlens,
                                      int n_seqs, int B, int T, int H, int dk, int dv, int chunk,
                                      int signed_gate, int io_dtype, int o_dtype, void *o,
                                      float *S_T, void *stream) {
  const size_t need = ckda_chunk_fwd_workspace_size(B, T, H, dk, dv, chunk, n_seqs);
  if (need > kNoAllocScratchBytes) return CKDA_ERR_WORKSPACE;
  void *scratch = nullptr;
  const int rc = scratch_for_current_device(&scratch);
  if (rc != CKDA_OK) return rc;
  // ckda_chunk_fwd clears the status header of the scratch on `stream` before
  // its kernels run, so nothing a previous call left behind leaks into this one.
  return ckda_chunk_fwd(q, k, v, a, b, S0, cu_seqlens, n_seqs, B, T, H, dk, dv, chunk, signed_gate,
                        io_dtype, o_dtype, o, S_T, scratch, kNoAllocScratchBytes, stream);
}

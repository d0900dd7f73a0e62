// ckda_abi.cu -- host side of the C ABI declared in include/ckda.h:
// argument validation, device check, workspace layout and kernel dispatch.
// Nothing here allocates device memory or synchronises (except the explicit
// status read-back, which says so).
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cstdint>
#include <cstring>

#include "../../include/ckda.h"
#include "internal.h"

namespace {

bool valid_dim(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }
bool aligned(const void *p, uintptr_t n) {
  return p == nullptr || (reinterpret_cast<uintptr_t>(p) & (n - 1)) == 0;
}
bool aligned16(const void *p) { return aligned(p, 16); }
// a gate form 0..4, optionally with CKDA_GATE_PER_HEAD, CKDA_QK_L2NORM, CKDA_DELTA_PRODUCT2
bool valid_gate(int sg) {
  return sg >= 0 && (sg & 15) <= 4 &&
         (sg & ~(15 | CKDA_GATE_PER_HEAD | CKDA_QK_L2NORM | CKDA_DELTA_PRODUCT2)) == 0;
}

// sm_100 check for the current device, cached per device (atomics: host threads may call the
// library concurrently; the cached value is the same whoever writes it).
int check_device() {
  static std::atomic<int> cached[64];  // 0 unknown, 1 ok, -1 not sm_100
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return CKDA_ERR_CUDA;
  const int known = dev >= 0 && dev < 64 ? cached[dev].load(std::memory_order_relaxed) : 0;
  if (known != 0) return known > 0 ? CKDA_OK : CKDA_ERR_DEVICE;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return CKDA_ERR_CUDA;
  const bool ok = (major == 10 && minor == 0);
  if (dev >= 0 && dev < 64) cached[dev].store(ok ? 1 : -1, std::memory_order_relaxed);
  return ok ? CKDA_OK : CKDA_ERR_DEVICE;
}

// ckda_debug_wait_injection's settings (process-wide, read at each launch)
std::atomic<int> g_inject_chunk{-1};
std::atomic<unsigned long long> g_inject_wait_ns{0};
// ckda_debug_segment_split's settings (process-wide, read at each launch)
std::atomic<int> g_force_split{0};
std::atomic<int> g_force_nseg{0};

// The cost model's choice for a packed batch of these lengths (what the planner decides).
ckda::SegChoice seg_choice_for_lengths(const int32_t *lengths, int n, int H, int P) {
  // the planner's view: chunk counts in descending order, their sum over all heads
  int top[ckda::kSegMaxSplit + 1] = {};
  long W = 0;
  for (int x = 0; x < n; ++x) {
    const int ch = lengths[x] > 0 ? (lengths[x] + 63) / 64 : 0;   // chunks of 64 rows
    W += (long)ch * H;
    for (int i = 0; i <= ckda::kSegMaxSplit; ++i)
      if (ch > top[i]) {
        for (int j = ckda::kSegMaxSplit; j > i; --j) top[j] = top[j - 1];
        top[i] = ch;
        break;
      }
  }
  return ckda::seg_choose(top, n, W, H, P, 0, 0);
}


}  // namespace

namespace ckda {

int check_chunk_args(const void *q, const void *k, const void *v, const void *a, const float *b,
                     const float *S0, const int32_t *cu_seqlens, int n_seqs, int B, int T, int H,
                     int dk, int dv, int chunk, int signed_gate, int io_dtype, int o_dtype,
                     const void *o, const float *S_T) {
  if (!q || !k || !v || !a || !b) return CKDA_ERR_NULL;
  if (!valid_dim(dk) || !valid_dim(dv) || B < 0 || T < 0 || H <= 0) return CKDA_ERR_DIM;
  if (chunk != 16 && chunk != 32 && chunk != 64) return CKDA_ERR_CHUNK;
  if (!valid_gate(signed_gate) || (io_dtype != CKDA_F32 && io_dtype != CKDA_BF16) ||
      (o_dtype != CKDA_F32 && o_dtype != CKDA_BF16))
    return CKDA_ERR_DTYPE;
  if (cu_seqlens && (B != 1 || n_seqs < 0)) return CKDA_ERR_DIM;
  // token rows are 32-bit coordinates in the kernels (TMA tile coordinates included); a
  // DeltaProduct2 token is two rows
  const long long rows = (long long)B * T * ((signed_gate & CKDA_DELTA_PRODUCT2) ? 2 : 1);
  if (rows > (long long)INT32_MAX || rows * H > (1LL << 41)) return CKDA_ERR_DIM;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(a) || !aligned(b, 4) ||
      !aligned16(S0) || !aligned16(o) || !aligned16(S_T) || !aligned(cu_seqlens, 4))
    return CKDA_ERR_ALIGN;
  return CKDA_OK;
}

}  // namespace ckda

extern "C" {

void ckda_debug_wait_injection(int chunk_index, unsigned long long wait_ns) {
  g_inject_wait_ns.store(wait_ns, std::memory_order_relaxed);
  g_inject_chunk.store(chunk_index < 0 ? -1 : chunk_index, std::memory_order_relaxed);
}

int ckda_debug_segment_choice(const int32_t *lengths, int n_seqs, int H, int sm_count,
                              int *n_cut, int *segments) {
  if (!lengths || !n_cut || !segments) return CKDA_ERR_NULL;
  if (n_seqs < 0 || n_seqs > ckda::kSegMaxSeqs || H <= 0 || sm_count <= 0) return CKDA_ERR_DIM;
  for (int x = 0; x < n_seqs; ++x)
    if (lengths[x] < 0) return CKDA_ERR_DIM;
  const ckda::SegChoice c = seg_choice_for_lengths(lengths, n_seqs, H, sm_count);
  *n_cut = c.k;
  for (int i = 0; i < ckda::kSegMaxSplit; ++i) segments[i] = i < c.k ? c.m[i] : 0;
  return CKDA_OK;
}

void ckda_debug_segment_split(int n_split, int n_segments) {
  const bool on = n_split > 0 && n_split <= ckda::kSegMaxSplit && n_segments >= 3 &&
                  n_segments <= ckda::kSegMaxSeg;
  g_force_nseg.store(on ? n_segments : 0, std::memory_order_relaxed);
  g_force_split.store(on ? n_split : 0, std::memory_order_relaxed);
}

const char *ckda_status_string(int status) {
  switch (status) {
    case CKDA_OK: return "ok";
    case CKDA_ERR_NULL: return "a required pointer is NULL";
    case CKDA_ERR_DIM: return "unsupported dimension (dk, dv must be 16, 32, 64 or 128; B, T, H, n_seqs valid)";
    case CKDA_ERR_CHUNK: return "unsupported chunk size (16, 32 or 64)";
    case CKDA_ERR_DTYPE: return "unsupported dtype code or signed_gate value";
    case CKDA_ERR_ALIGN: return "a pointer is not aligned as its argument requires";
    case CKDA_ERR_SEQLENS: return "invalid cu_seqlens offsets";
    case CKDA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case CKDA_ERR_TIMEOUT: return "a bounded device wait timed out";
    case CKDA_ERR_CUDA: return "CUDA runtime error";
    case CKDA_ERR_DEVICE: return "current device is not an sm_100 (B200-class) GPU";
  }
  return "unknown status";
}

int ckda_version(void) { return 100; }

size_t ckda_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv, int chunk, int n_seqs) {
  const bool packed = n_seqs > 0;
  const int N = packed ? n_seqs : B;
  if (dk == 128 && dv == 128 && chunk == 64 && N > 0 && H > 0) {
    const bool plan = ckda::tc_plans(packed, B, T, H, N, ckda::kSegAssumedSMs);
    return std::max(ckda::kWorkspaceHeader, ckda::tc_workspace_layout(N, H, plan).total);
  }
  return ckda::kWorkspaceHeader;
}

int ckda_chunk_fwd(const void *q, const void *k, const void *v, const void *a, const float *b,
                   const float *S0, const int32_t *cu_seqlens, int n_seqs, int B, int T, int H,
                   int dk, int dv, int chunk, int signed_gate, int io_dtype, int o_dtype,
                   void *o, float *S_T, void *workspace, size_t workspace_bytes, void *stream) {
  const int arg_rc = ckda::check_chunk_args(q, k, v, a, b, S0, cu_seqlens, n_seqs, B, T, H, dk, dv,
                                            chunk, signed_gate, io_dtype, o_dtype, o, S_T);
  if (arg_rc != CKDA_OK) return arg_rc;
  const int N = cu_seqlens ? n_seqs : B;
  // the header is the minimum; ckda_chunk_fwd_workspace_size() bytes also let fast-decaying
  // gates stay on the tensor cores
  if (!workspace || workspace_bytes < ckda::kWorkspaceHeader ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return CKDA_ERR_WORKSPACE;
  const int dev_rc = check_device();
  if (dev_rc != CKDA_OK) return dev_rc;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(workspace, 0, ckda::kWorkspaceHeader, s) != cudaSuccess) return CKDA_ERR_CUDA;
  ckda::ChunkArgs g;
  g.q = q; g.k = k; g.v = v; g.a = a; g.b = b; g.S0 = S0; g.cu_seqlens = cu_seqlens;
  g.o = o; g.S_T = S_T; g.n_seqs = N; g.B = B; g.T = T; g.H = H; g.dk = dk; g.dv = dv;
  g.chunk = chunk; g.signed_gate = signed_gate; g.io_dtype = io_dtype; g.o_dtype = o_dtype;
  g.status = static_cast<int *>(workspace);
  g.workspace = workspace;
  g.workspace_bytes = workspace_bytes;
  g.inject_chunk = g_inject_chunk.load(std::memory_order_relaxed);
  g.inject_wait_ns = g_inject_wait_ns.load(std::memory_order_relaxed);
  g.force_split = g_force_split.load(std::memory_order_relaxed);
  g.force_nseg = g_force_nseg.load(std::memory_order_relaxed);
  if (ckda::chunk_tc_supported(g)) return ckda::launch_chunk_tc(g, s);
  return ckda::launch_chunk_simt(g, s);
}

size_t ckda_chunk_bwd_workspace_size(int B, int T, int H, int dk, int dv, int n_seqs) {
  if (B < 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0 || n_seqs < 0) return ckda::kWorkspaceHeader;
  const bool packed = n_seqs > 0;
  const long slots = ckda::chunk_slots(packed, packed ? 1 : B, (long)(packed ? T : T),
                                       packed ? n_seqs : B, ckda::bwd_chunk_rows());
  const size_t per_slot_head = 2 * (size_t)dk * dv + ckda::bwd_record_floats(ckda::bwd_chunk_rows(), dk);
  return ckda::kWorkspaceHeader + (size_t)slots * H * per_slot_head * sizeof(float);
}

int ckda_chunk_bwd(const void *q, const void *k, const void *v, const void *a, const float *b,
                   const float *S0, const int32_t *cu_seqlens, int n_seqs, int B, int T, int H,
                   int dk, int dv, int signed_gate, int io_dtype, const void *dO, int do_dtype,
                   const float *dS_T, float *dq, float *dk_out, float *dv_out, float *da,
                   float *db, float *dS0, void *workspace, size_t workspace_bytes, void *stream) {
  const int arg_rc = ckda::check_chunk_args(q, k, v, a, b, S0, cu_seqlens, n_seqs, B, T, H, dk, dv,
                                            16, signed_gate, io_dtype, CKDA_F32, nullptr, nullptr);
  if (arg_rc != CKDA_OK) return arg_rc;
  if (!dq || !dk_out || !dv_out || !da || !db) return CKDA_ERR_NULL;
  if (do_dtype != CKDA_F32 && do_dtype != CKDA_BF16) return CKDA_ERR_DTYPE;
  if (signed_gate & CKDA_DELTA_PRODUCT2) return CKDA_ERR_DTYPE;   // forward only
  if (!aligned16(dO) || !aligned16(dS_T) || !aligned16(dq) || !aligned16(dk_out) ||
      !aligned16(dv_out) || !aligned16(da) || !aligned(db, 4) || !aligned16(dS0))
    return CKDA_ERR_ALIGN;
  const int N = cu_seqlens ? n_seqs : B;
  const size_t need = ckda_chunk_bwd_workspace_size(B, T, H, dk, dv, cu_seqlens ? n_seqs : 0);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return CKDA_ERR_WORKSPACE;
  const int dev_rc = check_device();
  if (dev_rc != CKDA_OK) return dev_rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(workspace, 0, ckda::kWorkspaceHeader, s) != cudaSuccess) return CKDA_ERR_CUDA;
  const long slots = ckda::chunk_slots(cu_seqlens != nullptr, cu_seqlens ? 1 : B, T, N,
                                       ckda::bwd_chunk_rows());
  float *base = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + ckda::kWorkspaceHeader);
  ckda::BwdArgs g;
  g.q = q; g.k = k; g.v = v; g.a = a; g.b = b; g.S0 = S0; g.dS_T = dS_T; g.cu_seqlens = cu_seqlens;
  g.dO = dO; g.gq = dq; g.gk = dk_out; g.gv = dv_out; g.ga = da; g.gb = db; g.gS0 = dS0;
  g.S_chunks = base;
  g.dS_chunks = base + (size_t)slots * H * dk * dv;
  g.rec = base + 2 * (size_t)slots * H * dk * dv;
  g.status = static_cast<int *>(workspace);
  g.n_seqs = N; g.B = B; g.T = T; g.H = H; g.dk = dk; g.dv = dv; g.signed_gate = signed_gate;
  g.io_dtype = io_dtype; g.do_dtype = do_dtype; g.n_slots = slots;
  return ckda::launch_chunk_bwd(g, s);
}

int ckda_decode_step(const void *q, const void *k, const void *v, const void *a, const float *b,
                     float *S, int B, int H, int dk, int dv, int signed_gate, int io_dtype,
                     int o_dtype, void *o, void *stream) {
  if (!q || !k || !v || !a || !b || !S) return CKDA_ERR_NULL;
  if (!valid_dim(dk) || !valid_dim(dv) || B < 0 || H <= 0) return CKDA_ERR_DIM;
  if ((long long)B * H > (1LL << 31) - 1) return CKDA_ERR_DIM;
  if (!valid_gate(signed_gate) || (io_dtype != CKDA_F32 && io_dtype != CKDA_BF16) ||
      (o_dtype != CKDA_F32 && o_dtype != CKDA_BF16))
    return CKDA_ERR_DTYPE;
  const uintptr_t in_sz = io_dtype == CKDA_BF16 ? 2 : 4, out_sz = o_dtype == CKDA_BF16 ? 2 : 4;
  if (!aligned(q, in_sz) || !aligned(k, in_sz) || !aligned(v, in_sz) || !aligned(a, in_sz) ||
      !aligned(b, 4) || !aligned16(S) || !aligned(o, out_sz))
    return CKDA_ERR_ALIGN;
  const int dev_rc = check_device();
  if (dev_rc != CKDA_OK) return dev_rc;
  ckda::DecodeArgs g;
  g.q = q; g.k = k; g.v = v; g.a = a; g.b = b; g.S = S; g.o = o;
  g.B = B; g.H = H; g.dk = dk; g.dv = dv; g.signed_gate = signed_gate;
  g.io_dtype = io_dtype; g.o_dtype = o_dtype;
  return ckda::launch_decode(g, static_cast<cudaStream_t>(stream));
}

int ckda_workspace_status(const void *workspace, int *status, void *stream) {
  if (!workspace || !status) return CKDA_ERR_NULL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int host = 0;
  if (cudaMemcpyAsync(&host, workspace, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return CKDA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return CKDA_ERR_CUDA;
  *status = host;
  return CKDA_OK;
}

}  // extern "C"

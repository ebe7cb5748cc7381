// attn_noalloc.cu -- sparse attention forward that allocates nothing.
//
// For callers that cannot allocate device memory (a plugin handed only its
// inputs and outputs; a serving loop that must not call cudaMalloc after start-
// up, since it can synchronise the device).  The split partials of decode-shaped
// calls live in one file-scope device array instead of a caller workspace.
#include <cstdio>
#include <mutex>

#include "lsa_common.cuh"
#include "lsa_internal.h"

namespace {

// Built-in scratch for split partials; every device that loads the library
// holds it until the process exits.  Shared by all calls (see lsa.h).
static __device__ __align__(256) float g_attn_scratch[LSA_NOALLOC_SCRATCH_BYTES / sizeof(float)];

constexpr int kMaxDevices = 128;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_attn_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device (with that device current) and reused.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_attn_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" int lsa_sparse_attn_noalloc(const void* Q, int32_t T, int32_t Hq, const void* K, const void* V,
                                       int32_t n_heads, int64_t n_cap, int32_t d, int32_t dtype,
                                       const int32_t* idx, int32_t K_sel, const int32_t* q_pos,
                                       int32_t causal, int64_t tail_begin, int64_t tail_end, float scale,
                                       void* O, float* LSE, int32_t* status, void* stream) {
  // A call without queries launches nothing; lsa_sparse_attn validates the
  // rest of its arguments and returns.
  if (T == 0)
    return lsa_sparse_attn(Q, T, Hq, K, V, n_heads, n_cap, d, dtype, idx, K_sel, q_pos, causal, tail_begin,
                           tail_end, scale, O, LSE, nullptr, 0, status, stream);
  const int64_t tail_len = tail_end >= tail_begin ? tail_end - tail_begin : -1;
  size_t need = 0;
  int rc = lsa_attn_workspace_bytes(T, Hq, n_heads, d, K_sel, tail_len, &need);
  if (rc != LSA_OK) return rc;
  if (need > LSA_NOALLOC_SCRATCH_BYTES) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "lsa_sparse_attn_noalloc: this call needs %zu bytes of split scratch but the built-in array "
             "holds %u bytes; split the queries over several calls or use lsa_sparse_attn",
             need, (unsigned)LSA_NOALLOC_SCRATCH_BYTES);
    return lsa::report_error(LSA_ERR_WORKSPACE, msg);
  }
  void* scratch = nullptr;
  if (need > 0) {
    cudaError_t e = scratch_address(&scratch);
    if (e != cudaSuccess) {
      char msg[256];
      snprintf(msg, sizeof(msg), "lsa_sparse_attn_noalloc: device scratch lookup failed: %s", cudaGetErrorString(e));
      return lsa::report_error(LSA_ERR_CUDA, msg);
    }
  }
  return lsa_sparse_attn(Q, T, Hq, K, V, n_heads, n_cap, d, dtype, idx, K_sel, q_pos, causal, tail_begin,
                         tail_end, scale, O, LSE, scratch, need > 0 ? (size_t)LSA_NOALLOC_SCRATCH_BYTES : 0,
                         status, stream);
}

// noalloc.cu — an allocation-free variant of the forward entry point.
//
// Some callers cannot hand the library a workspace: a plugin that a host
// framework gives only its input and output buffers (the framework owns the
// device memory pool and forbids raw cudaMalloc), or a latency-critical loop
// that must not call cudaMalloc/cudaFree because they can synchronise the
// device.  For them, qlora_linear_fwd_noalloc runs the same forward as
// qlora_linear_fwd with its scratch in a fixed array of device memory that the
// library declares statically: every GPU that loads the library holds
// kNoAllocScratchBytes of it until the process exits.
#include <mutex>

#include "kernels.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB per device

// The forward's workspace (split-K partial sums of X A^T, the bf16 hi/lo
// copy of s*U and, for small M, the split-K partials of Y).  Every call
// overwrites what it reads, so nothing here has to start at zero.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the array on the current device.  In host code the name
// g_noalloc_scratch is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
qlora_status scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return QLORA_ERR_CUDA;
  std::lock_guard<std::mutex> g(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return QLORA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return QLORA_OK;
}

}  // namespace

extern "C" {

qlora_status qlora_linear_fwd_noalloc(const uint16_t* X, int64_t M, nf4_weight W, const uint16_t* A,
                                      const uint16_t* B, int32_t r, float s, void* Y, int32_t y_dtype,
                                      float* U_out, int32_t* d_status, void* stream) {
  // The same checks, in the same order, as qlora_linear_fwd; then, in place
  // of its workspace check, the problem must fit the fixed scratch.  Nothing
  // is enqueued when a check fails.
  if (qlora_status st = qnf4::check_fwd_args(X, X, M, W, A, B, r, Y, y_dtype, U_out, d_status)) return st;
  if (M == 0) return QLORA_OK;
  if (qlora_fwd_workspace_size(M, W.n_out, W.k_in, r) > kNoAllocScratchBytes) return QLORA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (qlora_status st = scratch_for_current_device(&scratch)) return st;
  return qlora_linear_fwd(X, M, W, A, B, r, s, Y, y_dtype, U_out, scratch, kNoAllocScratchBytes, d_status,
                          stream);
}

}  // extern "C"

// The materialise-then-top-k path with its scratch in a fixed device array, for
// callers that cannot allocate device memory (see more_route_unfused_static in
// more_route.h).  It runs the same three kernels as more_route_unfused.
#include <mutex>

#include "more_internal.cuh"

namespace more {
namespace {

// Scratch of more_route_unfused_static: z (fp32 N x r) and the logits (fp32 N x M).
// It lives in the module for as long as the library is loaded, on every device
// that loads it, and is shared by all calls.
static __device__ __align__(256) unsigned char g_static_scratch[MORE_STATIC_SCRATCH_BYTES];

// Device address of g_static_scratch on the current device, looked up once per device and
// kept for the life of the process (a device reset invalidates it; see more_route.h).
void* static_scratch_address(cudaError_t* err) {
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= 64) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    *err = cudaGetSymbolAddress(&p, g_static_scratch);
    if (*err != cudaSuccess) return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace
}  // namespace more

extern "C" more_status more_route_unfused_static(const void* X, const void* R1, const void* R2, int64_t N,
                                                 int h, int r, int M, int k, int32_t* out_idx,
                                                 float* out_gate, int32_t* out_expert_count,
                                                 float* out_logits, void* stream) {
  // the arguments are checked first, as more_route_unfused checks them; only a valid
  // problem that does not fit the fixed scratch is reported as unsupported
  const more_status st =
      more::validate_route(X, R1, R2, N, h, r, M, k, out_idx, out_gate, out_expert_count, out_logits);
  if (st != MORE_OK) return st;
  if (N > 0 && more_route_unfused_scratch_bytes(N, r, M) > (size_t)MORE_STATIC_SCRATCH_BYTES)
    return MORE_ERR_UNSUPPORTED;
  cudaError_t err = cudaSuccess;
  void* scratch = more::static_scratch_address(&err);
  if (!scratch) return MORE_ERR_CUDA;
  // Same validation and launches as the caller-scratch entry point; it allocates nothing.
  return more_route_unfused(X, R1, R2, N, h, r, M, k, out_idx, out_gate, out_expert_count, out_logits,
                            scratch, (size_t)MORE_STATIC_SCRATCH_BYTES, stream);
}

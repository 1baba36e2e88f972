// C ABI of the router: argument validation, variant choice, the device error word.
#include <mutex>

#include "more_internal.cuh"

namespace more {

// Device error word of this library (one per device; MORE_DEVERR_* bits).
__device__ unsigned int g_device_status;

namespace {

unsigned int* status_word() {
  // The symbol address differs per device; cache it per device ordinal.
  static std::mutex mu;
  static unsigned int* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<unsigned int*>(p);
  }
  return addr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

RouteArgs make_args(const void* X, const void* R1, const void* R2, int64_t N, int h, int r, int M,
                    int k, int32_t* out_idx, float* out_gate, int32_t* out_count,
                    float* out_logits, void* stream) {
  RouteArgs a;
  a.X = static_cast<const __nv_bfloat16*>(X);
  a.R1 = static_cast<const __nv_bfloat16*>(R1);
  a.R2 = static_cast<const __nv_bfloat16*>(R2);
  a.N = N;
  a.h = h;
  a.r = r;
  a.M = M;
  a.k = k;
  a.out_idx = out_idx;
  a.out_gate = out_gate;
  a.out_count = out_count;
  a.out_logits = out_logits;
  a.status = nullptr;
  a.stream = static_cast<cudaStream_t>(stream);
  a.zero_counts = 0;
  return a;
}

// AUTO's choice of kernel, from per-call times measured on a B200 (CUDA-graph replays of
// back-to-back calls; h = 2048, M = 4096 with r = 16, 32 and 128):
// - up to 148 tokens the small-N kernel runs one CTA per token, one CTA per SM: a single wave
//   on the 148 SMs of a B200.  Its time follows the weights one SM reads, r * (h + M) bf16
//   values: 7.3 us at r = 16, 13.1 us at r = 32, 48 us at r = 128.  The cluster kernel spreads
//   them over eight SMs and wins from r * (h + M) = 196608 (r = 32 at this shape: 12.6 against
//   13.2 us at N = 1) while it holds at most 8 clusters (N <= 64), and from twice that at any
//   N (r = 128: 36 against 49 us at N = 64);
// - beyond 148 tokens the small-N kernel needs a second wave and the cluster kernel overtakes it.
//   Its time grows linearly, about 9 us + N * (0.013 us + 1.53e-7 us * r * (h + M)) (r = 16:
//   35 us at N = 1024, 121 us at 4096; r = 32: 56 us at 1024, 188 us at 4096);
// - the fused kernel's time has a floor until every SM holds a tile: the chain of one
//   128-token tile (Z over h, then two sweeps over the M / 128 expert tiles), about
//   5 us + 0.0056 us * h + 0.0133 us * M * (0.7 + 0.3 r / 32) (r = 32: 74 us; r = 16: 58 us).
// AUTO takes the cluster kernel while its estimate is below that floor, the fused kernel
// beyond (when its shared-memory plan fits the shape), and the cluster kernel at any N for
// shapes the fused kernel does not take.
constexpr int64_t kClusterMinTokens = 149;

double cluster_estimate_us(int64_t N, int h, int r, int M) {
  return 9.0 + (double)N * (0.013 + 1.53e-7 * r * ((double)h + M));
}

double fused_floor_us(int h, int r, int M) {
  return 5.0 + 0.0056 * h + 0.0133 * M * (0.7 + 0.3 * r / 32.0);
}

constexpr double kClusterWeights = 196608.0;  // r * (h + M) from which the cluster kernel wins at N <= 64

int auto_variant(const RouteArgs& a) {
  if (a.N < kClusterMinTokens) {
    const double w = (double)a.r * ((double)a.h + a.M);
    return (a.N <= 64 && w >= kClusterWeights) || w >= 2 * kClusterWeights ? MORE_VARIANT_CLUSTER
                                                                            : MORE_VARIANT_SMALL_N;
  }
  if (!fused_tc_fits(a)) return MORE_VARIANT_CLUSTER;
  return cluster_estimate_us(a.N, a.h, a.r, a.M) < fused_floor_us(a.h, a.r, a.M) ? MORE_VARIANT_CLUSTER
                                                                                  : MORE_VARIANT_FUSED_TC;
}

}  // namespace

namespace {
// Shapes that cannot mean anything (MORE_ERR_INVALID_ARG) and legal shapes outside the
// library's limits (MORE_ERR_UNSUPPORTED).
bool shape_invalid(int64_t N, int h, int r, int M, int k) {
  return N < 0 || h < 8 || (h & 7) || M < 8 || (M & 7) || k < 1 || k > M || r < 1;
}
bool shape_unsupported(int64_t N, int r, int M, int k) {
  return N > 0x7fffffffLL || k > MORE_KMAX || (r & 15) || r < 16 || r > 128 || M > MORE_MMAX;
}
}  // namespace

// Argument checks shared by every routing entry point (see more_route.h).
more_status validate_shape(int64_t N, int h, int r, int M, int k) {
  if (shape_invalid(N, h, r, M, k)) return MORE_ERR_INVALID_ARG;
  if (shape_unsupported(N, r, M, k)) return MORE_ERR_UNSUPPORTED;
  return MORE_OK;
}

more_status validate_route(const void* X, const void* R1, const void* R2, int64_t N, int h, int r, int M, int k,
                           const int32_t* out_idx, const float* out_gate, const int32_t* out_count,
                           const float* out_logits) {
  if (shape_invalid(N, h, r, M, k)) return MORE_ERR_INVALID_ARG;
  if (!R1 || !R2 || !out_count || (N > 0 && (!X || !out_idx || !out_gate))) return MORE_ERR_INVALID_ARG;
  if ((X && !aligned16(X)) || !aligned16(R1) || !aligned16(R2) || (out_idx && !aligned16(out_idx)) ||
      (out_gate && !aligned16(out_gate)) || !aligned16(out_count) || (out_logits && !aligned16(out_logits)))
    return MORE_ERR_INVALID_ARG;
  if (shape_unsupported(N, r, M, k)) return MORE_ERR_UNSUPPORTED;
  return MORE_OK;
}

}  // namespace more

using namespace more;

extern "C" {

int more_abi_version(void) { return MORE_ROUTE_ABI_VERSION; }

const char* more_status_string(more_status s) {
  switch (s) {
    case MORE_OK:
      return "MORE_OK";
    case MORE_ERR_INVALID_ARG:
      return "MORE_ERR_INVALID_ARG: null or misaligned pointer, or impossible shape";
    case MORE_ERR_UNSUPPORTED:
      return "MORE_ERR_UNSUPPORTED: request outside the library's limits";
    case MORE_ERR_CUDA:
      return "MORE_ERR_CUDA: a CUDA call or kernel launch failed";
    case MORE_ERR_DEVICE:
      return "MORE_ERR_DEVICE: a kernel recorded an error";
  }
  return "unknown more_status";
}

more_status more_route_variant(const void* X, const void* R1, const void* R2, int64_t N, int h, int r,
                               int M, int k, int32_t* out_idx, float* out_gate,
                               int32_t* out_expert_count, float* out_logits, int variant,
                               void* stream) {
  more_status st = validate_route(X, R1, R2, N, h, r, M, k, out_idx, out_gate, out_expert_count, out_logits);
  if (st != MORE_OK) return st;
  if (variant < MORE_VARIANT_AUTO || variant > MORE_VARIANT_CLUSTER) return MORE_ERR_INVALID_ARG;
  RouteArgs a = make_args(X, R1, R2, N, h, r, M, k, out_idx, out_gate, out_expert_count, out_logits,
                          stream);
  a.status = status_word();
  if (!a.status) return MORE_ERR_CUDA;
  if (N > 0 && variant == MORE_VARIANT_AUTO) variant = auto_variant(a);
  // a single token on the small-N kernel (one CTA), or up to 8 on the cluster kernel (one
  // cluster), is routed by a launch that zeroes the counts itself
  a.zero_counts = ((N == 1 && variant == MORE_VARIANT_SMALL_N) || (N >= 1 && N <= 8 && variant == MORE_VARIANT_CLUSTER))
                      ? 1 : 0;
  if (!a.zero_counts && cudaMemsetAsync(out_expert_count, 0, sizeof(int32_t) * (size_t)M, a.stream) != cudaSuccess)
    return MORE_ERR_CUDA;
  if (N == 0) return MORE_OK;
  cudaError_t err;
  if (variant == MORE_VARIANT_FUSED_TC) {
    if (!fused_tc_supports(a)) return MORE_ERR_UNSUPPORTED;
    err = launch_fused_tc(a);
  } else if (variant == MORE_VARIANT_CLUSTER) {
    err = launch_cluster(a);
  } else {
    err = launch_small_n(a);
  }
  return err == cudaSuccess ? MORE_OK : MORE_ERR_CUDA;
}

int more_route_auto_variant(int64_t N, int h, int r, int M, int k) {
  if (validate_shape(N, h, r, M, k) != MORE_OK) return MORE_VARIANT_AUTO;
  RouteArgs a = make_args(nullptr, nullptr, nullptr, N, h, r, M, k, nullptr, nullptr, nullptr, nullptr, nullptr);
  return auto_variant(a);
}

more_status more_route(const void* X, const void* R1, const void* R2, int64_t N, int h, int r, int M,
                       int k, int32_t* out_idx, float* out_gate, int32_t* out_expert_count,
                       float* out_logits, void* stream) {
  return more_route_variant(X, R1, R2, N, h, r, M, k, out_idx, out_gate, out_expert_count, out_logits,
                            MORE_VARIANT_AUTO, stream);
}

more_status more_route_train(const void* X, const void* R1, const void* R2, int64_t N, int h, int r, int M,
                             int k, int32_t* out_idx, float* out_gate, int32_t* out_expert_count,
                             float* out_logits, float* out_m, float* out_Z, float* out_psum, void* stream) {
  more_status st = validate_route(X, R1, R2, N, h, r, M, k, out_idx, out_gate, out_expert_count, out_logits);
  if (st != MORE_OK) return st;
  if (!out_psum || !aligned16(out_psum) || (N > 0 && (!out_m || !out_Z)) || (out_m && !aligned16(out_m)) ||
      (out_Z && !aligned16(out_Z)))
    return MORE_ERR_INVALID_ARG;
  if (M > MORE_STATS_MMAX) return MORE_ERR_UNSUPPORTED;
  st = more_route_variant(X, R1, R2, N, h, r, M, k, out_idx, out_gate, out_expert_count, out_logits,
                          MORE_VARIANT_AUTO, stream);
  if (st != MORE_OK) return st;
  RouteArgs a = make_args(X, R1, R2, N, h, r, M, k, out_idx, out_gate, out_expert_count, out_logits,
                          stream);
  if (cudaMemsetAsync(out_psum, 0, sizeof(float) * (size_t)M, a.stream) != cudaSuccess) return MORE_ERR_CUDA;
  if (N == 0) return MORE_OK;
  // the tensor-core statistics where the rank and shared-memory plan allow, else the CUDA-core kernel
  const cudaError_t err = train_stats_tc_supports(a) ? launch_train_stats_tc(a, out_m, out_Z, out_psum)
                                                     : launch_train_stats(a, out_m, out_Z, out_psum);
  return err == cudaSuccess ? MORE_OK : MORE_ERR_CUDA;
}

size_t more_dispatch_scratch_bytes(int64_t N, int k, int M) {
  if (N < 0 || k < 1 || M < 1 || M > MORE_MMAX || N * (int64_t)k > 0x7fffffffLL) return 0;
  return (size_t)dispatch_scratch_bytes(N * (int64_t)k, M);
}

more_status more_dispatch_variant(const int32_t* idx, int64_t N, int k, int M, int32_t* out_offsets,
                                  int32_t* out_sorted, void* scratch, size_t scratch_bytes, int variant,
                                  void* stream) {
  if (N < 0 || k < 1 || M < 1 || !out_offsets || !aligned16(out_offsets)) return MORE_ERR_INVALID_ARG;
  if (variant < MORE_DISPATCH_AUTO || variant > MORE_DISPATCH_SHARED) return MORE_ERR_INVALID_ARG;
  if (k > MORE_KMAX || M > MORE_MMAX || N * (int64_t)k > 0x7fffffffLL) return MORE_ERR_UNSUPPORTED;
  if (variant == MORE_DISPATCH_SHARED && !dispatch_shared_supports(M)) return MORE_ERR_UNSUPPORTED;
  // AUTO: the shared-memory kernels where they apply (measured at prefill r = 32: 79 us against
  // 260 us for the global histograms), the global ones beyond MORE_DISPATCH_SHARED_MMAX
  if (variant == MORE_DISPATCH_AUTO) variant = dispatch_shared_supports(M) ? MORE_DISPATCH_SHARED : MORE_DISPATCH_GLOBAL;
  const int64_t S = N * (int64_t)k;
  if (S > 0 && (!idx || !out_sorted || !scratch || !aligned16(idx) || !aligned16(out_sorted) ||
                !aligned16(scratch) || scratch_bytes < (size_t)dispatch_scratch_bytes(S, M)))
    return MORE_ERR_INVALID_ARG;
  unsigned int* status = status_word();
  if (!status) return MORE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const cudaError_t err = variant == MORE_DISPATCH_SHARED
                              ? launch_dispatch_shared(idx, S, M, out_offsets, out_sorted, scratch, status, s)
                              : launch_dispatch(idx, S, M, out_offsets, out_sorted, scratch, status, s);
  return err == cudaSuccess ? MORE_OK : MORE_ERR_CUDA;
}

more_status more_dispatch(const int32_t* idx, int64_t N, int k, int M, int32_t* out_offsets,
                          int32_t* out_sorted, void* scratch, size_t scratch_bytes, void* stream) {
  return more_dispatch_variant(idx, N, k, M, out_offsets, out_sorted, scratch, scratch_bytes, MORE_DISPATCH_AUTO,
                               stream);
}

size_t more_route_backward_scratch_bytes(int64_t N, int h, int r, int M) {
  if (N < 0 || N > 0x7fffffffLL || h < 1 || r < 1 || r > 128 || M < 1) return 0;
  return (size_t)backward_scratch_bytes(N, h, r, M);
}

more_status more_route_backward(const void* X, const void* R1, const void* R2, int64_t N, int h, int r, int M,
                                int k, const int32_t* top_idx, const float* top_vals_bar, const float* pbar,
                                const float* saved_m, const float* saved_Z, float* out_Xbar, float* out_R1bar,
                                float* out_R2bar, float* out_g, void* scratch, size_t scratch_bytes,
                                void* stream) {
  if (N < 0 || h < 8 || (h & 7) || M < 8 || (M & 7) || k < 1 || k > M || r < 1) return MORE_ERR_INVALID_ARG;
  if (!R1 || !R2 || !out_R1bar || !out_R2bar) return MORE_ERR_INVALID_ARG;
  if (N > 0 && (!X || !out_Xbar || !scratch || (top_vals_bar && !top_idx) || (pbar && (!saved_m || !saved_Z))))
    return MORE_ERR_INVALID_ARG;
  const void* ptrs[] = {X,       R1,      R2,       top_idx,   top_vals_bar, pbar, saved_m,
                        saved_Z, out_Xbar, out_R1bar, out_R2bar, out_g,        scratch};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MORE_ERR_INVALID_ARG;
  if (N > 0x7fffffffLL) return MORE_ERR_UNSUPPORTED;
  if (k > MORE_KMAX || (r & 15) || r < 16 || r > 128 || M > MORE_MMAX) return MORE_ERR_UNSUPPORTED;
  if (N > 0 && scratch_bytes < (size_t)backward_scratch_bytes(N, h, r, M)) return MORE_ERR_INVALID_ARG;
  BackwardArgs b;
  b.X = static_cast<const __nv_bfloat16*>(X);
  b.R1 = static_cast<const __nv_bfloat16*>(R1);
  b.R2 = static_cast<const __nv_bfloat16*>(R2);
  b.N = N;
  b.h = h;
  b.r = r;
  b.M = M;
  b.k = k;
  b.top_idx = top_idx;
  b.top_vals_bar = top_vals_bar;
  b.pbar = pbar;
  b.m = saved_m;
  b.Z = saved_Z;
  b.Xbar = out_Xbar;
  b.R1bar = out_R1bar;
  b.R2bar = out_R2bar;
  b.g = out_g;
  b.scratch = scratch;
  b.status = status_word();
  b.stream = static_cast<cudaStream_t>(stream);
  if (!b.status) return MORE_ERR_CUDA;
  return launch_backward(b) == cudaSuccess ? MORE_OK : MORE_ERR_CUDA;
}

size_t more_route_unfused_scratch_bytes(int64_t N, int r, int M) {
  if (N < 0 || r < 1 || M < 1) return 0;
  return unfused_scratch_bytes(N, r, M);
}

more_status more_route_unfused(const void* X, const void* R1, const void* R2, int64_t N, int h, int r,
                               int M, int k, int32_t* out_idx, float* out_gate,
                               int32_t* out_expert_count, float* out_logits, void* scratch,
                               size_t scratch_bytes, void* stream) {
  more_status st = validate_route(X, R1, R2, N, h, r, M, k, out_idx, out_gate, out_expert_count, out_logits);
  if (st != MORE_OK) return st;
  if (N > 0 && (!scratch || !aligned16(scratch) || scratch_bytes < unfused_scratch_bytes(N, r, M)))
    return MORE_ERR_INVALID_ARG;
  RouteArgs a = make_args(X, R1, R2, N, h, r, M, k, out_idx, out_gate, out_expert_count, out_logits,
                          stream);
  a.status = status_word();
  if (!a.status) return MORE_ERR_CUDA;
  if (cudaMemsetAsync(out_expert_count, 0, sizeof(int32_t) * (size_t)M, a.stream) != cudaSuccess)
    return MORE_ERR_CUDA;
  if (N == 0) return MORE_OK;
  return launch_unfused(a, scratch) == cudaSuccess ? MORE_OK : MORE_ERR_CUDA;
}

more_status more_route_unfused_tc(const void* X, const void* R1, const void* R2, int64_t N, int h, int r,
                                  int M, int k, int32_t* out_idx, float* out_gate,
                                  int32_t* out_expert_count, float* out_logits, void* scratch,
                                  size_t scratch_bytes, void* stream) {
  more_status st = validate_route(X, R1, R2, N, h, r, M, k, out_idx, out_gate, out_expert_count, out_logits);
  if (st != MORE_OK) return st;
  if (r != 16 && r != 32 && r != 64 && r != 128) return MORE_ERR_UNSUPPORTED;
  if (N > 0 && (!scratch || !aligned16(scratch) || scratch_bytes < unfused_scratch_bytes(N, r, M)))
    return MORE_ERR_INVALID_ARG;
  RouteArgs a = make_args(X, R1, R2, N, h, r, M, k, out_idx, out_gate, out_expert_count, out_logits,
                          stream);
  a.status = status_word();
  if (!a.status) return MORE_ERR_CUDA;
  if (N > 0 && !unfused_tc_supports(a)) return MORE_ERR_UNSUPPORTED;
  if (cudaMemsetAsync(out_expert_count, 0, sizeof(int32_t) * (size_t)M, a.stream) != cudaSuccess)
    return MORE_ERR_CUDA;
  if (N == 0) return MORE_OK;
  return launch_unfused_tc(a, scratch) == cudaSuccess ? MORE_OK : MORE_ERR_CUDA;
}

more_status more_route_fullrank(const void* X, const void* W, int64_t N, int h, int M, int k,
                                int32_t* out_idx, float* out_gate, int32_t* out_expert_count,
                                float* out_logits, void* stream) {
  // the shape rules of more_route with the rank check left out (r = 16 stands for "any")
  more_status st = validate_route(X, W, W, N, h, 16, M, k, out_idx, out_gate, out_expert_count, out_logits);
  if (st != MORE_OK) return st;
  RouteArgs a = make_args(X, nullptr, W, N, h, 0, M, k, out_idx, out_gate, out_expert_count, out_logits, stream);
  a.status = status_word();
  if (!a.status) return MORE_ERR_CUDA;
  if (cudaMemsetAsync(out_expert_count, 0, sizeof(int32_t) * (size_t)M, a.stream) != cudaSuccess)
    return MORE_ERR_CUDA;
  if (N == 0) return MORE_OK;
  return launch_fullrank(a) == cudaSuccess ? MORE_OK : MORE_ERR_CUDA;
}

more_status more_selftest_wait_timeout(int32_t* out_result, void* stream) {
  if (!out_result || (reinterpret_cast<uintptr_t>(out_result) & 3u)) return MORE_ERR_INVALID_ARG;
  unsigned int* status = status_word();
  if (!status) return MORE_ERR_CUDA;
  return launch_wait_timeout_probe(status, out_result, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MORE_OK
             : MORE_ERR_CUDA;
}

more_status more_device_status(void* stream, uint32_t* detail) {
  if (detail) *detail = 0;
  unsigned int* word = status_word();
  if (!word) return MORE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MORE_ERR_CUDA;
  unsigned int value = 0;
  if (cudaMemcpy(&value, word, sizeof(value), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MORE_ERR_CUDA;
  if (value != 0) {
    unsigned int zero = 0;
    if (cudaMemcpy(word, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return MORE_ERR_CUDA;
  }
  if (detail) *detail = value;
  return value ? MORE_ERR_DEVICE : MORE_OK;
}

}  // extern "C"

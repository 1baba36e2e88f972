// Internal declarations shared by the router's translation units (not part of the ABI).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "more_route.h"

namespace more {

// Arguments of one routing call after validation.
struct RouteArgs {
  const __nv_bfloat16* X;
  const __nv_bfloat16* R1;
  const __nv_bfloat16* R2;
  int64_t N;
  int h, r, M, k;
  int32_t* out_idx;
  float* out_gate;
  int32_t* out_count;
  float* out_logits;  // may be null
  unsigned int* status;  // device error word (MORE_DEVERR_* bits)
  cudaStream_t stream;
  int zero_counts;  // the kernel zeroes out_count itself (single-CTA calls; no memset issued)
};

// Argument checks of the routing entry points (more_route.h): MORE_OK or the error to return.
more_status validate_shape(int64_t N, int h, int r, int M, int k);
more_status validate_route(const void* X, const void* R1, const void* R2, int64_t N, int h, int r, int M, int k,
                           const int32_t* out_idx, const float* out_gate, const int32_t* out_count,
                           const float* out_logits);

// Launchers; each returns cudaSuccess or the launch error.
cudaError_t launch_small_n(const RouteArgs& a);
cudaError_t launch_cluster(const RouteArgs& a);
int64_t dispatch_scratch_bytes(int64_t S, int M);
cudaError_t launch_dispatch(const int32_t* idx, int64_t S, int M, int32_t* offsets, int32_t* sorted,
                            void* scratch, unsigned int* status, cudaStream_t stream);
bool dispatch_shared_supports(int M);
cudaError_t launch_dispatch_shared(const int32_t* idx, int64_t S, int M, int32_t* offsets, int32_t* sorted,
                                   void* scratch, unsigned int* status, cudaStream_t stream);
cudaError_t launch_train_stats(const RouteArgs& a, float* out_m, float* out_Z, float* out_psum);

// Arguments of one backward call after validation (pointers as in more_route_backward).
struct BackwardArgs {
  const __nv_bfloat16* X;
  const __nv_bfloat16* R1;
  const __nv_bfloat16* R2;
  int64_t N;
  int h, r, M, k;
  const int32_t* top_idx;     // may be null (with top_vals_bar)
  const float* top_vals_bar;  // may be null
  const float* pbar;          // may be null (then m and Z are not read)
  const float* m;
  const float* Z;
  float* Xbar;
  float* R1bar;
  float* R2bar;
  float* g;  // may be null
  void* scratch;
  unsigned int* status;
  cudaStream_t stream;
};
int64_t backward_scratch_bytes(int64_t N, int h, int r, int M);
cudaError_t launch_backward(const BackwardArgs& b);
cudaError_t launch_fused_tc(const RouteArgs& a);
// The fused kernel's shared-memory plan fits the shape (r, M, k); supports: it fits and the
// driver's tensor-map encoder is available.
bool fused_tc_fits(const RouteArgs& a);
bool fused_tc_supports(const RouteArgs& a);
cudaError_t launch_unfused(const RouteArgs& a, void* scratch);
size_t unfused_scratch_bytes(int64_t N, int r, int M);
// The fp32 [N][M] score tensor inside an unfused scratch buffer (after the z area).
float* unfused_scores_of(void* scratch, int64_t N, int r);
// Row-wise top-k and softmax over materialised scores: per-lane running lists (the CUDA-core
// unfused path), and a running list filtered by its k-th value (the tensor-core unfused path).
cudaError_t launch_scores_topk(const RouteArgs& a, const float* scores);
cudaError_t launch_threshold_topk(const RouteArgs& a, const float* scores);
// Tensor-core materialisation of the scores (same products as the fused kernel), then the
// row-wise top-k; scratch as for launch_unfused.
bool unfused_tc_supports(const RouteArgs& a);
cudaError_t launch_unfused_tc(const RouteArgs& a, void* scratch);
// Training statistics (App. F, Algorithm 2) from the same tensor-core logits: m, Z per token
// and psum per expert (psum accumulated with atomics: zero it first).
bool train_stats_tc_supports(const RouteArgs& a);
cudaError_t launch_train_stats_tc(const RouteArgs& a, float* out_m, float* out_Z, float* out_psum);
// Fused full-rank router: a.R2 holds W (h x M); a.R1 and a.r are unused.
cudaError_t launch_fullrank(const RouteArgs& a);
// One bounded wait that nothing completes (the failure path's self-test); writes 2 to
// *out_result when the wait gave up, 1 if it completed.
cudaError_t launch_wait_timeout_probe(unsigned int* status, int32_t* out_result, cudaStream_t stream);

// ---- small device helpers -------------------------------------------------

__device__ __forceinline__ float bf16_round(float v) {
  return __bfloat162float(__float2bfloat16_rn(v));
}

// z as the bf16 pair z_hi + z_lo (z_hi = bf16(z), z_lo = bf16(z - z_hi)), summed in fp32:
// the value every kernel multiplies with R2 (about 16 significant bits of z).
__device__ __forceinline__ float split_bf16_pair(float z) {
  float hi = bf16_round(z);
  return hi + bf16_round(z - hi);
}

// Routing order on (value, expert): a goes first iff it has the larger value,
// or the same value and the lower expert index.
__device__ __forceinline__ bool goes_first(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

}  // namespace more

// C entry points of the emulated library: the CUDA-core kernels' launchers, with the arguments
// the C ABI takes (host pointers here).  Each zeroes what the C ABI zeroes before launching.
#include "prelude.h"
#include "more_internal.cuh"

extern "C" long emu_backward_scratch_bytes(int64_t N, int h, int r, int M) {
  return (long)more::backward_scratch_bytes(N, h, r, M);
}

extern "C" int emu_backward(const void* X, const void* R1, const void* R2, int64_t N, int h, int r, int M, int k,
                            const int32_t* idx, const float* tvb, const float* pbar, const float* m, const float* Z,
                            float* Xbar, float* R1bar, float* R2bar, float* g, void* scratch, unsigned* status) {
  more::BackwardArgs b;
  b.X = (const __nv_bfloat16*)X;
  b.R1 = (const __nv_bfloat16*)R1;
  b.R2 = (const __nv_bfloat16*)R2;
  b.N = N;
  b.h = h;
  b.r = r;
  b.M = M;
  b.k = k;
  b.top_idx = idx;
  b.top_vals_bar = tvb;
  b.pbar = pbar;
  b.m = m;
  b.Z = Z;
  b.Xbar = Xbar;
  b.R1bar = R1bar;
  b.R2bar = R2bar;
  b.g = g;
  b.scratch = scratch;
  b.status = status;
  b.stream = nullptr;
  return (int)more::launch_backward(b);
}

extern "C" int emu_route_cluster(const void* X, const void* R1, const void* R2, int64_t N, int h, int r, int M, int k,
                                 int32_t* idx, float* gate, int32_t* cnt, float* logits, unsigned* status) {
  more::RouteArgs a;
  a.X = (const __nv_bfloat16*)X;
  a.R1 = (const __nv_bfloat16*)R1;
  a.R2 = (const __nv_bfloat16*)R2;
  a.N = N;
  a.h = h;
  a.r = r;
  a.M = M;
  a.k = k;
  a.out_idx = idx;
  a.out_gate = gate;
  a.out_count = cnt;
  a.out_logits = logits;
  a.status = status;
  a.stream = nullptr;
  a.zero_counts = 0;
  memset(cnt, 0, sizeof(int32_t) * M);  // the C entry point zeroes the counts before launching
  emu::cluster_size = 8;                 // cluster_route_kernel's __cluster_dims__
  const int rc = (int)more::launch_cluster(a);
  emu::cluster_size = 1;
  return rc;
}

namespace {
more::RouteArgs route_args(const void* X, const void* R1, const void* R2, int64_t N, int h, int r, int M, int k,
                           int32_t* idx, float* gate, int32_t* cnt, float* logits, unsigned* status) {
  more::RouteArgs a;
  a.X = (const __nv_bfloat16*)X;
  a.R1 = (const __nv_bfloat16*)R1;
  a.R2 = (const __nv_bfloat16*)R2;
  a.N = N;
  a.h = h;
  a.r = r;
  a.M = M;
  a.k = k;
  a.out_idx = idx;
  a.out_gate = gate;
  a.out_count = cnt;
  a.out_logits = logits;
  a.status = status;
  a.stream = nullptr;
  a.zero_counts = 0;
  if (cnt) memset(cnt, 0, sizeof(int32_t) * M);
  return a;
}
}  // namespace

extern "C" int emu_route_small(const void* X, const void* R1, const void* R2, int64_t N, int h, int r, int M, int k,
                               int32_t* idx, float* gate, int32_t* cnt, float* logits, unsigned* status) {
  return (int)more::launch_small_n(route_args(X, R1, R2, N, h, r, M, k, idx, gate, cnt, logits, status));
}

// Up to 8 tokens on the cluster kernel with the counts zeroed by its single cluster (as
// more_route does for N <= 8): the counts start as garbage here.
extern "C" int emu_route_cluster_self_zero(const void* X, const void* R1, const void* R2, int64_t N, int h, int r,
                                           int M, int k, int32_t* idx, float* gate, int32_t* cnt, float* logits,
                                           unsigned* status) {
  more::RouteArgs a = route_args(X, R1, R2, N, h, r, M, k, idx, gate, nullptr, logits, status);
  a.out_count = cnt;
  for (int e = 0; e < M; ++e) cnt[e] = 7;
  a.zero_counts = 1;
  emu::cluster_size = 8;
  const int rc = (int)more::launch_cluster(a);
  emu::cluster_size = 1;
  return rc;
}

// One token on the small-N kernel with the counts zeroed by the kernel itself (as more_route does
// for N == 1): the counts start as garbage here.
extern "C" int emu_route_small_self_zero(const void* X, const void* R1, const void* R2, int h, int r, int M, int k,
                                         int32_t* idx, float* gate, int32_t* cnt, float* logits, unsigned* status) {
  more::RouteArgs a = route_args(X, R1, R2, 1, h, r, M, k, idx, gate, nullptr, logits, status);
  a.out_count = cnt;
  for (int e = 0; e < M; ++e) cnt[e] = 7;
  a.zero_counts = 1;
  return (int)more::launch_small_n(a);
}

extern "C" long emu_unfused_scratch_bytes(int64_t N, int r, int M) { return (long)more::unfused_scratch_bytes(N, r, M); }

extern "C" int emu_route_unfused(const void* X, const void* R1, const void* R2, int64_t N, int h, int r, int M, int k,
                                 int32_t* idx, float* gate, int32_t* cnt, float* logits, void* scratch,
                                 unsigned* status) {
  return (int)more::launch_unfused(route_args(X, R1, R2, N, h, r, M, k, idx, gate, cnt, logits, status), scratch);
}

extern "C" int emu_threshold_topk(const float* scores, int64_t N, int M, int k, int32_t* idx, float* gate,
                                  int32_t* cnt, float* logits, unsigned* status) {
  return (int)more::launch_threshold_topk(
      route_args(nullptr, nullptr, nullptr, N, 8, 16, M, k, idx, gate, cnt, logits, status), scores);
}

extern "C" int emu_train_stats(const void* X, const void* R1, const void* R2, int64_t N, int h, int r, int M,
                               float* out_m, float* out_Z, float* out_psum, unsigned* status) {
  memset(out_psum, 0, sizeof(float) * M);
  return (int)more::launch_train_stats(route_args(X, R1, R2, N, h, r, M, 1, nullptr, nullptr, nullptr, nullptr,
                                                  status),
                                       out_m, out_Z, out_psum);
}

extern "C" long emu_dispatch_scratch_bytes(int64_t S, int M) { return (long)more::dispatch_scratch_bytes(S, M); }

extern "C" int emu_dispatch(const int32_t* idx, int64_t S, int M, int32_t* offsets, int32_t* sorted, void* scratch,
                            unsigned* status) {
  return (int)more::launch_dispatch(idx, S, M, offsets, sorted, scratch, status, nullptr);
}

extern "C" int emu_dispatch_shared(const int32_t* idx, int64_t S, int M, int32_t* offsets, int32_t* sorted,
                                   void* scratch, unsigned* status) {
  return (int)more::launch_dispatch_shared(idx, S, M, offsets, sorted, scratch, status, nullptr);
}

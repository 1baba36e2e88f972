// Small-batch (decode-sized) MoRE routing kernel on CUDA cores: one warp per token.
//
// Per token, following "MoRE: Scaling mixture of experts with hardware-aware
// low-rank routing", App. F, Algorithm 1 (z accumulated in fp32, one sweep over
// the experts with a running top-k) and Fig. 12 (softmax over the k selected
// logits):
//   1. z = x . R1: lanes stride over h, 16 outputs per pass, reduce-scatter
//      through shuffles; z is carried as the bf16 pair z_hi + z_lo (finer than
//      Algorithm 1's single bf16) and kept in shared memory.
//   2. lanes take expert pairs (2 lane + 64 j, +1); each lane keeps a sorted
//      running top-k of its experts (strict '>' insertion, so on equal logits
//      the lower expert index stays ahead).
//   3. k warp-wide arg-max rounds merge the 32 lists in routing order.
//   4. softmax over the k logits, outputs, and one atomic count per selection.
#include "more_internal.cuh"
#include "warp_simt.cuh"

namespace more {
namespace {

constexpr int kWarpsPerBlock = 8;


template <int K>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    small_n_route_kernel(RouteArgs a) {
  extern __shared__ float smem_z[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* zs = smem_z + warp * a.r;
  const int64_t stride = (int64_t)gridDim.x * kWarpsPerBlock;
  for (int64_t n = (int64_t)blockIdx.x * kWarpsPerBlock + warp; n < a.N; n += stride) {
    warp_project_token(a.X + (size_t)n * a.h, a.R1, a.h, a.r, zs, lane);
    __syncwarp();
    TopList<K> list;
    list.init();
    for (int e = 2 * lane; e < a.M; e += 64) {
      float acc0 = 0.f, acc1 = 0.f;
      const __nv_bfloat162* col = reinterpret_cast<const __nv_bfloat162*>(a.R2 + e);
      const int pitch = a.M >> 1;  // row pitch in bf16 pairs
      for (int i = 0; i < a.r; ++i) {
        float zi = zs[i];
        float2 w = __bfloat1622float2(col[(size_t)i * pitch]);
        acc0 = fmaf(zi, w.x, acc0);
        acc1 = fmaf(zi, w.y, acc1);
      }
      list.insert(acc0, e);
      list.insert(acc1, e + 1);
    }
    float my_v;
    int my_i;
    warp_merge_topk<K>(list, a.k, lane, my_v, my_i);
    warp_write_selection(a, n, lane, my_v, my_i);
    __syncwarp();
  }
}

template <int K>
cudaError_t launch_k(const RouteArgs& a) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = (a.N + kWarpsPerBlock - 1) / kWarpsPerBlock;
  int64_t cap = (int64_t)sms * 8;
  if (blocks > cap) blocks = cap;
  size_t smem = sizeof(float) * kWarpsPerBlock * a.r;
  small_n_route_kernel<K><<<(unsigned)blocks, kWarpsPerBlock * 32, smem, a.stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_small_n(const RouteArgs& a) {
  if (a.N == 0) return cudaSuccess;
  switch (a.k) {
#define MORE_CASE(K) \
  case K:            \
    return launch_k<K>(a);
    MORE_CASE(1) MORE_CASE(2) MORE_CASE(3) MORE_CASE(4) MORE_CASE(5) MORE_CASE(6) MORE_CASE(7)
    MORE_CASE(8) MORE_CASE(9) MORE_CASE(10) MORE_CASE(11) MORE_CASE(12) MORE_CASE(13)
    MORE_CASE(14) MORE_CASE(15) MORE_CASE(16)
#undef MORE_CASE
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace more

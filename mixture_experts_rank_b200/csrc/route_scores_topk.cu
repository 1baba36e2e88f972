// Row-wise top-k and softmax over a materialised fp32 score tensor [N][M]: the last kernel of
// the tensor-core unfused path (the unfused router of "MoRE: Scaling mixture of experts with
// hardware-aware low-rank routing", App. H.6, Fig. 24, where most of the time goes to this
// top-k over the stored scores).  Per token: the k largest scores in routing order (larger
// value first, lower expert first on equal values), the softmax over them, and the counts.
#include "more_internal.cuh"
#include "warp_simt.cuh"

namespace more {
namespace {

// One warp per token row.  The warp keeps the running top-k in routing order spread over
// lanes 0..k-1 (lane j: the j-th entry) and reads the row 128 experts at a time, one float4
// per lane.  A chunk is inspected only where a value beats the current k-th entry (strictly:
// every value of a later chunk has a larger expert index, so it loses ties); such values are
// inserted one at a time in expert order.  The first chunk is pre-filtered by the k-th
// largest of its 32 lane maxima, a lower bound on its k-th largest value (k of its values
// reach it), so only values at or above it are inserted.
constexpr int kTopkWarps = 8;
constexpr int kTopkUnroll = 4;  // chunks of 128 experts loaded per step

__device__ __forceinline__ float warp_kth_largest(float v, int k, int lane) {
  // bitonic sort of the 32 lane values, descending
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const float o = __shfl_xor_sync(0xffffffffu, v, stride);
      const bool keep_max = ((lane & size) == 0) == ((lane & stride) == 0);
      v = keep_max ? fmaxf(v, o) : fminf(v, o);
    }
  }
  return __shfl_sync(0xffffffffu, v, k - 1);
}

__global__ void __launch_bounds__(kTopkWarps * 32) threshold_topk_kernel(RouteArgs a, const float* __restrict__ scores) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k = a.k, M = a.M;
  for (int64_t n = (int64_t)blockIdx.x * kTopkWarps + warp; n < a.N; n += (int64_t)gridDim.x * kTopkWarps) {
    const float* row = scores + (size_t)n * M;
    float lv = -INFINITY;  // lane j < k: value of the j-th entry
    int li = 0x7fffffff;   // and its expert
    float thr = -INFINITY; // value of the k-th entry (-infinity while fewer than k)
    for (int base = 0; base < M; base += 128 * kTopkUnroll) {
      float4 x[kTopkUnroll];
#pragma unroll
      for (int u = 0; u < kTopkUnroll; ++u) {
        const int e = base + 128 * u + 4 * lane;
        x[u] = e < M ? __ldcs(reinterpret_cast<const float4*>(row + e))  // M % 8 == 0: all four or none
                     : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      }
#pragma unroll
      for (int u = 0; u < kTopkUnroll; ++u) {
        const int e0 = base + 128 * u;
        if (e0 >= M) break;
        const bool valid = e0 + 4 * lane < M;
        const float lmax = fmaxf(fmaxf(x[u].x, x[u].y), fmaxf(x[u].z, x[u].w));
        const bool first = e0 == 0;
        const float floor0 = first ? warp_kth_largest(valid ? lmax : -INFINITY, k, lane) : 0.f;
        const bool cand = valid && (first ? lmax >= floor0 : lmax > thr);
        unsigned mask = __ballot_sync(0xffffffffu, cand);
        while (mask) {
          const int src = __ffs(mask) - 1;
          mask &= mask - 1;
          const float xs[4] = {__shfl_sync(0xffffffffu, x[u].x, src), __shfl_sync(0xffffffffu, x[u].y, src),
                               __shfl_sync(0xffffffffu, x[u].z, src), __shfl_sync(0xffffffffu, x[u].w, src)};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float xv = xs[q];
            if (xv > thr && (!first || xv >= floor0)) {  // warp-uniform
              const int pos = __popc(__ballot_sync(0xffffffffu, lane < k && lv >= xv));
              const float up_v = __shfl_up_sync(0xffffffffu, lv, 1);
              const int up_i = __shfl_up_sync(0xffffffffu, li, 1);
              if (lane > pos && lane < k) {
                lv = up_v;
                li = up_i;
              }
              if (lane == pos) {
                lv = xv;
                li = e0 + 4 * src + q;
              }
              thr = __shfl_sync(0xffffffffu, lv, k - 1);
            }
          }
        }
      }
    }
    warp_write_selection(a, n, lane, lv, li);
    __syncwarp();
  }
}

}  // namespace

cudaError_t launch_threshold_topk(const RouteArgs& a, const float* scores) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = (a.N + kTopkWarps - 1) / kTopkWarps;
  if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
  threshold_topk_kernel<<<(unsigned)blocks, kTopkWarps * 32, 0, a.stream>>>(a, scores);
  return cudaGetLastError();
}

}  // namespace more

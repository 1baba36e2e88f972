// Small-batch (decode-sized) MoRE routing kernel on CUDA cores: one CTA of 16 warps
// per token, so that one token's reads of R1 and R2 are spread over 512 threads.
//
// Per token, following "MoRE: Scaling mixture of experts with hardware-aware
// low-rank routing", App. F, Algorithm 1 (z accumulated in fp32, one sweep over
// the experts with a running top-k) and Fig. 12 (softmax over the k selected
// logits):
//   1. z = x . R1: warp w sums hidden rows w*32 + lane + 512 j, 16 outputs per pass
//      with a shuffle reduce-scatter; the sixteen warps' partial sums are added in
//      shared memory, and z is carried as the bf16 pair z_hi + z_lo (finer than
//      Algorithm 1's single bf16), as in every kernel of this library.
//   2. warp w takes the 256-expert blocks w, w + 16, ...: lane l the experts
//      8 l .. 8 l + 7 of a block (one 16-byte load per R2 row), into a sorted
//      running top-k of its own (strict '>' insertion in increasing expert order,
//      so on equal logits the lower expert index stays ahead).
//   3. k warp-wide arg-max rounds merge each warp's lanes, then warp 0 merges the
//      sixteen warp lists in routing order, applies the softmax and writes the outputs
//      and one atomic count per selection.
#include <atomic>

#include "more_internal.cuh"
#include "warp_simt.cuh"

namespace more {
namespace {

constexpr int kWarpsPerBlock = 16;
constexpr int kRMax = 128;

// The same with warp w taking hidden rows w*32 + lane + 512 j (all 16 warps on one token).
__device__ __forceinline__ void warp_partial_z16(const __nv_bfloat16* __restrict__ x,
                                                 const __nv_bfloat16* __restrict__ R1, int h, int r, int b,
                                                 int warp, int lane, float& value, int& index) {
  warp_partial_z16_strided(x, R1, h, r, b, warp * 32 + lane, kWarpsPerBlock * 32, lane, value, index);
}

// The same for 32 columns b .. b + 31 (r a multiple of 32): every hidden row's 64-byte slice of
// R1 is loaded at once, and the 5-step reduce-scatter leaves column b + lane on lane `lane`.
__device__ __forceinline__ float warp_partial_z32(const __nv_bfloat16* __restrict__ x,
                                                  const __nv_bfloat16* __restrict__ R1, int h, int r, int b,
                                                  int warp, int lane) {
  constexpr int kStride = kWarpsPerBlock * 32;
  float acc[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) acc[j] = 0.f;
  for (int t0 = warp * 32 + lane; t0 < h; t0 += 4 * kStride) {
    float xt[4];
    uint4 w[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int t = t0 + j * kStride;
      const bool ok = t < h;
      xt[j] = ok ? __bfloat162float(x[t]) : 0.f;
      const uint4* src = reinterpret_cast<const uint4*>(R1 + (size_t)(ok ? t : 0) * r + b);
#pragma unroll
      for (int q = 0; q < 4; ++q) w[j][q] = ok ? __ldg(src + q) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const __nv_bfloat162* wp = reinterpret_cast<const __nv_bfloat162*>(&w[j][q]);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float2 f = __bfloat1622float2(wp[u]);
          acc[8 * q + 2 * u] = fmaf(xt[j], f.x, acc[8 * q + 2 * u]);
          acc[8 * q + 2 * u + 1] = fmaf(xt[j], f.y, acc[8 * q + 2 * u + 1]);
        }
      }
  }
  // reduce-scatter: after the step with distance dd a lane keeps the half of its columns
  // selected by its own bit dd; lane L ends with column L
#pragma unroll
  for (int dd = 16, wd = 16; dd >= 1; dd >>= 1, wd >>= 1) {
    const bool up = lane & dd;
#pragma unroll
    for (int q = 0; q < wd; ++q) {
      const float send = up ? acc[q] : acc[q + wd];
      acc[q] = (up ? acc[q + wd] : acc[q]) + __shfl_xor_sync(0xffffffffu, send, dd);
    }
  }
  return acc[0];
}

// Logits of this lane's 8 experts e0 .. e0 + 7 (one 16-byte load per R2 row, batches of
// 16 rows whose loads are issued together); zs holds z_i as the bf16 pair sum.  ok is false
// for a lane past the last expert.
__device__ __forceinline__ void lane_logits8(const RouteArgs& a, const float* zs, int e0, bool ok, float* acc) {
  const uint4* src = reinterpret_cast<const uint4*>(a.R2) + (ok ? (e0 >> 3) : 0);
  const size_t rowv = (size_t)(a.M >> 3);
#pragma unroll
  for (int q = 0; q < 8; ++q) acc[q] = 0.f;
  for (int i0 = 0; i0 < a.r; i0 += 16) {  // r is a multiple of 16
    uint4 w[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) w[j] = ok ? __ldg(src + (size_t)(i0 + j) * rowv) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float zi = zs[i0 + j];
      const __nv_bfloat162* wp = reinterpret_cast<const __nv_bfloat162*>(&w[j]);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = __bfloat1622float2(wp[q]);
        acc[2 * q] = fmaf(zi, f.x, acc[2 * q]);
        acc[2 * q + 1] = fmaf(zi, f.y, acc[2 * q + 1]);
      }
    }
  }
}

template <int K>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    small_n_route_kernel(RouteArgs a) {
  __shared__ float zpart[kWarpsPerBlock][kRMax];
  __shared__ float zs[kRMax];
  __shared__ float pv[kWarpsPerBlock][K];
  __shared__ int pe[kWarpsPerBlock][K];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (a.zero_counts) {
    // a single-token call on one CTA: the counts are zeroed here instead of by a separate
    // memset, and this CTA's own atomics below follow the barrier
    for (int i = threadIdx.x; i < a.M; i += blockDim.x) a.out_count[i] = 0;
    __syncthreads();
  }
  for (int64_t n = blockIdx.x; n < a.N; n += gridDim.x) {
    // 1. z = x . R1 (32 columns per pass where r allows, else 16)
    const __nv_bfloat16* x = a.X + (size_t)n * a.h;
    if ((a.r & 31) == 0) {
      for (int b = 0; b < a.r; b += 32) zpart[warp][b + lane] = warp_partial_z32(x, a.R1, a.h, a.r, b, warp, lane);
    } else {
      for (int b = 0; b < a.r; b += 16) {
        float v;
        int i;
        warp_partial_z16(x, a.R1, a.h, a.r, b, warp, lane, v, i);
        if ((lane & 1) == 0) zpart[warp][i] = v;
      }
    }
    __syncthreads();
    if (threadIdx.x < a.r) {
      float z = 0.f;
#pragma unroll
      for (int w = 0; w < kWarpsPerBlock; ++w) z += zpart[w][threadIdx.x];
      zs[threadIdx.x] = split_bf16_pair(z);
    }
    __syncthreads();
    // 2. this warp's 256-expert blocks
    TopList<K> list;
    list.init();
    for (int eb = 256 * warp; eb < a.M; eb += 256 * kWarpsPerBlock) {
      const int e0 = eb + 8 * lane;
      const bool ok = e0 < a.M;  // M is a multiple of 8: the lane's 8 experts are all in range
      float acc[8];
      lane_logits8(a, zs, e0, ok, acc);
      if (ok) {
#pragma unroll
        for (int q = 0; q < 8; ++q) list.insert(acc[q], e0 + q);
      }
    }
    // 3. merge: lanes, then warps
    float v;
    int e;
    warp_merge_topk<K>(list, a.k, lane, v, e);
    if (lane < K) {
      pv[warp][lane] = v;
      pe[warp][lane] = e;
    }
    __syncthreads();
    if (warp == 0) {
      TopList<K> all;
      all.init();
      for (int q = lane; q < kWarpsPerBlock * K; q += 32)
        if (q % K < a.k) all.insert_any(pv[q / K][q % K], pe[q / K][q % K]);
      warp_merge_topk<K>(all, a.k, lane, v, e);
      warp_write_selection(a, n, lane, v, e);
    }
    __syncthreads();
  }
}

// Merge of two (running maximum, sum of exp(l - maximum)) pairs, App. F eq. (8).
__device__ __forceinline__ void merge_max_sum(float& m, float& s, float om, float os) {
  const float nm = fmaxf(m, om);
  if (nm == -INFINITY) return;  // both empty
  s = (m == -INFINITY ? 0.f : s * expf(m - nm)) + (om == -INFINITY ? 0.f : os * expf(om - nm));
  m = nm;
}

constexpr int kStatTokens = 4;  // tokens per iteration of the statistics kernel

// Logits of this lane's 8 experts e0 .. e0 + 7 for kStatTokens tokens at once (one
// 16-byte load per R2 row, shared by the tokens); zs[j][i] holds token j's z_i.
__device__ __forceinline__ void lane_logits8_tokens(const RouteArgs& a, const float (*zs)[kRMax], int e0, bool ok,
                                                    float (&acc)[kStatTokens][8]) {
  const uint4* src = reinterpret_cast<const uint4*>(a.R2) + (ok ? (e0 >> 3) : 0);
  const size_t rowv = (size_t)(a.M >> 3);
#pragma unroll
  for (int j = 0; j < kStatTokens; ++j)
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[j][q] = 0.f;
  for (int i0 = 0; i0 < a.r; i0 += 8) {
    uint4 w[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) w[u] = ok ? __ldg(src + (size_t)(i0 + u) * rowv) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const __nv_bfloat162* wp = reinterpret_cast<const __nv_bfloat162*>(&w[u]);
      float f[8];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 t = __bfloat1622float2(wp[q]);
        f[2 * q] = t.x;
        f[2 * q + 1] = t.y;
      }
#pragma unroll
      for (int j = 0; j < kStatTokens; ++j) {
        const float zi = zs[j][i0 + u];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[j][q] = fmaf(zi, f[q], acc[j][q]);
      }
    }
  }
}

// Training statistics of App. F, Algorithm 2 (eqs. (6)-(8)).  A CTA of 16 warps takes
// kStatTokens tokens per iteration (grid-stride): warps 4 j .. 4 j + 3 project token j
// (each a quarter of the hidden rows); then every warp takes its 256-expert blocks for all
// the tokens at once, so each R2 row load serves every token.  Sweep 1 keeps, per lane and
// token, the running maximum m and the rescaled sum Z (eq. (8)) and merges lanes, then
// warps; sweep 2 recomputes the same logits and adds exp(l - m) / Z into the CTA's column
// sums in shared memory.  Each expert belongs to one lane of one warp, so the shared sums
// need no atomics; at the end each CTA adds its sums to psum, one atomic per expert.
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    train_stats_kernel(RouteArgs a, float* __restrict__ out_m, float* __restrict__ out_Z,
                       float* __restrict__ out_psum) {
  static_assert(kWarpsPerBlock == 4 * kStatTokens, "four warps project each token");
  extern __shared__ float psum_s[];  // M column sums of this CTA
  __shared__ float zpart[kWarpsPerBlock][kRMax];
  __shared__ float zs[kStatTokens][kRMax];
  __shared__ float wm[kWarpsPerBlock][kStatTokens], wz[kWarpsPerBlock][kStatTokens];
  __shared__ float tok_m[kStatTokens], tok_z[kStatTokens];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = threadIdx.x; e < a.M; e += blockDim.x) psum_s[e] = 0.f;
  for (int64_t n0 = (int64_t)blockIdx.x * kStatTokens; n0 < a.N; n0 += (int64_t)gridDim.x * kStatTokens) {
    const int nt = a.N - n0 < kStatTokens ? (int)(a.N - n0) : kStatTokens;
    // z of token j = warp / 4 (a token past the batch end projects token n0 instead; it is not used)
    {
      const int j = warp >> 2;
      const __nv_bfloat16* x = a.X + (size_t)(n0 + (j < nt ? j : 0)) * a.h;
      for (int b = 0; b < a.r; b += 16) {
        float v;
        int i;
        warp_partial_z16_strided(x, a.R1, a.h, a.r, b, (warp & 3) * 32 + lane, 128, lane, v, i);
        if ((lane & 1) == 0) zpart[warp][i] = v;
      }
    }
    __syncthreads();
    for (int q = threadIdx.x; q < kStatTokens * a.r; q += blockDim.x) {
      const int j = q / a.r, i = q - j * a.r;
      zs[j][i] = split_bf16_pair(zpart[4 * j][i] + zpart[4 * j + 1][i] + zpart[4 * j + 2][i] + zpart[4 * j + 3][i]);
    }
    __syncthreads();
    // sweep 1: running maximum and rescaled sum per token
    float lm[kStatTokens], ls[kStatTokens];
#pragma unroll
    for (int j = 0; j < kStatTokens; ++j) {
      lm[j] = -INFINITY;
      ls[j] = 0.f;
    }
    for (int eb = 256 * warp; eb < a.M; eb += 256 * kWarpsPerBlock) {
      const int e0 = eb + 8 * lane;
      const bool ok = e0 < a.M;  // M is a multiple of 8: the lane's 8 experts are all in range
      float acc[kStatTokens][8];
      lane_logits8_tokens(a, zs, e0, ok, acc);
      if (ok) {
#pragma unroll
        for (int j = 0; j < kStatTokens; ++j) {
          float bm = acc[j][0];
#pragma unroll
          for (int q = 1; q < 8; ++q) bm = fmaxf(bm, acc[j][q]);
          float bs = 0.f;
#pragma unroll
          for (int q = 0; q < 8; ++q) bs += expf(acc[j][q] - bm);
          merge_max_sum(lm[j], ls[j], bm, bs);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kStatTokens; ++j) {
#pragma unroll
      for (int d = 16; d > 0; d >>= 1) {
        const float om = __shfl_xor_sync(0xffffffffu, lm[j], d), os = __shfl_xor_sync(0xffffffffu, ls[j], d);
        merge_max_sum(lm[j], ls[j], om, os);
      }
      if (lane == 0) {
        wm[warp][j] = lm[j];
        wz[warp][j] = ls[j];
      }
    }
    __syncthreads();
    if (threadIdx.x < kStatTokens) {
      const int j = threadIdx.x;
      float m = -INFINITY, sz = 0.f;
      for (int w = 0; w < kWarpsPerBlock; ++w) merge_max_sum(m, sz, wm[w][j], wz[w][j]);
      tok_m[j] = m;
      tok_z[j] = sz;
      if (j < nt) {
        out_m[n0 + j] = m;
        out_Z[n0 + j] = sz;
      }
    }
    __syncthreads();
    // sweep 2: the tokens' softmax probabilities into the column sums
    float m[kStatTokens], inv_z[kStatTokens];
#pragma unroll
    for (int j = 0; j < kStatTokens; ++j) {
      m[j] = tok_m[j];
      inv_z[j] = 1.f / tok_z[j];
    }
    for (int eb = 256 * warp; eb < a.M; eb += 256 * kWarpsPerBlock) {
      const int e0 = eb + 8 * lane;
      const bool ok = e0 < a.M;
      float acc[kStatTokens][8];
      lane_logits8_tokens(a, zs, e0, ok, acc);
      if (ok) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float add = 0.f;
#pragma unroll
          for (int j = 0; j < kStatTokens; ++j)
            if (j < nt) add += expf(acc[j][q] - m[j]) * inv_z[j];
          psum_s[e0 + q] += add;
        }
      }
    }
    __syncthreads();  // zs and tok_m/tok_z are rewritten by the next iteration
  }
  __syncthreads();
  for (int e = threadIdx.x; e < a.M; e += blockDim.x) atomicAdd(out_psum + e, psum_s[e]);
}

template <int K>
cudaError_t launch_k(const RouteArgs& a) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = a.N;  // one CTA per token, up to 4 resident per SM
  const int64_t cap = (int64_t)sms * 4;
  if (blocks > cap) blocks = cap;
  small_n_route_kernel<K><<<(unsigned)blocks, kWarpsPerBlock * 32, 0, a.stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_train_stats(const RouteArgs& a, float* out_m, float* out_Z, float* out_psum) {
  if (a.N == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const size_t smem = sizeof(float) * (size_t)a.M;
  static std::atomic<int> configured[64] = {};
  if (dev >= 0 && dev < 64 && !configured[dev].load(std::memory_order_acquire)) {
    cudaError_t e = cudaFuncSetAttribute(train_stats_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(sizeof(float) * MORE_STATS_MMAX));
    if (e != cudaSuccess) return e;
    configured[dev].store(1, std::memory_order_release);
  }
  // tokens are independent; a CTA keeps its column sums over its tokens (one CTA per SM fits)
  int64_t blocks = (a.N + kStatTokens - 1) / kStatTokens;
  const int64_t cap = (int64_t)sms;
  if (blocks > cap) blocks = cap;
  train_stats_kernel<<<(unsigned)blocks, kWarpsPerBlock * 32, smem, a.stream>>>(a, out_m, out_Z, out_psum);
  return cudaGetLastError();
}

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

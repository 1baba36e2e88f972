// CUDA-core building blocks shared by the small-N and cluster kernels and the unfused path.
#pragma once
#include "more_internal.cuh"

namespace more {

// Sorted running top-k of one lane: entries in routing order (larger value
// first; on equal values the earlier-inserted, i.e. lower, expert first).
template <int K>
struct TopList {
  float v[K];
  int i[K];
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int p = 0; p < K; ++p) {
      v[p] = -INFINITY;
      i[p] = 0x7fffffff;
    }
  }
  // Insert (x, e) if it beats the current k-th entry.  Experts arrive in
  // increasing index order, so a strict comparison keeps the lower index ahead.
  __device__ __forceinline__ void insert(float x, int e) {
    if (!(x > v[K - 1])) return;
#pragma unroll
    for (int p = K - 1; p > 0; --p) {
      if (x > v[p - 1]) {
        v[p] = v[p - 1];
        i[p] = i[p - 1];
      } else if (x > v[p]) {
        v[p] = x;
        i[p] = e;
      }
    }
    if (x > v[0]) {
      v[0] = x;
      i[0] = e;
    }
  }
  // Insert (x, e) arriving in any order: compares by routing order, value then index.
  __device__ __forceinline__ void insert_any(float x, int e) {
    if (!goes_first(x, e, v[K - 1], i[K - 1])) return;
#pragma unroll
    for (int p = K - 1; p > 0; --p) {
      if (goes_first(x, e, v[p - 1], i[p - 1])) {
        v[p] = v[p - 1];
        i[p] = i[p - 1];
      } else if (goes_first(x, e, v[p], i[p])) {
        v[p] = x;
        i[p] = e;
      }
    }
    if (goes_first(x, e, v[0], i[0])) {
      v[0] = x;
      i[0] = e;
    }
  }
  __device__ __forceinline__ void pop() {
#pragma unroll
    for (int p = 0; p < K - 1; ++p) {
      v[p] = v[p + 1];
      i[p] = i[p + 1];
    }
    v[K - 1] = -INFINITY;
    i[K - 1] = 0x7fffffff;
  }
};

// The 16 sums z[b .. b + 16) over this warp's hidden rows tstart + kStride j (tstart holds
// the lane), reduced across the warp by a reduce-scatter: afterwards every value sits on
// two neighbouring lanes; `value` is this lane's value and `index` its z index.
__device__ __forceinline__ void warp_partial_z16_strided(const __nv_bfloat16* __restrict__ x,
                                                         const __nv_bfloat16* __restrict__ R1, int h, int r,
                                                         int b, int tstart, int kStride, int lane, float& value,
                                                         int& index) {
  float acc[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) acc[j] = 0.f;
  // batches of 4 hidden rows: all loads first, then the arithmetic, so the loads overlap
  for (int t0 = tstart; t0 < h; t0 += 4 * kStride) {
    float xt[4];
    uint4 w0[4], w1[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int t = t0 + j * kStride;
      const bool ok = t < h;
      xt[j] = ok ? __bfloat162float(x[t]) : 0.f;
      const uint4* w = reinterpret_cast<const uint4*>(R1 + (size_t)(ok ? t : 0) * r + b);
      w0[j] = ok ? __ldg(w) : make_uint4(0u, 0u, 0u, 0u);
      w1[j] = ok ? __ldg(w + 1) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __nv_bfloat162* p0 = reinterpret_cast<const __nv_bfloat162*>(&w0[j]);
      const __nv_bfloat162* p1 = reinterpret_cast<const __nv_bfloat162*>(&w1[j]);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 u = __bfloat1622float2(p0[q]);
        const float2 v = __bfloat1622float2(p1[q]);
        acc[2 * q] = fmaf(xt[j], u.x, acc[2 * q]);
        acc[2 * q + 1] = fmaf(xt[j], u.y, acc[2 * q + 1]);
        acc[8 + 2 * q] = fmaf(xt[j], v.x, acc[8 + 2 * q]);
        acc[8 + 2 * q + 1] = fmaf(xt[j], v.y, acc[8 + 2 * q + 1]);
      }
    }
  }
  // reduce-scatter: after the step with distance d a lane keeps the half selected by its bit d
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const bool hi = lane & 16;
    const float send = hi ? acc[j] : acc[j + 8];
    acc[j] = (hi ? acc[j + 8] : acc[j]) + __shfl_xor_sync(0xffffffffu, send, 16);
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const bool hi = lane & 8;
    const float send = hi ? acc[j] : acc[j + 4];
    acc[j] = (hi ? acc[j + 4] : acc[j]) + __shfl_xor_sync(0xffffffffu, send, 8);
  }
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const bool hi = lane & 4;
    const float send = hi ? acc[j] : acc[j + 2];
    acc[j] = (hi ? acc[j + 2] : acc[j]) + __shfl_xor_sync(0xffffffffu, send, 4);
  }
  {
    const bool hi = lane & 2;
    const float send = hi ? acc[0] : acc[1];
    acc[0] = (hi ? acc[1] : acc[0]) + __shfl_xor_sync(0xffffffffu, send, 2);
  }
  acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], 1);
  value = acc[0];
  index = b + ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1);
}

// z = x . R1 for one token; writes z, carried as the bf16 pair z_hi + z_lo, into zs[0..r).
__device__ __forceinline__ void warp_project_token(const __nv_bfloat16* __restrict__ x,
                                              const __nv_bfloat16* __restrict__ R1, int h, int r,
                                              float* zs, int lane) {
  for (int b = 0; b < r; b += 16) {
    float acc[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) acc[j] = 0.f;
    for (int t = lane; t < h; t += 32) {
      float xt = __bfloat162float(x[t]);
      const uint4* w = reinterpret_cast<const uint4*>(R1 + (size_t)t * r + b);
      uint4 w0 = __ldg(w), w1 = __ldg(w + 1);
      const __nv_bfloat162* p0 = reinterpret_cast<const __nv_bfloat162*>(&w0);
      const __nv_bfloat162* p1 = reinterpret_cast<const __nv_bfloat162*>(&w1);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float2 a = __bfloat1622float2(p0[q]);
        float2 c = __bfloat1622float2(p1[q]);
        acc[2 * q] = fmaf(xt, a.x, acc[2 * q]);
        acc[2 * q + 1] = fmaf(xt, a.y, acc[2 * q + 1]);
        acc[8 + 2 * q] = fmaf(xt, c.x, acc[8 + 2 * q]);
        acc[8 + 2 * q + 1] = fmaf(xt, c.y, acc[8 + 2 * q + 1]);
      }
    }
    // Reduce-scatter: after the step with distance d, a lane keeps the half of
    // its values selected by its own bit d.  Values left: 8, 4, 2, 1.
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      bool hi = lane & 16;
      float send = hi ? acc[j] : acc[j + 8];
      float keep = hi ? acc[j + 8] : acc[j];
      acc[j] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      bool hi = lane & 8;
      float send = hi ? acc[j] : acc[j + 4];
      float keep = hi ? acc[j + 4] : acc[j];
      acc[j] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      bool hi = lane & 4;
      float send = hi ? acc[j] : acc[j + 2];
      float keep = hi ? acc[j + 2] : acc[j];
      acc[j] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    {
      bool hi = lane & 2;
      float send = hi ? acc[0] : acc[1];
      float keep = hi ? acc[1] : acc[0];
      acc[0] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
    acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], 1);
    int j = ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1);
    if ((lane & 1) == 0) zs[b + j] = split_bf16_pair(acc[0]);
  }
}


// Merge the 32 lane lists of a warp in routing order: k rounds of a warp-wide
// arg-max.  Lane j < k receives the j-th selection in (v, e).
template <int K>
__device__ __forceinline__ void warp_merge_topk(TopList<K>& list, int k, int lane, float& v, int& e) {
  v = -INFINITY;
  e = 0;
  for (int j = 0; j < k; ++j) {
    float bv = list.v[0];
    int bi = list.i[0];
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) {
      float ov = __shfl_xor_sync(0xffffffffu, bv, d);
      int oi = __shfl_xor_sync(0xffffffffu, bi, d);
      if (goes_first(ov, oi, bv, bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (list.i[0] == bi) list.pop();
    if (lane == j) {
      v = bv;
      e = bi;
    }
  }
}

// Softmax over the k selections held by lanes 0..k-1, then the outputs of token n.
__device__ __forceinline__ void warp_write_selection(const RouteArgs& a, int64_t n, int lane, float v,
                                                     int e) {
  float top = __shfl_sync(0xffffffffu, v, 0);
  float ex = (lane < a.k) ? expf(v - top) : 0.f;
  float sum = ex;
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, d);
  if (lane < a.k) {
    size_t o = (size_t)n * a.k + lane;
    a.out_idx[o] = e;
    a.out_gate[o] = ex / sum;
    if (a.out_logits) a.out_logits[o] = v;
    if ((unsigned)e < (unsigned)a.M) atomicAdd(a.out_count + e, 1);
  }
}

}  // namespace more

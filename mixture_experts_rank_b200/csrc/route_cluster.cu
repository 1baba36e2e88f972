// Decode-sized MoRE routing on a thread-block cluster: the experts of 8 tokens are split over
// a cluster of 8 CTAs, and the partial top-k lists are merged through distributed shared
// memory (DSMEM).  For one token the single-CTA kernel leaves the weights' 393 KB (h = 2048,
// r = 32, M = 4096) to one SM; here eight SMs share them.
//
// Per cluster (tokens n0 .. n0 + 7), following "MoRE: Scaling mixture of experts with
// hardware-aware low-rank routing", App. F, Algorithm 1 (z accumulated in fp32, a sweep over
// the experts with a running top-k) and Fig. 12 (softmax over the k selected logits):
//   1. CTA q sums z = x . R1 over its eighth of the hidden rows into its own shared memory.
//      The rows and the tokens' x come in chunks of 16 KB of R1, staged in shared memory by
//      coalesced 16-byte loads that are all in flight at once; then warp w takes every
//      eighth row of the chunk and lane c the columns c, c + 32, ..., for all tokens, and
//      the eight warps' sums are added in warp order;                   cluster barrier
//   2. every CTA adds the eight partial sums (read through DSMEM, in rank order, so every
//      CTA holds the same z) and carries z as the bf16 pair z_hi + z_lo, as every kernel of
//      this library does;
//   3. CTA q takes its eighth of the experts, 512 at a time: thread i the experts 2 i and
//      2 i + 1 of the pass for all eight tokens, with its r R2 loads issued together; warp t
//      keeps token t's running top-k;
//   4. every CTA writes its k candidates per token into CTA 0's shared memory;
//                                                                         cluster barrier
//   5. CTA 0 merges the 8 k candidates of each token in routing order (larger logit first,
//      lower expert on ties), applies the softmax and writes the outputs and one atomic
//      count per selection.
// Every CTA reaches both barriers (tokens past N are computed on zeros and not written), and
// after the second barrier only CTA 0 reads shared memory, its own.  A launch of one cluster
// may zero the counts itself (each CTA its eighth of the experts, before the first barrier,
// which orders those stores before CTA 0's atomics), so that no memset is issued.
#include <cooperative_groups.h>

#include <atomic>

#include "more_internal.cuh"
#include "warp_simt.cuh"

namespace more {
namespace {

namespace cg = cooperative_groups;

constexpr int kCluster = 8;      // CTAs per cluster
constexpr int kTok = 8;          // tokens per cluster, one warp each in steps 3 and 5
constexpr int kThreads = kTok * 32;
constexpr int kWarps = kThreads / 32;
constexpr int kRMax = 128;
constexpr int kWBytes = 16384;   // R1 rows staged per chunk in step 1: 8192 / r rows (a multiple of 8)
constexpr int kRowsMax = 512;    // ... at most (r = 16)
constexpr int kPass = 2 * kThreads;  // experts per pass in step 3
static_assert(kTok == 8, "a row's x (bf16) and z (fp32) of all tokens are read as 16 and 32 bytes");

__host__ __device__ __forceinline__ int chunk_rows(int r) {
  const int n = (kWBytes / 2 / r) & ~7;
  return n < kRowsMax ? n : kRowsMax;
}

// Dynamic shared memory, sized by r (byte offsets; the same in every CTA of a cluster, so a
// peer's buffer sits at the same offset in its own shared memory).
struct Layout {
  uint32_t zpart;  // [kTok][r] fp32: this CTA's partial z (read by the whole cluster)
  uint32_t zs;     // [r][kTok] fp32: z as the bf16 pair sum, the 8 tokens of a row together
  uint32_t part;   // [kWarps][kTok][r] fp32: step 1, each warp's sums
  uint32_t u;      // step 1: R1 chunk [rows][r] bf16 and x [rows][kTok] bf16;
                   // step 3: logits of one pass [kTok][kPass] fp32
  uint32_t cand_v; // [kCluster][kTok][MORE_KMAX] fp32: CTA 0's table of every CTA's candidates
  uint32_t cand_e; // [kCluster][kTok][MORE_KMAX] int32
  uint32_t total;
};

__host__ __device__ __forceinline__ Layout layout_for(int r) {
  Layout L;
  uint32_t off = 0;
  L.zpart = off;
  off += kTok * r * 4;
  L.zs = off;
  off += kTok * r * 4;
  L.part = off;
  off += kWarps * kTok * r * 4;
  L.u = off;
  const uint32_t rows = (uint32_t)chunk_rows(r);
  const uint32_t st = rows * r * 2 + kTok * rows * 2, lg = kTok * kPass * 4;
  const uint32_t un = st > lg ? st : lg;
  off += (un + 15) & ~15u;
  L.cand_v = off;
  off += kCluster * kTok * MORE_KMAX * 4;
  L.cand_e = off;
  off += kCluster * kTok * MORE_KMAX * 4;
  L.total = off;
  return L;
}

// Resident CTAs per SM: four (64 registers) up to k = 8, three (80 registers) above, where the
// running top-k lists need the room.
template <int K>
__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kThreads, K <= 8 ? 4 : 3)
    cluster_route_kernel(RouteArgs a) {
  extern __shared__ float4 smem4[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(smem4);
  const Layout L = layout_for(a.r);
  float* zpart = reinterpret_cast<float*>(smem + L.zpart);
  float* zs = reinterpret_cast<float*>(smem + L.zs);
  __nv_bfloat16* stw = reinterpret_cast<__nv_bfloat16*>(smem + L.u);
  float* part = reinterpret_cast<float*>(smem + L.part);
  float* lg = reinterpret_cast<float*>(smem + L.u);
  float* cand_v = reinterpret_cast<float*>(smem + L.cand_v);
  int* cand_e = reinterpret_cast<int*>(smem + L.cand_e);
  cg::cluster_group cluster = cg::this_cluster();
  const unsigned q = cluster.block_rank();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n0 = (int64_t)(blockIdx.x / kCluster) * kTok;
  const int nt = a.N - n0 < kTok ? (int)(a.N - n0) : kTok;
  const int r = a.r;

  // this CTA's experts [eb, ee) in step 3 (and its share of the counts to zero)
  const int me = ((a.M + kCluster - 1) / kCluster + 7) & ~7;
  const int eb = (int)q * me < a.M ? (int)q * me : a.M;
  const int ee = eb + me < a.M ? eb + me : a.M;
  if (a.zero_counts)
    for (int e = eb + (int)threadIdx.x; e < ee; e += kThreads) a.out_count[e] = 0;

  // 1. partial z over hidden rows [hb, he) of this CTA
  const int hs = ((a.h + kCluster - 1) / kCluster + 7) & ~7;  // a multiple of 8 rows: 16-byte aligned x chunks
  const int hb = (int)q * hs < a.h ? (int)q * hs : a.h;
  const int he = hb + hs < a.h ? hb + hs : a.h;
  const int rows = chunk_rows(r);
  __nv_bfloat16* stx = stw + rows * r;  // [rows][kTok]: the 8 tokens' x of a row in 16 bytes
  for (int c0 = hb; c0 < he; c0 += rows) {
    const int nr = he - c0 < rows ? he - c0 : rows;  // rows of this chunk, a multiple of 8
    // R1 rows [c0, c0 + nr) are contiguous: nr * r / 8 chunks of 16 bytes
    const uint4* wsrc = reinterpret_cast<const uint4*>(a.R1 + (size_t)c0 * r);
    uint4* wdst = reinterpret_cast<uint4*>(stw);
    const int nw = nr * r / 8;
    for (int i = threadIdx.x; i < nw; i += kThreads) wdst[i] = __ldg(wsrc + i);
    // x of token t over the same rows: nr / 8 chunks of 16 bytes per token, stored transposed
    // (tokens past N as zeros)
    const int nx = nr / 8;
    for (int i = threadIdx.x; i < kTok * nx; i += kThreads) {
      const int t = i / nx, c = i % nx;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (t < nt) v = __ldg(reinterpret_cast<const uint4*>(a.X + (size_t)(n0 + t) * a.h + c0) + c);
      const __nv_bfloat16* b = reinterpret_cast<const __nv_bfloat16*>(&v);
#pragma unroll
      for (int u = 0; u < 8; ++u) stx[(8 * c + u) * kTok + t] = b[u];
    }
    __syncthreads();
    // Block m of 32 columns: lane c takes column 32 m + c.  Where only 16 columns remain
    // (r % 32 == 16) the half warps take alternate rows and add their sums with a shuffle.
    // The warp's sums over its rows of each chunk go to its own slots of `part`, added in
    // chunk order.
    for (int m = 0; 32 * m < r; ++m) {
      const bool half = r - 32 * m < 32;
      const int c = 32 * m + (half ? (lane & 15) : lane);
      const int slot = half ? (lane >> 4) : 0, step = half ? 2 * kWarps : kWarps;
      float acc[kTok];
#pragma unroll
      for (int t = 0; t < kTok; ++t) acc[t] = 0.f;
      for (int j = warp + slot * kWarps; j < nr; j += step) {
        const float wv = __bfloat162float(stw[j * r + c]);
        const uint4 xq = *reinterpret_cast<const uint4*>(stx + j * kTok);  // same address across a half warp
        const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&xq);
#pragma unroll
        for (int t2 = 0; t2 < kTok / 2; ++t2) {
          const float2 xv = __bfloat1622float2(x2[t2]);
          acc[2 * t2] = fmaf(xv.x, wv, acc[2 * t2]);
          acc[2 * t2 + 1] = fmaf(xv.y, wv, acc[2 * t2 + 1]);
        }
      }
      if (half) {
#pragma unroll
        for (int t = 0; t < kTok; ++t) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], 16);
      }
      if (slot == 0) {
        float* pw = part + warp * kTok * r + c;
#pragma unroll
        for (int t = 0; t < kTok; ++t) pw[t * r] = c0 == hb ? acc[t] : pw[t * r] + acc[t];
      }
    }
    __syncthreads();  // the chunk is consumed before the next one overwrites it
  }
  for (int idx = threadIdx.x; idx < kTok * r; idx += kThreads) {
    const int t = idx / r, i = idx % r;
    float z = 0.f;
    if (t < nt && he > hb)  // a CTA without hidden rows wrote no sums
#pragma unroll
      for (int w = 0; w < kWarps; ++w) z += part[(w * kTok + t) * r + i];
    zpart[t * r + i] = z;
  }
  cluster.sync();

  // 2. z = the sum of the eight partials, in rank order
  for (int idx = threadIdx.x; idx < kTok * r; idx += kThreads) {
    const int t = idx / r, i = idx % r;
    float z = 0.f;
#pragma unroll
    for (int p = 0; p < kCluster; ++p) z += cluster.map_shared_rank(zpart, p)[t * r + i];
    zs[i * kTok + t] = t < nt ? split_bf16_pair(z) : 0.f;  // [r][kTok]
  }
  __syncthreads();

  // 3. logits of experts [eb, ee), 512 per pass; warp t keeps token t's running top-k
  TopList<K> list;
  list.init();
  for (int p0 = eb; p0 < ee; p0 += kPass) {
    const int e = p0 + 2 * (int)threadIdx.x;  // experts e and e + 1 (both < ee when e < ee: M, me % 8 == 0)
    float acc0[kTok], acc1[kTok];
#pragma unroll
    for (int t = 0; t < kTok; ++t) acc0[t] = acc1[t] = 0.f;
    if (e < ee) {
      const __nv_bfloat162* col = reinterpret_cast<const __nv_bfloat162*>(a.R2 + e);
      const size_t stride = (size_t)(a.M / 2);
      for (int i0 = 0; i0 < r; i0 += 16) {  // r % 16 == 0; each batch's 16 loads are in flight together
        __nv_bfloat162 w[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) w[u] = col[(size_t)(i0 + u) * stride];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const float2 wf = __bfloat1622float2(w[u]);
          const float4 za = *reinterpret_cast<const float4*>(zs + (i0 + u) * kTok);  // same address across the CTA
          const float4 zb = *reinterpret_cast<const float4*>(zs + (i0 + u) * kTok + 4);
          const float zv[kTok] = {za.x, za.y, za.z, za.w, zb.x, zb.y, zb.z, zb.w};
#pragma unroll
          for (int t = 0; t < kTok; ++t) {
            acc0[t] = fmaf(zv[t], wf.x, acc0[t]);
            acc1[t] = fmaf(zv[t], wf.y, acc1[t]);
          }
        }
      }
    }
    __syncthreads();  // the previous pass's logits are merged
#pragma unroll
    for (int t = 0; t < kTok; ++t)
      *reinterpret_cast<float2*>(&lg[t * kPass + 2 * threadIdx.x]) = make_float2(acc0[t], acc1[t]);
    __syncthreads();
#pragma unroll 4
    for (int j = 0; j < kPass / 32; ++j) {  // this lane's experts, in increasing order
      const int pe = p0 + lane + 32 * j;
      if (pe < ee) list.insert(lg[warp * kPass + lane + 32 * j], pe);
    }
  }

  // 4. this CTA's k best of token `warp`, into CTA 0's candidate table
  float v;
  int e;
  warp_merge_topk<K>(list, a.k, lane, v, e);
  if (lane < a.k) {
    cluster.map_shared_rank(cand_v, 0)[(q * kTok + warp) * MORE_KMAX + lane] = v;
    cluster.map_shared_rank(cand_e, 0)[(q * kTok + warp) * MORE_KMAX + lane] = e;
  }
  cluster.sync();

  // 5. CTA 0 merges the cluster's candidates of token `warp` and writes its outputs
  if (q == 0 && warp < nt) {
    TopList<K> all;
    all.init();
    for (int p = lane; p < kCluster * a.k; p += 32) {
      const int c = p / a.k, j = p % a.k;
      all.insert_any(cand_v[(c * kTok + warp) * MORE_KMAX + j], cand_e[(c * kTok + warp) * MORE_KMAX + j]);
    }
    warp_merge_topk<K>(all, a.k, lane, v, e);
    warp_write_selection(a, n0 + warp, lane, v, e);
  }
}

template <int K>
cudaError_t configure_once(int dev) {
  static std::atomic<int> done[64] = {};
  if (dev >= 0 && dev < 64 && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(cluster_route_kernel<K>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)layout_for(kRMax).total);
  if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev].store(1, std::memory_order_release);
  return e;
}

template <int K>
cudaError_t launch_cluster_k(const RouteArgs& a) {
  const int64_t clusters = (a.N + kTok - 1) / kTok;
  if (clusters * kCluster > 0x7fffffffLL) return cudaErrorInvalidValue;
  if (a.zero_counts && clusters != 1) return cudaErrorInvalidValue;  // one cluster may zero the counts
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if ((e = configure_once<K>(dev)) != cudaSuccess) return e;
  cluster_route_kernel<K><<<(unsigned)(clusters * kCluster), kThreads, layout_for(a.r).total, a.stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_cluster(const RouteArgs& a) {
  if (a.N == 0) return cudaSuccess;
  switch (a.k) {
#define MORE_CASE(K) \
  case K:            \
    return launch_cluster_k<K>(a);
    MORE_CASE(1) MORE_CASE(2) MORE_CASE(3) MORE_CASE(4) MORE_CASE(5) MORE_CASE(6) MORE_CASE(7)
    MORE_CASE(8) MORE_CASE(9) MORE_CASE(10) MORE_CASE(11) MORE_CASE(12) MORE_CASE(13)
    MORE_CASE(14) MORE_CASE(15) MORE_CASE(16)
#undef MORE_CASE
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace more

// Decode-sized MoRE routing on a thread-block cluster: the experts of 8 tokens are split over
// a cluster of 8 CTAs, and the partial top-k lists are merged through distributed shared
// memory (DSMEM).  For one token the single-CTA kernel leaves the weights' 393 KB (h = 2048,
// r = 32, M = 4096) to one SM; here eight SMs share them.
//
// Per cluster (tokens n0 .. n0 + 7), following "MoRE: Scaling mixture of experts with
// hardware-aware low-rank routing", App. F, Algorithm 1 (z accumulated in fp32, a sweep over
// the experts with a running top-k) and Fig. 12 (softmax over the k selected logits):
//   1. CTA q sums z = x . R1 over its eighth of the hidden rows, warp t for token t, into
//      its own shared memory;                                             cluster barrier
//   2. every CTA adds the eight partial sums (read through DSMEM, in rank order, so every
//      CTA holds the same z) and carries z as the bf16 pair z_hi + z_lo, as every kernel of
//      this library does;
//   3. CTA q takes its eighth of the experts, 256 at a time (thread i the expert i of the
//      pass, all eight tokens), and warp t keeps token t's running top-k;
//   4. every CTA writes its k candidates per token into CTA 0's shared memory;
//                                                                         cluster barrier
//   5. CTA 0 merges the 8 k candidates of each token in routing order (larger logit first,
//      lower expert on ties), applies the softmax and writes the outputs and one atomic
//      count per selection.
// Every CTA reaches both barriers (tokens past N are computed on zeros and not written), and
// after the second barrier only CTA 0 reads shared memory, its own.
#include <cooperative_groups.h>

#include "more_internal.cuh"
#include "warp_simt.cuh"

namespace more {
namespace {

namespace cg = cooperative_groups;

constexpr int kCluster = 8;      // CTAs per cluster
constexpr int kTok = 8;          // tokens per cluster, one warp each in steps 1, 3 and 5
constexpr int kThreads = kTok * 32;
constexpr int kRMax = 128;

struct ClusterSmem {
  float zpart[kTok][kRMax];                      // this CTA's partial z (read by the whole cluster)
  float zs[kTok][kRMax];                         // z as the bf16 pair sum
  float lg[kTok][kThreads];                      // logits of one 256-expert pass
  float cand_v[kCluster][kTok][MORE_KMAX];       // CTA 0: every CTA's candidates
  int cand_e[kCluster][kTok][MORE_KMAX];
};

template <int K>
__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kThreads) cluster_route_kernel(RouteArgs a) {
  extern __shared__ float4 smem4[];
  ClusterSmem& s = *reinterpret_cast<ClusterSmem*>(smem4);
  cg::cluster_group cluster = cg::this_cluster();
  const unsigned q = cluster.block_rank();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n0 = (int64_t)(blockIdx.x / kCluster) * kTok;
  const int nt = a.N - n0 < kTok ? (int)(a.N - n0) : kTok;

  // 1. partial z over hidden rows [hb, he) of this CTA; warp t for token t
  const int hs = (a.h + kCluster - 1) / kCluster;
  const int hb = (int)q * hs, he = hb + hs < a.h ? hb + hs : a.h;
  for (int i = lane; i < kRMax; i += 32) s.zpart[warp][i] = 0.f;
  __syncwarp();
  if (warp < nt) {
    const __nv_bfloat16* x = a.X + (size_t)(n0 + warp) * a.h;
    for (int b = 0; b < a.r; b += 16) {
      float v;
      int i;
      warp_partial_z16_strided(x, a.R1, he, a.r, b, hb + lane, 32, lane, v, i);
      if ((lane & 1) == 0) s.zpart[warp][i] = v;
    }
  }
  cluster.sync();

  // 2. z = the sum of the eight partials, in rank order
  for (int idx = threadIdx.x; idx < kTok * a.r; idx += kThreads) {
    const int t = idx / a.r, i = idx % a.r;
    float z = 0.f;
#pragma unroll
    for (int p = 0; p < kCluster; ++p) z += cluster.map_shared_rank(&s.zpart[0][0], p)[t * kRMax + i];
    s.zs[t][i] = t < nt ? split_bf16_pair(z) : 0.f;
  }
  __syncthreads();

  // 3. logits of experts [eb, ee), 256 per pass; warp t keeps token t's running top-k
  const int me = ((a.M + kCluster - 1) / kCluster + 7) & ~7;
  const int eb = (int)q * me < a.M ? (int)q * me : a.M;
  const int ee = eb + me < a.M ? eb + me : a.M;
  TopList<K> list;
  list.init();
  for (int p0 = eb; p0 < ee; p0 += kThreads) {
    const int e = p0 + (int)threadIdx.x;
    float acc[kTok];
#pragma unroll
    for (int t = 0; t < kTok; ++t) acc[t] = 0.f;
    if (e < ee) {
      const __nv_bfloat16* col = a.R2 + e;
      for (int i0 = 0; i0 < a.r; i0 += 8) {
        float w[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) w[u] = __bfloat162float(col[(size_t)(i0 + u) * a.M]);
#pragma unroll
        for (int u = 0; u < 8; ++u)
#pragma unroll
          for (int t = 0; t < kTok; ++t) acc[t] = fmaf(s.zs[t][i0 + u], w[u], acc[t]);
      }
    }
    __syncthreads();  // the previous pass's logits are merged
#pragma unroll
    for (int t = 0; t < kTok; ++t) s.lg[t][threadIdx.x] = acc[t];
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kThreads / 32; ++j) {  // this lane's experts, in increasing order
      const int pe = p0 + lane + 32 * j;
      if (pe < ee) list.insert(s.lg[warp][lane + 32 * j], pe);
    }
  }

  // 4. this CTA's k best of token `warp`, into CTA 0's candidate table
  float v;
  int e;
  warp_merge_topk<K>(list, a.k, lane, v, e);
  if (lane < a.k) {
    cluster.map_shared_rank(&s.cand_v[0][0][0], 0)[(q * kTok + warp) * MORE_KMAX + lane] = v;
    cluster.map_shared_rank(&s.cand_e[0][0][0], 0)[(q * kTok + warp) * MORE_KMAX + lane] = e;
  }
  cluster.sync();

  // 5. CTA 0 merges the cluster's candidates of token `warp` and writes its outputs
  if (q == 0 && warp < nt) {
    TopList<K> all;
    all.init();
    for (int p = lane; p < kCluster * a.k; p += 32) {
      const int c = p / a.k, j = p % a.k;
      all.insert_any(s.cand_v[c][warp][j], s.cand_e[c][warp][j]);
    }
    warp_merge_topk<K>(all, a.k, lane, v, e);
    warp_write_selection(a, n0 + warp, lane, v, e);
  }
}

template <int K>
cudaError_t launch_cluster_k(const RouteArgs& a) {
  const int64_t clusters = (a.N + kTok - 1) / kTok;
  if (clusters * kCluster > 0x7fffffffLL) return cudaErrorInvalidValue;
  cluster_route_kernel<K><<<(unsigned)(clusters * kCluster), kThreads, sizeof(ClusterSmem), a.stream>>>(a);
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

// Materialise-then-top-k comparison path: the unfused low-rank router of
// "MoRE: Scaling mixture of experts with hardware-aware low-rank routing",
// App. H.6 (Fig. 24), rebuilt with this library's own kernels.
//   kernel 1: z = X . R1, carried as z_hi + z_lo, written to scratch fp32 [N][r];
//   kernel 2: l = z . R2 in fp32, written to scratch [N][M]  (the N x M tensor
//             the fused kernel never writes);
//   kernel 3: one warp per row reads l back, keeps per-lane running top-k
//             lists, merges them in routing order, applies the softmax.
// The arithmetic matches the fused path (z as a bf16 pair, fp32 logits), so both
// return the same selections up to the order of fp32 accumulation.
#include "more_internal.cuh"
#include "warp_simt.cuh"

namespace more {
namespace {

constexpr int kProjWarps = 8;

__global__ void __launch_bounds__(kProjWarps * 32)
    unfused_projection_kernel(const __nv_bfloat16* __restrict__ X, const __nv_bfloat16* __restrict__ R1,
                              int64_t N, int h, int r, float* __restrict__ z_out) {
  extern __shared__ float smem_z[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* zs = smem_z + warp * r;
  for (int64_t n = (int64_t)blockIdx.x * kProjWarps + warp; n < N; n += (int64_t)gridDim.x * kProjWarps) {
    warp_project_token(X + (size_t)n * h, R1, h, r, zs, lane);
    __syncwarp();
    for (int i = lane; i < r; i += 32) z_out[(size_t)n * r + i] = zs[i];
    __syncwarp();
  }
}

// Scores tile: 64 tokens x 128 experts per block of 256 threads; each thread
// owns 4 tokens x 8 consecutive experts.
constexpr int kTileTok = 64, kTileExp = 128;

__global__ void __launch_bounds__(256)
    unfused_scores_kernel(const float* __restrict__ z, const __nv_bfloat16* __restrict__ R2,
                          int64_t N, int r, int M, float* __restrict__ scores) {
  extern __shared__ float smem[];
  float* zt = smem;                       // [kTileTok][r]
  float* wt = smem + kTileTok * r;        // [r][kTileExp]
  const int64_t n0 = (int64_t)blockIdx.x * kTileTok;
  const int e0 = blockIdx.y * kTileExp;
  for (int q = threadIdx.x; q < kTileTok * r; q += 256) {
    int t = q / r, i = q % r;
    zt[q] = (n0 + t < N) ? z[(size_t)(n0 + t) * r + i] : 0.f;
  }
  for (int q = threadIdx.x; q < r * kTileExp; q += 256) {
    int i = q / kTileExp, c = q % kTileExp;
    wt[q] = (e0 + c < M) ? __bfloat162float(R2[(size_t)i * M + e0 + c]) : 0.f;
  }
  __syncthreads();
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;  // 16 expert groups x 16 token groups
  float acc[4][8];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;
  for (int i = 0; i < r; ++i) {
    float w[8];
#pragma unroll
    for (int b = 0; b < 8; ++b) w[b] = wt[i * kTileExp + tx * 8 + b];
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      float zv = zt[(ty * 4 + a) * r + i];
#pragma unroll
      for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(zv, w[b], acc[a][b]);
    }
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    int64_t n = n0 + ty * 4 + a;
    int e = e0 + tx * 8;
    if (n >= N) continue;
    float* dst = scores + (size_t)n * M + e;
    if (e < M) {  // M % 8 == 0, so a group of 8 is either wholly inside or wholly outside
      reinterpret_cast<float4*>(dst)[0] = make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
      reinterpret_cast<float4*>(dst)[1] = make_float4(acc[a][4], acc[a][5], acc[a][6], acc[a][7]);
    }
  }
}

constexpr int kTopkWarps = 8;

template <int K>
__global__ void __launch_bounds__(kTopkWarps * 32) unfused_topk_kernel(RouteArgs a, const float* __restrict__ scores) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int64_t n = (int64_t)blockIdx.x * kTopkWarps + warp; n < a.N; n += (int64_t)gridDim.x * kTopkWarps) {
    const float* row = scores + (size_t)n * a.M;
    TopList<K> list;
    list.init();
    for (int e = 4 * lane; e < a.M; e += 128) {
      float4 v = __ldcs(reinterpret_cast<const float4*>(row + e));  // M % 8 == 0
      list.insert(v.x, e);
      list.insert(v.y, e + 1);
      list.insert(v.z, e + 2);
      list.insert(v.w, e + 3);
    }
    float my_v;
    int my_i;
    warp_merge_topk<K>(list, a.k, lane, my_v, my_i);
    warp_write_selection(a, n, lane, my_v, my_i);
    __syncwarp();
  }
}

template <int K>
cudaError_t launch_topk(const RouteArgs& a, const float* scores, int blocks) {
  unfused_topk_kernel<K><<<blocks, kTopkWarps * 32, 0, a.stream>>>(a, scores);
  return cudaGetLastError();
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace

size_t unfused_scratch_bytes(int64_t N, int r, int M) {
  return align_up((size_t)N * r * sizeof(float), 256) + (size_t)N * M * sizeof(float);
}

float* unfused_scores_of(void* scratch, int64_t N, int r) {
  return reinterpret_cast<float*>(static_cast<char*>(scratch) + align_up((size_t)N * r * sizeof(float), 256));
}

cudaError_t launch_scores_topk(const RouteArgs& a, const float* scores) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t tblocks = (a.N + kTopkWarps - 1) / kTopkWarps;
  if (tblocks > (int64_t)sms * 16) tblocks = (int64_t)sms * 16;
  switch (a.k) {
#define MORE_CASE(K) \
  case K:            \
    return launch_topk<K>(a, scores, (int)tblocks);
    MORE_CASE(1) MORE_CASE(2) MORE_CASE(3) MORE_CASE(4) MORE_CASE(5) MORE_CASE(6) MORE_CASE(7)
    MORE_CASE(8) MORE_CASE(9) MORE_CASE(10) MORE_CASE(11) MORE_CASE(12) MORE_CASE(13)
    MORE_CASE(14) MORE_CASE(15) MORE_CASE(16)
#undef MORE_CASE
    default:
      return cudaErrorInvalidValue;
  }
}

cudaError_t launch_unfused(const RouteArgs& a, void* scratch) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  auto* z = static_cast<float*>(scratch);
  float* scores = unfused_scores_of(scratch, a.N, a.r);
  int64_t pblocks = (a.N + kProjWarps - 1) / kProjWarps;
  if (pblocks > (int64_t)sms * 8) pblocks = (int64_t)sms * 8;
  unfused_projection_kernel<<<(unsigned)pblocks, kProjWarps * 32, sizeof(float) * kProjWarps * a.r, a.stream>>>(
      a.X, a.R1, a.N, a.h, a.r, z);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  dim3 grid((unsigned)((a.N + kTileTok - 1) / kTileTok), (a.M + kTileExp - 1) / kTileExp);
  size_t smem = sizeof(float) * (size_t)(kTileTok + kTileExp) * a.r;
  if (smem > 48 * 1024) {
    err = cudaFuncSetAttribute(unfused_scores_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
  }
  unfused_scores_kernel<<<grid, 256, smem, a.stream>>>(z, a.R2, a.N, a.r, a.M, scores);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  return launch_scores_topk(a, scores);
}

}  // namespace more

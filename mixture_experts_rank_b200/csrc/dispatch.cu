// Dispatch bookkeeping after routing ("MoRE: Scaling mixture of experts with hardware-aware
// low-rank routing", App. E, Fig. 9, "Sort + Count"): the N k routing slots s = n k + j,
// stably sorted by their expert, and the per-expert offsets.  A deterministic counting
// sort in four kernels:
//   1. per-chunk histograms of the expert ids (a chunk is a contiguous run of slots);
//   2. per expert, an exclusive scan of its counts over the chunks (column scan) and the
//      expert's total;
//   3. the offsets: an exclusive scan of the totals (one CTA);
//   4. one warp per chunk walks its slots in order, 32 at a time; lanes naming the same
//      expert are ranked by lane (match-any), so every expert's slots land in slot order.
// An expert id outside [0, M) is skipped and sets MORE_DEVERR_BAD_INPUT.
//
// The shared-memory variant (M <= kSharedMMax) computes the same result with fewer, larger
// chunks, about two per SM:
//   1. each CTA counts its chunk into a shared-memory histogram of M counters and writes it
//      as one row of G[chunk][expert];
//   2. per 32 experts, eight warps each sum a band of chunks; after a shared-memory scan of
//      the eight sums, each warp rewrites its band as the column's exclusive prefix;
//   3. the offsets, as above;
//   4. each CTA walks its chunk 256 slots at a time: match-any ranks equal experts within a
//      warp, and the eight warps take their expert counters from shared memory in warp order
//      (one barrier each), so every expert's slots still land in slot order.
#include <algorithm>

#include <atomic>

#include "more_internal.cuh"

namespace more {
namespace {

constexpr int64_t kChunkSlots = 2048;
constexpr int64_t kHistCap = int64_t(1) << 26;  // histogram entries at most (256 MB)

int64_t chunk_count(int64_t S, int M) {
  const int64_t c = (S + kChunkSlots - 1) / kChunkSlots;
  const int64_t cap = std::max<int64_t>(1, kHistCap / M);
  return std::max<int64_t>(1, std::min(c, cap));
}

__global__ void dispatch_hist_kernel(const int32_t* __restrict__ idx, int64_t S, int M, int64_t chunk,
                                     int32_t* __restrict__ hist, unsigned int* status) {
  const int64_t c = blockIdx.x, b = c * chunk, end = b + chunk < S ? b + chunk : S;
  for (int64_t s = b + threadIdx.x; s < end; s += blockDim.x) {
    const int v = idx[s];
    if ((unsigned)v < (unsigned)M)
      atomicAdd(hist + c * M + v, 1);
    else
      atomicOr(status, MORE_DEVERR_BAD_INPUT);
  }
}

// hist[c][e] <- slots of expert e in chunks before c; totals[e] <- slots of expert e
__global__ void dispatch_colscan_kernel(int32_t* __restrict__ hist, int64_t nchunks, int M,
                                        int32_t* __restrict__ totals) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= M) return;
  int32_t run = 0;
  for (int64_t c = 0; c < nchunks; ++c) {
    const int32_t v = hist[c * M + e];
    hist[c * M + e] = run;
    run += v;
  }
  totals[e] = run;
}

// offsets[e] = sum of totals below e, offsets[M] = all (one CTA of 1024 threads, each a run)
__global__ void __launch_bounds__(1024) dispatch_offsets_kernel(const int32_t* __restrict__ totals, int M,
                                                                int32_t* __restrict__ offsets) {
  __shared__ int32_t part[1024];
  const int per = (M + 1023) / 1024;
  const int b = threadIdx.x * per, end = b + per < M ? b + per : M;
  int32_t run = 0;
  for (int i = b; i < end; ++i) run += totals[i];
  part[threadIdx.x] = run;
  __syncthreads();
  for (int d = 1; d < 1024; d <<= 1) {  // inclusive scan of the run sums
    const int32_t v = threadIdx.x >= d ? part[threadIdx.x - d] : 0;
    __syncthreads();
    part[threadIdx.x] += v;
    __syncthreads();
  }
  int32_t before = threadIdx.x ? part[threadIdx.x - 1] : 0;
  for (int i = b; i < end; ++i) {
    offsets[i] = before;
    before += totals[i];
  }
  if (threadIdx.x == 1023) offsets[M] = part[1023];
}

__global__ void dispatch_scatter_kernel(const int32_t* __restrict__ idx, int64_t S, int M, int64_t chunk,
                                        int64_t nchunks, int32_t* __restrict__ hist,
                                        const int32_t* __restrict__ offsets, int32_t* __restrict__ sorted) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t c = (int64_t)blockIdx.x * (blockDim.x >> 5) + warp;
  if (c >= nchunks) return;
  const int64_t b = c * chunk, end = b + chunk < S ? b + chunk : S;
  int32_t* hrow = hist + c * M;  // this chunk's running position within each expert
  const unsigned int below = (1u << lane) - 1u;
  for (int64_t s0 = b; s0 < end; s0 += 32) {
    const int64_t s = s0 + lane;
    const bool in = s < end;
    const int v = in ? idx[s] : -1;
    const bool ok = in && (unsigned)v < (unsigned)M;
    const unsigned int peers = __match_any_sync(0xffffffffu, ok ? v : -1);
    if (ok) sorted[offsets[v] + hrow[v] + __popc(peers & below)] = (int32_t)s;
    __syncwarp();
    if (ok && (peers & below) == 0) hrow[v] += __popc(peers);  // the lowest lane advances the run
    __syncwarp();
  }
}

constexpr int kSharedMMax = 32768;    // experts the shared-memory histogram holds (128 KB)
constexpr int64_t kSharedChunks = 296;  // chunks of the shared-memory variant: two per SM

int64_t shared_chunk_count(int64_t S) {
  return std::max<int64_t>(1, std::min<int64_t>(kSharedChunks, (S + kChunkSlots - 1) / kChunkSlots));
}

// Slots [c L, min(S, (c + 1) L)) of chunk c, for L = ceil(S / C).
__device__ __forceinline__ void chunk_range(int64_t S, int64_t C, int64_t c, int64_t& b, int64_t& e) {
  const int64_t L = (S + C - 1) / C;
  b = c * L < S ? c * L : S;
  e = b + L < S ? b + L : S;
}

// 1. G[c][v] = slots of chunk c naming expert v (shared-memory atomics, one coalesced row write)
__global__ void __launch_bounds__(512) dsh_hist_kernel(const int32_t* __restrict__ idx, int64_t S, int M, int64_t C,
                                                       int32_t* __restrict__ G, unsigned int* status) {
  extern __shared__ int32_t hist_s[];
  for (int v = threadIdx.x; v < M; v += blockDim.x) hist_s[v] = 0;
  __syncthreads();
  int64_t b, e;
  chunk_range(S, C, blockIdx.x, b, e);
  for (int64_t s = b + threadIdx.x; s < e; s += blockDim.x) {
    const int v = idx[s];
    if ((unsigned)v < (unsigned)M)
      atomicAdd(hist_s + v, 1);
    else
      atomicOr(status, MORE_DEVERR_BAD_INPUT);
  }
  __syncthreads();
  int32_t* row = G + (int64_t)blockIdx.x * M;
  for (int v = threadIdx.x; v < M; v += blockDim.x) row[v] = hist_s[v];
}

// 2. per column v: G[c][v] <- sum of G[c'][v] over c' < c; totals[v] <- the column's sum.
//    CTA = 32 experts (lane = expert), warp w = the band of chunks [w R, (w + 1) R).
__global__ void __launch_bounds__(256) dsh_colscan_kernel(int32_t* __restrict__ G, int64_t C, int M,
                                                          int32_t* __restrict__ totals) {
  __shared__ int32_t band[8][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int v = blockIdx.x * 32 + lane;
  const int64_t R = (C + 7) / 8, c0 = warp * R, c1 = c0 + R < C ? c0 + R : C;
  int32_t sum = 0;
  if (v < M)
    for (int64_t c = c0; c < c1; ++c) sum += G[c * M + v];
  band[warp][lane] = sum;
  __syncthreads();
  int32_t run = 0, total = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    run += w < warp ? band[w][lane] : 0;
    total += band[w][lane];
  }
  if (v < M) {
    for (int64_t c = c0; c < c1; ++c) {
      const int32_t x = G[c * M + v];
      G[c * M + v] = run;
      run += x;
    }
    if (warp == 0) totals[v] = total;
  }
}

// 4. CTA c walks its chunk 256 slots at a time: lane order within a warp (match-any), warp
//    order across the warps (their counter updates take turns, one barrier each).
__global__ void __launch_bounds__(256) dsh_scatter_kernel(const int32_t* __restrict__ idx, int64_t S, int M, int64_t C,
                                                          const int32_t* __restrict__ G,
                                                          const int32_t* __restrict__ offsets,
                                                          int32_t* __restrict__ sorted) {
  extern __shared__ int32_t ctr_s[];  // next output position of each expert's slots of this chunk
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t* row = G + (int64_t)blockIdx.x * M;
  for (int v = threadIdx.x; v < M; v += blockDim.x) ctr_s[v] = offsets[v] + row[v];
  __syncthreads();
  int64_t b, e;
  chunk_range(S, C, blockIdx.x, b, e);
  const unsigned int below = (1u << lane) - 1u;
  for (int64_t b0 = b; b0 < e; b0 += 256) {
    const int64_t s = b0 + threadIdx.x;
    const bool in = s < e;
    const int v = in ? idx[s] : -1;
    const bool ok = in && (unsigned)v < (unsigned)M;
    const unsigned int peers = __match_any_sync(0xffffffffu, ok ? v : -1);
    const bool leader = ok && (peers & below) == 0;
    int32_t base = 0;
    for (int w = 0; w < 8; ++w) {
      if (warp == w && leader) {
        base = ctr_s[v];
        ctr_s[v] = base + __popc(peers);
      }
      __syncthreads();
    }
    base = __shfl_sync(0xffffffffu, base, __ffs(peers) - 1);
    if (ok) sorted[base + __popc(peers & below)] = (int32_t)s;
  }
}

}  // namespace

// Covers both variants: for M <= kSharedMMax the shared variant's chunk count is at most chunk_count.
int64_t dispatch_scratch_bytes(int64_t S, int M) { return (chunk_count(S, M) * M + M) * 4 + 16; }

cudaError_t launch_dispatch(const int32_t* idx, int64_t S, int M, int32_t* offsets, int32_t* sorted,
                            void* scratch, unsigned int* status, cudaStream_t stream) {
  if (S == 0) return cudaMemsetAsync(offsets, 0, sizeof(int32_t) * ((size_t)M + 1), stream);
  const int64_t nchunks = chunk_count(S, M);
  const int64_t chunk = (S + nchunks - 1) / nchunks;
  int32_t* hist = static_cast<int32_t*>(scratch);
  int32_t* totals = hist + nchunks * M;
  cudaError_t e = cudaMemsetAsync(hist, 0, sizeof(int32_t) * (size_t)(nchunks * M), stream);
  if (e != cudaSuccess) return e;
  dispatch_hist_kernel<<<(unsigned)nchunks, 256, 0, stream>>>(idx, S, M, chunk, hist, status);
  dispatch_colscan_kernel<<<(unsigned)((M + 255) / 256), 256, 0, stream>>>(hist, nchunks, M, totals);
  dispatch_offsets_kernel<<<1, 1024, 0, stream>>>(totals, M, offsets);
  dispatch_scatter_kernel<<<(unsigned)((nchunks + 7) / 8), 256, 0, stream>>>(idx, S, M, chunk, nchunks, hist,
                                                                            offsets, sorted);
  return cudaGetLastError();
}

bool dispatch_shared_supports(int M) { return M <= kSharedMMax; }

cudaError_t launch_dispatch_shared(const int32_t* idx, int64_t S, int M, int32_t* offsets, int32_t* sorted,
                                   void* scratch, unsigned int* status, cudaStream_t stream) {
  if (S == 0) return cudaMemsetAsync(offsets, 0, sizeof(int32_t) * ((size_t)M + 1), stream);
  if (M > kSharedMMax) return cudaErrorInvalidValue;
  static std::atomic<int> configured[64] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  const int smem = (int)sizeof(int32_t) * kSharedMMax;
  if (dev < 0 || dev >= 64 || !configured[dev].load(std::memory_order_acquire)) {
    if ((err = cudaFuncSetAttribute(dsh_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
        cudaSuccess)
      return err;
    if ((err = cudaFuncSetAttribute(dsh_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
        cudaSuccess)
      return err;
    if (dev >= 0 && dev < 64) configured[dev].store(1, std::memory_order_release);
  }
  const int64_t C = shared_chunk_count(S);
  int32_t* G = static_cast<int32_t*>(scratch);  // C x M, every entry written by the histogram kernel
  int32_t* totals = G + C * M;
  const size_t hist_bytes = sizeof(int32_t) * (size_t)M;
  dsh_hist_kernel<<<(unsigned)C, 512, hist_bytes, stream>>>(idx, S, M, C, G, status);
  dsh_colscan_kernel<<<(unsigned)((M + 31) / 32), 256, 0, stream>>>(G, C, M, totals);
  dispatch_offsets_kernel<<<1, 1024, 0, stream>>>(totals, M, offsets);
  dsh_scatter_kernel<<<(unsigned)C, 256, hist_bytes, stream>>>(idx, S, M, C, G, offsets, sorted);
  return cudaGetLastError();
}

}  // namespace more

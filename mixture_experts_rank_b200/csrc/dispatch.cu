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
#include <algorithm>

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

}  // namespace

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

}  // namespace more

// Fused full-rank router: the standard MoE router softmax(TopK(x . W)), W of shape h x M,
// fused as "MoRE: Scaling mixture of experts with hardware-aware low-rank routing" App. H.3
// ("Fusing a standard MoE layer", Figs. 20-22) describes: the router weight is streamed past
// every 128-token tile, one 128-expert tile of W (all h rows) at a time, and the N x M scores
// never leave the chip.
//   warp 0      TMA producer: stages of X (128 tokens x 64 hidden, K-major) and W (64 hidden
//               x 128 experts, MN-major), both 128B-swizzled;
//   warp 1      tcgen05 MMAs (M = 128 tokens, N = 128 experts, K = 16), h / 16 of them per
//               score tile, into four 128-column TMEM buffers;
//   warps 4-11  one token and 64 of each tile's experts per thread: a running top-k in
//               registers that inserts only scores beating its current k-th entry, then the
//               two halves of each token are merged, the softmax is taken over the k, and the
//               outputs and counts are written.
// Every score is the fp32 sum of exact bf16 products; the selection is the exact top-k of
// those scores in routing order (larger first, lower expert first on equal scores).
#include <cudaTypedefs.h>

#include <atomic>

#include "mbar_wait.cuh"
#include "more_internal.cuh"
#include "sm100_ptx.cuh"
#include "warp_simt.cuh"

namespace more {
namespace full {

using namespace sm100;

constexpr int kBT = 128;        // tokens per tile
constexpr int kBE = 128;        // experts per score tile
constexpr int kBK = 64;         // hidden elements per stage
constexpr int kRoleWarps = 4;   // producer, MMA issuer, two idle (keep warp % 4 = TMEM lane group)
constexpr int kEpiWarps = 8;    // two per TMEM lane group, 64 columns each
constexpr int kThreads = (kRoleWarps + kEpiWarps) * 32;
constexpr uint32_t kTmemCols = 512;
constexpr int kNS = 4;                              // 128-column score buffers
constexpr uint32_t kXStage = kBT * kBK * 2;         // 16 KB
constexpr uint32_t kWBox = kBK * 64 * 2;            // 8 KB: 64 hidden rows x 64 experts
constexpr uint32_t kStage = kXStage + 2 * kWBox;    // 32 KB
constexpr int kMaxStages = 6;
constexpr uint32_t kSmemLimit = 227 * 1024;
constexpr uint32_t kIdesc = idesc_bf16_f32(128, 128, 0, 1);  // A = X (K-major), B = W (MN-major)

struct Params {
  RouteArgs a;  // R2 holds W (h x M); R1 and r are unused
  int num_tiles, kb_count, p_count, stages;
  uint32_t off_stage, off_merge, off_bar;
};

struct Bars {
  uint64_t* full;     // [kMaxStages] X + W stage loaded
  uint64_t* empty;    // [kMaxStages] stage read by the MMAs
  uint64_t* s_full;   // [kNS] score tile complete
  uint64_t* s_empty;  // [kNS] score tile read by the epilogue warps
  uint64_t* m_full;   // [2] second-half lists written
  uint64_t* m_empty;  // [2] second-half lists read
  uint64_t* drain;    // [1]
  uint32_t* tmem_slot;
  int* abort_flag;
};
constexpr uint32_t kBarSlots = 2 * kMaxStages + 2 * kNS + 4 + 1;
constexpr uint32_t kBarBytes = kBarSlots * 8 + 16;

__device__ __forceinline__ Bars bars_at(uint8_t* smem, const Params& p) {
  uint64_t* b = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  Bars r;
  r.full = b;
  r.empty = b + kMaxStages;
  r.s_full = r.empty + kMaxStages;
  r.s_empty = r.s_full + kNS;
  r.m_full = r.s_empty + kNS;
  r.m_empty = r.m_full + 2;
  r.drain = r.m_empty + 2;
  r.tmem_slot = reinterpret_cast<uint32_t*>(r.drain + 1);
  r.abort_flag = reinterpret_cast<int*>(r.tmem_slot + 1);
  return r;
}

__device__ __forceinline__ int local_tiles(const Params& p) {
  return (int)blockIdx.x < p.num_tiles ? (p.num_tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
}

// ---- role: TMA producer --------------------------------------------------------------------
__device__ void producer(const Params& p, const Bars& b, uint8_t* smem, const CUtensorMap* tmX,
                         const CUtensorMap* tmW) {
  RingPos s;
  const int T = local_tiles(p);
  for (int j = 0; j < T; ++j) {
    const int tile = (int)blockIdx.x + j * (int)gridDim.x;
    for (int pt = 0; pt < p.p_count; ++pt) {
      for (int kb = 0; kb < p.kb_count; ++kb) {
        if (!bounded_wait(&b.empty[s.i], s.phase ^ 1u, b.abort_flag, p.a.status)) return;
        uint8_t* st = smem + p.off_stage + s.i * kStage;
        mbar_arrive_expect_tx(&b.full[s.i], kStage);
        tma_load_2d(st, tmX, &b.full[s.i], kb * kBK, tile * kBT);
        tma_load_2d(st + kXStage, tmW, &b.full[s.i], pt * kBE, kb * kBK);
        tma_load_2d(st + kXStage + kWBox, tmW, &b.full[s.i], pt * kBE + 64, kb * kBK);
        s.next(p.stages);
      }
    }
  }
}

// ---- role: MMA issuer -------------------------------------------------------------------------
__device__ void mma_scores(const Params& p, const Bars& b, uint8_t* smem, uint32_t tmem_base) {
  RingPos s, d;
  const int T = local_tiles(p);
  const uint32_t st0 = smem_u32(smem + p.off_stage);
  for (int j = 0; j < T; ++j) {
    for (int pt = 0; pt < p.p_count; ++pt) {
      if (!bounded_wait(&b.s_empty[d.i], d.phase ^ 1u, b.abort_flag, p.a.status)) goto done;
      tc_fence_after();
      for (int kb = 0; kb < p.kb_count; ++kb) {
        if (!bounded_wait(&b.full[s.i], s.phase, b.abort_flag, p.a.status)) goto done;
        tc_fence_after();
        const uint32_t st = st0 + s.i * kStage;
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint64_t ad = smem_desc(st + kk * 32, 16, 1024, kSwizzle128B);
          const uint64_t bd = smem_desc(st + kXStage + kk * 2048, kWBox, 1024, kSwizzle128B);
          mma_bf16(tmem_base + d.i * 128, ad, bd, kIdesc, (kb | kk) != 0);
        }
        mma_commit(&b.empty[s.i]);
        s.next(p.stages);
      }
      mma_commit(&b.s_full[d.i]);
      d.next(kNS);
    }
  }
done:
  mma_commit(&b.drain[0]);
  bounded_wait(&b.drain[0], 0, b.abort_flag, p.a.status);
}

// ---- epilogue warps: running top-k, merge, softmax, outputs ------------------------------------
template <int KCAP>
__device__ void epilogue(const Params& p, const Bars& b, uint8_t* smem, uint32_t tmem_base) {
  const RouteArgs& a = p.a;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ew = warp - kRoleWarps;  // 0..7
  const int sp = warp & 3;           // TMEM lane group: tokens 32 sp .. 32 sp + 31
  const int hh = ew >> 2;            // experts hh * 64 .. hh * 64 + 63 of each tile
  const int t = sp * 32 + lane;
  const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
  uint2* merge = reinterpret_cast<uint2*>(smem + p.off_merge);  // [2][kBT][KCAP] (value bits, expert)
  RingPos d;
  const int T = local_tiles(p);
  for (int j = 0; j < T; ++j) {
    const int64_t n0 = ((int64_t)blockIdx.x + (int64_t)j * gridDim.x) * kBT;
    TopList<KCAP> list;
    list.init();
    for (int pt = 0; pt < p.p_count; ++pt) {
      if (!bounded_wait(&b.s_full[d.i], d.phase, b.abort_flag, a.status)) return;
      tc_fence_after();
      uint32_t v[64];
      const uint32_t col = tmem_base + lane_base + d.i * 128 + hh * 64;
      tmem_ld_x32(col, v);
      tmem_ld_x32(col + 32, v + 32);
      tmem_wait_ld();
      reg_fence<64>(v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&b.s_empty[d.i]);
      d.next(kNS);
      // experts arrive in increasing order, so a strict comparison keeps the lower one on ties
      const int e0 = pt * kBE + hh * 64;
      if (e0 + 64 <= a.M) {
#pragma unroll
        for (int q = 0; q < 64; ++q) list.insert(__uint_as_float(v[q]), e0 + q);
      } else {
#pragma unroll
        for (int q = 0; q < 64; ++q)
          if (e0 + q < a.M) list.insert(__uint_as_float(v[q]), e0 + q);
      }
    }
    // token t's two halves: the hh = 1 thread hands its list to the hh = 0 thread
    const int mb = j & 1, mu = j >> 1;
    uint2* mrow = merge + ((size_t)mb * kBT + t) * KCAP;
    if (hh == 1) {
      if (mu > 0 && !bounded_wait(&b.m_empty[mb], (mu - 1) & 1, b.abort_flag, a.status)) return;
#pragma unroll
      for (int q = 0; q < KCAP; ++q) mrow[q] = make_uint2(__float_as_uint(list.v[q]), (uint32_t)list.i[q]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&b.m_full[mb]);
      continue;
    }
    if (!bounded_wait(&b.m_full[mb], mu & 1, b.abort_flag, a.status)) return;
#pragma unroll
    for (int q = 0; q < KCAP; ++q) {
      const uint2 c = mrow[q];
      if (q < a.k) list.insert_any(__uint_as_float(c.x), (int)c.y);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&b.m_empty[mb]);
    if (n0 + t >= a.N) continue;
    const float top = list.v[0];
    float ex[KCAP], sum = 0.f;
#pragma unroll
    for (int q = 0; q < KCAP; ++q) {
      ex[q] = q < a.k ? expf(list.v[q] - top) : 0.f;
      sum += ex[q];
    }
    const float inv = 1.f / sum;
    const size_t o = (size_t)(n0 + t) * a.k;
#pragma unroll
    for (int q = 0; q < KCAP; ++q) {
      if (q >= a.k) break;
      a.out_idx[o + q] = list.i[q];
      a.out_gate[o + q] = ex[q] * inv;
      if (a.out_logits) a.out_logits[o + q] = list.v[q];
      atomicAdd(a.out_count + list.i[q], 1);
    }
  }
}

template <int KCAP>
__global__ void __launch_bounds__(kThreads, 1)
    fullrank_route_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                          const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Bars b = bars_at(smem, p);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < p.stages; ++i) {
      mbar_init(&b.full[i], 1);
      mbar_init(&b.empty[i], 1);
    }
    for (int i = 0; i < kNS; ++i) {
      mbar_init(&b.s_full[i], 1);
      mbar_init(&b.s_empty[i], kEpiWarps);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&b.m_full[i], 4);   // the four hh = 1 warps
      mbar_init(&b.m_empty[i], 4);  // the four hh = 0 warps
    }
    mbar_init(&b.drain[0], 1);
    *b.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmX);
    prefetch_tensormap(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(b.tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *b.tmem_slot;

  if (warp == 0) {
    if (lane == 0) producer(p, b, smem, &tmX, &tmW);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) mma_scores(p, b, smem, tmem_base);
    __syncwarp();
  } else if (warp >= kRoleWarps) {
    epilogue<KCAP>(p, b, smem, tmem_base);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ---- host side ---------------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::atomic<PFN_cuTensorMapEncodeTiled_v12000> fn{nullptr};
  PFN_cuTensorMapEncodeTiled_v12000 f = fn.load(std::memory_order_acquire);
  if (!f) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      f = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
      fn.store(f, std::memory_order_release);
    }
  }
  return f;
}

bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
              uint32_t box_outer) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

uint32_t align_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

// Shared memory: the stage ring first (as deep as fits, up to kMaxStages), then the merge
// lists and the barriers.  Returns the total bytes, or 0 when fewer than 2 stages fit.
template <int KCAP>
uint32_t plan(Params& p) {
  for (int st = kMaxStages; st >= 2; --st) {
    uint32_t off = 0;
    p.off_stage = off;
    off += st * kStage;
    p.off_merge = off = align_up(off, 16);
    off += 2 * kBT * KCAP * 8;
    p.off_bar = off = align_up(off, 8);
    off += kBarBytes;
    const uint32_t total = off + 1024;  // alignment slack of the dynamic base
    if (total <= kSmemLimit) {
      p.stages = st;
      return total;
    }
  }
  return 0;
}

template <int KCAP>
cudaError_t configure_once(int dev) {
  static std::atomic<int> done[64] = {};
  if (dev >= 0 && dev < 64 && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(fullrank_route_kernel<KCAP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemLimit);
  if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev].store(1, std::memory_order_release);
  return e;
}

template <int KCAP>
cudaError_t launch(const RouteArgs& a) {
  Params p;
  p.a = a;
  p.num_tiles = (int)((a.N + kBT - 1) / kBT);
  p.kb_count = (a.h + kBK - 1) / kBK;
  p.p_count = (a.M + kBE - 1) / kBE;
  const uint32_t smem = plan<KCAP>(p);
  if (!smem) return cudaErrorInvalidConfiguration;
  CUtensorMap tmX, tmW;
  if (!make_map(&tmX, a.X, (uint64_t)a.h, (uint64_t)a.N, kBK, kBT) ||
      !make_map(&tmW, a.R2, (uint64_t)a.M, (uint64_t)a.h, 64, kBK))
    return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = configure_once<KCAP>(dev);
  if (e != cudaSuccess) return e;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = p.num_tiles < sms ? p.num_tiles : sms;
  fullrank_route_kernel<KCAP><<<grid, kThreads, smem, a.stream>>>(tmX, tmW, p);
  return cudaGetLastError();
}

}  // namespace full

cudaError_t launch_fullrank(const RouteArgs& a) {
  if (a.N < 1 || a.N > 0x7fffffffLL - full::kBT) return cudaErrorInvalidValue;
  if (a.k <= 4) return full::launch<4>(a);
  if (a.k <= 8) return full::launch<8>(a);
  return full::launch<16>(a);
}

}  // namespace more

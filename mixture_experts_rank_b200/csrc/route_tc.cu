// Fused MoRE routing kernel for B200 (sm_100a): TMA-staged X, tcgen05 MMAs into
// TMEM, an exact two-pass top-k on the CUDA cores, softmax gates and counts.
//
// What it computes is the router of "MoRE: Scaling mixture of experts with
// hardware-aware low-rank routing": §2 "MoRE layer" (softmax over TopK of the
// rank-r logits), App. F eq. (5) and Algorithm 1 (z = X R1 accumulated in fp32,
// one B_N x B_M logit tile at a time, out-of-range experts at -infinity, only
// the (N, k) selection written), Fig. 12 (gates) and eq. (9) (counts).  The N x M
// logits exist only in TMEM.
//
// How (one persistent CTA per SM, 128-token tiles, 20 warps):
//   warp 0  TMA producer of X (128 x BK bf16, swizzled) and R1 (BK x r) stages.
//   warp 1  MMA issuer for Z = X R1: M=128 tokens, N=r, K=16 steps over h, into a
//           double-buffered TMEM accumulator (the next tile streams while the
//           current one is routed, so HBM never waits on the top-k).
//   warp 2  MMA issuer for the logit tiles: pass 1 D[tok, exp] = z_hi R2 (K = r),
//           pass 2 D^T[exp, tok] = R2^T [z_hi | z_lo]^T (K = 2r, exact to ~16 bits of z).
//   warp 3  TMA producer of R2 tiles (r x 128 experts); R2 stays resident in
//           shared memory when it fits, else it is streamed from L2.
//   warps 4-19  four consumer warpgroups (TMEM lanes = tokens in pass 1, experts
//           in pass 2; warpgroup g takes lane group warp % 4):
//     epilogue  Z from TMEM -> (z_hi, z_lo) bf16 pair -> shared memory (K-major),
//               plus |z_hi|, |z_lo| per token and the largest column norm of R2.
//     pass 1    every 32-expert chunk of a token is reduced to the maximum of its
//               z_hi logits, packed into a 32-bit key (order-preserving value bits
//               above the chunk id); a branch-free sorted list keeps the best
//               k + 6 keys per warpgroup.
//     select    the four lists are merged.  z_hi logits differ from the exact ones
//               by at most eps (|z_lo| times the largest R2 column norm, plus fp32
//               rounding), so the exact k-th logit is at least tlow - eps (tlow: the
//               k-th chunk maximum) and only chunks whose maximum reaches
//               tlow - 2 eps can hold a top-k expert.  (token, chunk) pairs are
//               bucketed by chunk with a counting sort.
//     pass 2    a tile is worked by two warpgroups (0-1 for even tiles, 2-3 for odd):
//               the two warps of a lane group split the pairs of their chunk, read
//               each pair's token column and ballot the experts whose exact logit
//               reaches tlow - eps (the candidates).
//     finalize  four threads per token rank its few candidates in routing order
//               (larger logit, then lower expert) into a shared-memory staging of the
//               outputs, which the tile writes with coalesced stores; softmax, counts.
//               A list too short to certify the cut, or more candidates than the
//               slots hold, sends the token to an exact recomputation on CUDA
//               cores shared by all sixteen consumer warps.
// Every consumer warp waits for every logit tile and arrives once on its empty
// barrier, so no warp can fall two phases behind a buffer (a parity wait cannot tell
// those apart).  Every barrier wait, the consumers' own barrier included, is bounded
// (a few seconds); on expiry the kernel records MORE_DEVERR_WAIT_TIMEOUT in the
// library's device error word and every role unwinds.
#include <cudaTypedefs.h>

#include "more_internal.cuh"
#include "sm100_ptx.cuh"
#include "warp_simt.cuh"

namespace more {
namespace tc {

using namespace sm100;

constexpr int kBT = 128;        // tokens per tile (MMA M of Z and pass 1, N of pass 2)
constexpr int kBE = 128;        // experts per logit tile
constexpr int kThreads = 640;   // 4 role warps + 16 consumer warps
constexpr int kConsumerThreads = 512;
constexpr int kConsumerWarps = 16;
constexpr int kPairBatch = 4;   // TMEM column loads in flight per warp in pass 2
constexpr int kPoolSlots = 4;   // per-token overflow slots for chunks with more than S candidates
constexpr int kFbBatch = 8;     // fallback tokens ranked per round of the cooperative fallback
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kTimeoutNs = 4000000000ull;
constexpr uint32_t kRealKey = 0x00800000u;  // ordered value of -FLT_MAX: keys below are not real chunks

// ---- parameters -----------------------------------------------------------------------

struct Params {
  RouteArgs a;
  int num_tiles;     // token tiles
  int kb_count;      // hidden blocks of kBK
  int p_count;       // expert tiles of kBE
  int nchunks;       // 32-expert chunks
  uint32_t low_mask; // chunk-id bits of a key
  int x_stages;
  int r2_stages;
  int r2_resident;   // every expert tile stays in shared memory
  uint32_t off_x, off_r1, off_r2, off_zs, off_lists, off_cand, off_thr, off_flag, off_nq, off_fb, off_pc, off_pairs,
      off_ccount, off_cbase, off_scan, off_pool, off_poolcnt, off_znorm, off_cnorm, off_bar;
};

template <int R, int KCAP>
struct Cfg {
  static constexpr int KL = KCAP + 6;                  // chunk keys kept per token
  static constexpr int KLP = (KL + 15) & ~15;          // row stride of the candidate slots and counts
  static constexpr int S = 1;                          // candidate slots per (token, needed chunk)
  static constexpr int RK = 2 * R;                     // z_hi | z_lo columns of the z buffer
  static constexpr int BK = R >= 128 ? 32 : 64;        // hidden elements per X stage
  static constexpr uint32_t X_STAGE = kBT * BK * 2;    // 16 KB (8 KB at BK = 32)
  static constexpr uint32_t X_LAYOUT = BK == 64 ? kSwizzle128B : kSwizzle64B;
  static constexpr uint32_t X_SBO = 8 * BK * 2;        // bytes per 8-row swizzle atom
  static constexpr int R1_BOX = R < 64 ? R : 64;       // inner box of R1 (elements)
  static constexpr int R1_BOXES = R / R1_BOX;
  static constexpr uint32_t R1_BOX_BYTES = BK * R1_BOX * 2;
  static constexpr uint32_t R1_STAGE = R1_BOX_BYTES * R1_BOXES;
  static constexpr uint32_t R1_ROW = R1_BOX * 2;       // bytes per R1 row inside a box
  static constexpr uint32_t R1_LAYOUT = R1_ROW == 32 ? kSwizzle32B : (R1_ROW == 64 ? kSwizzle64B : kSwizzle128B);
  static constexpr uint32_t R2_BOX_BYTES = 64 * R * 2; // 64 experts x R rows
  static constexpr uint32_t R2_STAGE = 2 * R2_BOX_BYTES;
  static constexpr uint32_t ZS_BYTES = kBT * RK * 2;   // z pair of 128 tokens, K-major core matrices
  static constexpr uint32_t ZS_SBO = (RK / 8) * 128;   // byte stride of 8-token groups
  static constexpr int ZCOLS = R < 32 ? 32 : R;        // TMEM columns per Z accumulator
  static constexpr int ND = (512 - 2 * ZCOLS) / 128 < 3 ? (512 - 2 * ZCOLS) / 128 : 3;  // logit tile buffers
  static constexpr int ZCOL0 = ND * 128;               // first TMEM column of the Z accumulators
  static constexpr uint32_t IDESC_Z = idesc_bf16_f32(128, R, 0, 1);    // A = X (K-major), B = R1 (MN-major)
  static constexpr uint32_t IDESC_P1 = idesc_bf16_f32(128, 128, 0, 1); // A = z pair, B = R2 tile
  static constexpr uint32_t IDESC_P2 = idesc_bf16_f32(128, 128, 1, 0); // A = R2 tile^T, B = z pair^T
};

// Barrier block layout (uint64_t slots).
struct Bars {
  uint64_t* x_full;
  uint64_t* x_empty;
  uint64_t* r2_full;
  uint64_t* r2_empty;
  uint64_t* zacc_full;   // [2]
  uint64_t* zacc_empty;  // [2]
  uint64_t* zsm_full;
  uint64_t* zsm_empty;
  uint64_t* d_full;      // [3]
  uint64_t* d_empty;     // [3]
  uint64_t* drain;       // [2]
  uint64_t* cbar;        // consumer-warp barrier (16 arrivals per phase)
  uint32_t* tmem_slot;
  int* abort_flag;
};

__device__ __forceinline__ Bars bars_at(uint8_t* smem, const Params& p) {
  uint64_t* b = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  Bars r;
  r.x_full = b;
  r.x_empty = b + 8;
  r.r2_full = b + 16;
  r.r2_empty = r.r2_full + 64;
  r.zacc_full = r.r2_empty + 64;
  r.zacc_empty = r.zacc_full + 2;
  r.zsm_full = r.zacc_empty + 2;
  r.zsm_empty = r.zsm_full + 1;
  r.d_full = r.zsm_empty + 1;
  r.d_empty = r.d_full + 3;
  r.drain = r.d_empty + 3;
  r.cbar = r.drain + 2;
  r.tmem_slot = reinterpret_cast<uint32_t*>(r.cbar + 1);
  r.abort_flag = reinterpret_cast<int*>(r.tmem_slot + 1);
  return r;
}
constexpr uint32_t kBarBytes = (16 + 128 + 15) * 8 + 16;

// Slow path of the bounded mbarrier wait: false once the limit passes or another
// thread gave up.
__device__ __noinline__ bool wait_bar_slow(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                           unsigned int* status) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t spin = 1;; ++spin) {
    if (mbar_try_wait_sleep(bar, parity, 200000u)) return true;
    if ((spin & 3u) == 0) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > kTimeoutNs) {
        atomicOr(status, MORE_DEVERR_WAIT_TIMEOUT);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

// The first attempt suspends in hardware until the phase completes (or ~65 us pass),
// so a normal wait is one instruction and the bounded loop is a rare call.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                         unsigned int* status) {
  if (mbar_try_wait_sleep(bar, parity, 65536u)) return true;
  return wait_bar_slow(bar, parity, abort_flag, status);
}


// Barrier of the 16 consumer warps on an mbarrier, so that it is bounded like every
// other wait: if any role gives up (and raises the abort flag), a warp waiting here
// leaves too instead of waiting for a warp that has already returned.  `phase` is
// the calling thread's parity of the barrier, flipped at every use.
__device__ __forceinline__ bool consumer_sync(const Bars& b, uint32_t& phase, unsigned int* status) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(b.cbar);
  const bool ok = wait_bar(b.cbar, phase, b.abort_flag, status);
  phase ^= 1u;
  return ok;
}

// Order-preserving map of fp32 onto uint32 and its inverse.
__device__ __forceinline__ uint32_t ord_key(float f) {
  uint32_t b = __float_as_uint(f);
  return b ^ ((uint32_t)((int32_t)b >> 31) | 0x80000000u);
}
__device__ __forceinline__ float ord_inv(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float m;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(a), "f"(b), "f"(c));
  return m;
}

// Maximum of 32 fp32 values held as raw bits.
__device__ __forceinline__ float max32(const uint32_t* v) {
  float a[11];
#pragma unroll
  for (int i = 0; i < 10; ++i)
    a[i] = max3f(__uint_as_float(v[3 * i]), __uint_as_float(v[3 * i + 1]), __uint_as_float(v[3 * i + 2]));
  a[10] = fmaxf(__uint_as_float(v[30]), __uint_as_float(v[31]));
  float b0 = max3f(a[0], a[1], a[2]), b1 = max3f(a[3], a[4], a[5]), b2 = max3f(a[6], a[7], a[8]);
  float b3 = fmaxf(a[9], a[10]);
  return max3f(b0, b1, fmaxf(b2, b3));
}

// Branch-free insertion of key x into the descending list kl[0..L).
template <int L>
__device__ __forceinline__ void key_insert(uint32_t* kl, uint32_t x) {
#pragma unroll
  for (int i = L - 1; i > 0; --i) kl[i] = min(kl[i - 1], max(kl[i], x));
  kl[0] = max(kl[0], x);
}

// Byte offset of the 16-byte core-matrix row (token t, K chunk c) in the z pair buffer.
template <int R, int KCAP>
__device__ __forceinline__ uint32_t zs_offset(int t, int c) {
  return (uint32_t)(((t >> 3) * (Cfg<R, KCAP>::RK / 8) + c) * 128 + (t & 7) * 16);
}

// z_t[i] (fp32 value of the pair) read back from the z pair buffer.
template <int R, int KCAP>
__device__ __forceinline__ float zs_value(const uint8_t* zs, int t, int i) {
  const __nv_bfloat16* hi = reinterpret_cast<const __nv_bfloat16*>(zs + zs_offset<R, KCAP>(t, i >> 3)) + (i & 7);
  const __nv_bfloat16* lo =
      reinterpret_cast<const __nv_bfloat16*>(zs + zs_offset<R, KCAP>(t, (R + i) >> 3)) + (i & 7);
  return __bfloat162float(*hi) + __bfloat162float(*lo);
}

// ---- role: TMA producer of X and R1 -----------------------------------------------

template <int R, int KCAP>
__device__ void producer_x(const Params& p, const Bars& b, uint8_t* smem, const CUtensorMap* tmX,
                           const CUtensorMap* tmR1) {
  using C = Cfg<R, KCAP>;
  int s = 0;
  uint32_t ph = 0;
  for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
    for (int kb = 0; kb < p.kb_count; ++kb) {
      if (!wait_bar(&b.x_empty[s], ph ^ 1u, b.abort_flag, p.a.status)) return;
      mbar_arrive_expect_tx(&b.x_full[s], C::X_STAGE + C::R1_STAGE);
      tma_load_2d(smem + p.off_x + s * C::X_STAGE, tmX, &b.x_full[s], kb * C::BK, tile * kBT);
#pragma unroll
      for (int q = 0; q < C::R1_BOXES; ++q)
        tma_load_2d(smem + p.off_r1 + s * C::R1_STAGE + q * C::R1_BOX_BYTES, tmR1, &b.x_full[s], q * 64,
                    kb * C::BK);
      if (++s == p.x_stages) {
        s = 0;
        ph ^= 1u;
      }
    }
  }
}

// ---- role: TMA producer of R2 tiles ----------------------------------------------------

template <int R, int KCAP>
__device__ void producer_r2(const Params& p, const Bars& b, uint8_t* smem, const CUtensorMap* tmR2) {
  using C = Cfg<R, KCAP>;
  if (p.r2_resident) {
    for (int t = 0; t < p.p_count; ++t) {
      uint8_t* dst = smem + p.off_r2 + t * C::R2_STAGE;
      mbar_arrive_expect_tx(&b.r2_full[t], C::R2_STAGE);
      tma_load_2d(dst, tmR2, &b.r2_full[t], t * kBE, 0);
      tma_load_2d(dst + C::R2_BOX_BYTES, tmR2, &b.r2_full[t], t * kBE + 64, 0);
    }
    return;
  }
  int s = 0;
  uint32_t ph = 0;
  for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
    for (int pass = 0; pass < 2; ++pass) {
      for (int t = 0; t < p.p_count; ++t) {
        if (!wait_bar(&b.r2_empty[s], ph ^ 1u, b.abort_flag, p.a.status)) return;
        uint8_t* dst = smem + p.off_r2 + s * C::R2_STAGE;
        mbar_arrive_expect_tx(&b.r2_full[s], C::R2_STAGE);
        tma_load_2d(dst, tmR2, &b.r2_full[s], t * kBE, 0);
        tma_load_2d(dst + C::R2_BOX_BYTES, tmR2, &b.r2_full[s], t * kBE + 64, 0);
        if (++s == p.r2_stages) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
  }
}

// ---- role: MMA issuer of Z = X R1 ------------------------------------------------------

template <int R, int KCAP>
__device__ void mma_z(const Params& p, const Bars& b, uint8_t* smem, uint32_t tmem_base) {
  using C = Cfg<R, KCAP>;
  int s = 0;
  uint32_t ph = 0;
  int lt = 0;
  const uint32_t x0 = smem_u32(smem + p.off_x), r10 = smem_u32(smem + p.off_r1);
  for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++lt) {
    const int buf = lt & 1;
    if (!wait_bar(&b.zacc_empty[buf], ((lt >> 1) & 1) ^ 1u, b.abort_flag, p.a.status)) break;
    tc_fence_after();
    const uint32_t d = tmem_base + C::ZCOL0 + buf * C::ZCOLS;
    for (int kb = 0; kb < p.kb_count; ++kb) {
      if (!wait_bar(&b.x_full[s], ph, b.abort_flag, p.a.status)) goto done;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < C::BK / 16; ++kk) {
        uint64_t ad = smem_desc(x0 + s * C::X_STAGE + kk * 32, 16, C::X_SBO, C::X_LAYOUT);
        uint64_t bd = smem_desc(r10 + s * C::R1_STAGE + kk * 16 * C::R1_ROW, C::R1_BOX_BYTES, 8 * C::R1_ROW,
                                C::R1_LAYOUT);
        mma_bf16(d, ad, bd, C::IDESC_Z, (kb | kk) != 0);
      }
      mma_commit(&b.x_empty[s]);
      if (++s == p.x_stages) {
        s = 0;
        ph ^= 1u;
      }
    }
    mma_commit(&b.zacc_full[buf]);
  }
done:
  mma_commit(&b.drain[0]);
  wait_bar(&b.drain[0], 0, b.abort_flag, p.a.status);
}

// ---- role: MMA issuer of the logit tiles -------------------------------------------------

template <int R, int KCAP>
__device__ void mma_scores(const Params& p, const Bars& b, uint8_t* smem, uint32_t tmem_base) {
  using C = Cfg<R, KCAP>;
  int rs = 0;
  uint32_t rph = 0;
  int ds = 0;
  uint32_t dph = 0;
  int lt = 0;
  const uint32_t zs = smem_u32(smem + p.off_zs), r20 = smem_u32(smem + p.off_r2);
  for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++lt) {
    if (!wait_bar(b.zsm_full, lt & 1, b.abort_flag, p.a.status)) goto done;
    for (int pass = 0; pass < 2; ++pass) {
      for (int t = 0; t < p.p_count; ++t) {
        int st;
        if (p.r2_resident) {
          st = t;
          if (lt == 0 && pass == 0 && !wait_bar(&b.r2_full[t], 0, b.abort_flag, p.a.status)) goto done;
        } else {
          st = rs;
          if (!wait_bar(&b.r2_full[rs], rph, b.abort_flag, p.a.status)) goto done;
        }
        if (!wait_bar(&b.d_empty[ds], dph ^ 1u, b.abort_flag, p.a.status)) goto done;
        tc_fence_after();
        const uint32_t d = tmem_base + ds * 128;
        const uint32_t r2 = r20 + st * C::R2_STAGE;
        // pass 1 reads z_hi only (K = r); pass 2 reads z_hi | z_lo (K = 2r) for exact logits
        const int ksteps = pass == 0 ? R / 16 : C::RK / 16;
#pragma unroll
        for (int kk = 0; kk < ksteps; ++kk) {
          uint64_t zd = smem_desc(zs + kk * 256, 128, C::ZS_SBO, kSwizzleNone);
          uint64_t rd = smem_desc(r2 + (kk % (R / 16)) * 2048, C::R2_BOX_BYTES, 1024, kSwizzle128B);
          if (pass == 0)
            mma_bf16(d, zd, rd, C::IDESC_P1, kk != 0);
          else
            mma_bf16(d, rd, zd, C::IDESC_P2, kk != 0);
        }
        mma_commit(&b.d_full[ds]);
        if (!p.r2_resident) {
          mma_commit(&b.r2_empty[rs]);
          if (++rs == p.r2_stages) {
            rs = 0;
            rph ^= 1u;
          }
        }
        if (++ds == C::ND) {
          ds = 0;
          dph ^= 1u;
        }
      }
    }
    mma_commit(b.zsm_empty);
  }
done:
  mma_commit(&b.drain[1]);
  wait_bar(&b.drain[1], 0, b.abort_flag, p.a.status);
}

// ---- consumers ----------------------------------------------------------------------------

// Exact recomputation on CUDA cores of the logits of one token (ties at the threshold,
// candidate overflow), for the 256-expert block eb .. eb + 255: lane l takes experts
// eb + 8 l .. eb + 8 l + 7 (one 16-byte load per R2 row) and inserts them into its list
// in increasing index order.  zr holds z_i (z_hi + z_lo) in lane i mod 32 of entry i / 32.
template <int R, int KCAP>
__device__ __forceinline__ void fallback_block(const RouteArgs& a, const float (&zr)[(R + 31) / 32], int eb,
                                               int lane, TopList<KCAP>& list) {
  constexpr int L = R < 32 ? R : 32;
  const int e0 = eb + 8 * lane;
  const bool ok = e0 < a.M;  // M is a multiple of 8, so the lane's 8 experts are all in range
  const uint4* src = reinterpret_cast<const uint4*>(a.R2) + (ok ? (e0 >> 3) : 0);
  const size_t rowv = (size_t)(a.M >> 3);
  float acc[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) acc[q] = 0.f;
#pragma unroll
  for (int j = 0; j < (R + 31) / 32; ++j) {
#pragma unroll 4
    for (int l = 0; l < L; ++l) {
      const float zi = __shfl_sync(0xffffffffu, zr[j], l);
      const uint4 w = ok ? __ldg(src + (size_t)(32 * j + l) * rowv) : make_uint4(0u, 0u, 0u, 0u);
      const __nv_bfloat162* wp = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = __bfloat1622float2(wp[q]);
        acc[2 * q] = fmaf(zi, f.x, acc[2 * q]);
        acc[2 * q + 1] = fmaf(zi, f.y, acc[2 * q + 1]);
      }
    }
  }
  if (ok) {
#pragma unroll
    for (int q = 0; q < 8; ++q) list.insert(acc[q], e0 + q);
  }
}

// The cooperative fallback's first step: this warp's partial top-k (over the 256-expert
// blocks cw, cw + 16, ...) of each of the nb tokens in tok, written to part.
template <int R, int KCAP>
__device__ __forceinline__ void fallback_rank(const RouteArgs& a, const uint8_t* zs, const uint8_t* tok, int nb,
                                           uint2* part, int cw, int lane) {
  for (int j = 0; j < nb; ++j) {
    const int tf = tok[j];
    float zr[(R + 31) / 32];
#pragma unroll
    for (int q = 0; q < (R + 31) / 32; ++q)
      zr[q] = (32 * q + lane < R) ? zs_value<R, KCAP>(zs, tf, 32 * q + lane) : 0.f;
    TopList<KCAP> list;
    list.init();
    for (int eb = 256 * cw; eb < a.M; eb += 256 * kConsumerWarps) fallback_block<R, KCAP>(a, zr, eb, lane, list);
    float v;
    int e;
    warp_merge_topk<KCAP>(list, a.k, lane, v, e);
    if (lane < KCAP) part[(j * kConsumerWarps + cw) * KCAP + lane] = make_uint2(__float_as_uint(v), (uint32_t)e);
  }
}

// The second step: merge the sixteen partial lists of one token (part: warp-major, KCAP
// entries each, the first k valid) and write the token's outputs.
template <int KCAP>
__device__ __forceinline__ void fallback_merge(const RouteArgs& a, const uint2* part, int64_t n, int lane) {
  TopList<KCAP> list;
  list.init();
  for (int q = lane; q < kConsumerWarps * KCAP; q += 32) {
    const uint2 c = part[q];
    if ((q % KCAP) < a.k) list.insert_any(__uint_as_float(c.x), (int)c.y);
  }
  float v;
  int e;
  warp_merge_topk<KCAP>(list, a.k, lane, v, e);
  warp_write_selection(a, n, lane, v, e);
}

// Byte offset of R2 element (row i, expert e_local of a 128-expert stage) in the
// MN-major 128B-swizzled stage written by TMA (two boxes of 64 experts x R rows).
template <int R>
__device__ __forceinline__ uint32_t r2_offset(int i, int e_local) {
  const int box = e_local >> 6, col = e_local & 63;
  return (uint32_t)(box * (64 * R * 2) + i * 128 + ((((col >> 3) ^ (i & 7))) << 4) + (col & 7) * 2);
}

template <int R, int KCAP>
__device__ void consumers(const Params& p, const Bars& b, uint8_t* smem, uint32_t tmem_base) {
  using C = Cfg<R, KCAP>;
  constexpr int KL = C::KL;
  const RouteArgs& a = p.a;
  uint32_t cph = 0;  // parity of the consumer barrier
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sp = warp & 3;              // TMEM subpartition: lanes 32 sp .. 32 sp + 31
  const int g = (warp - 4) >> 2;        // consumer warpgroup 0..3
  const int cw = warp - 4;              // consumer warp 0..15
  const int ctid = threadIdx.x - 128;   // 0..511
  const int t = sp * 32 + lane;         // token of this thread in pass 1 and finalize
  const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
  uint8_t* zs = smem + p.off_zs;
  const uint8_t* r2s = smem + p.off_r2;
  uint32_t* lists = reinterpret_cast<uint32_t*>(smem + p.off_lists);
  uint32_t* stage = lists + 2 * KL * kBT;  // (chunk, rank) of each needed pair, after the two list slots
  uint2* cand = reinterpret_cast<uint2*>(smem + p.off_cand);
  float* thr = reinterpret_cast<float*>(smem + p.off_thr);
  int* flag = reinterpret_cast<int*>(smem + p.off_flag);
  uint8_t* nq = smem + p.off_nq;
  int* fbcount = reinterpret_cast<int*>(smem + p.off_fb);
  uint8_t* fblist = smem + p.off_fb + 4;
  uint8_t* fbmark = smem + p.off_fb + 4 + kBT;  // 1: the token's outputs come from the fallback
  uint2* part = reinterpret_cast<uint2*>(smem + p.off_lists);  // fallback partial lists (finalize only)
  uint8_t* pc = smem + p.off_pc;
  uint2* pairs = reinterpret_cast<uint2*>(smem + p.off_pairs);
  int* ccount = reinterpret_cast<int*>(smem + p.off_ccount);
  int* cbase = reinterpret_cast<int*>(smem + p.off_cbase);
  int* scan = reinterpret_cast<int*>(smem + p.off_scan);
  uint2* pool = reinterpret_cast<uint2*>(smem + p.off_pool);
  int* poolcnt = reinterpret_cast<int*>(smem + p.off_poolcnt);
  float* znorm = reinterpret_cast<float*>(smem + p.off_znorm);  // [hi g0 | hi g1 | lo g0 | lo g1][token]
  float* cnorm = reinterpret_cast<float*>(smem + p.off_cnorm);
  const uint32_t low = p.low_mask;
  int ds = 0, rs = 0;
  uint32_t dph = 0, rph = 0;
  int lt = 0;
  float colmax2 = 0.f;  // this warp's largest squared R2 column norm (first tile)

  // R2 stage of the current logit tile: wait until it is in shared memory.
  auto r2_stage = [&](int pt, int& st) -> bool {
    if (p.r2_resident) {
      st = pt;
      return wait_bar(&b.r2_full[pt], 0, b.abort_flag, a.status);
    }
    st = rs;
    return wait_bar(&b.r2_full[rs], rph, b.abort_flag, a.status);
  };
  // This warp is done with the R2 stage of the current logit tile; it arrives for
  // `count` consumer warps (0: only advance the stage counters).
  auto r2_release = [&](uint32_t count) {
    if (p.r2_resident) return;
    if (count) {
      __syncwarp();
      if (lane == 0) mbar_arrive_count(&b.r2_empty[rs], count);
    }
    if (++rs == p.r2_stages) {
      rs = 0;
      rph ^= 1u;
    }
  };

  for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++lt) {
    const int64_t n0 = (int64_t)tile * kBT;
    const int buf = lt & 1;
    // ---------------- Z epilogue (warpgroups 0, 1): TMEM -> (z_hi, z_lo) -> smem ----------
    if (g < 2) {
      if (!wait_bar(&b.zacc_full[buf], (lt >> 1) & 1, b.abort_flag, a.status)) return;
      tc_fence_after();
      constexpr int HALF = R / 2;
      uint32_t zr[HALF];
      const uint32_t taddr = tmem_base + lane_base + C::ZCOL0 + buf * C::ZCOLS + g * HALF;
      if constexpr (HALF == 8) {
        tmem_ld_x8(taddr, zr);
      } else if constexpr (HALF == 16) {
        tmem_ld_x16(taddr, zr);
      } else {
#pragma unroll
        for (int q = 0; q < HALF / 32; ++q) tmem_ld_x32(taddr + q * 32, zr + q * 32);
      }
      tmem_wait_ld();
      reg_fence<HALF>(zr);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&b.zacc_empty[buf]);
      // the previous tile's logit MMAs must be done with the z buffer
      if (lt > 0 && !wait_bar(b.zsm_empty, (lt - 1) & 1, b.abort_flag, a.status)) return;
      float hi2 = 0.f, lo2 = 0.f;
#pragma unroll
      for (int q = 0; q < HALF / 8; ++q) {
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float z0 = __uint_as_float(zr[q * 8 + 2 * j]), z1 = __uint_as_float(zr[q * 8 + 2 * j + 1]);
          __nv_bfloat16 h0 = __float2bfloat16_rn(z0), h1 = __float2bfloat16_rn(z1);
          __nv_bfloat16 l0 = __float2bfloat16_rn(z0 - __bfloat162float(h0));
          __nv_bfloat16 l1 = __float2bfloat16_rn(z1 - __bfloat162float(h1));
          const float fh0 = __bfloat162float(h0), fh1 = __bfloat162float(h1);
          const float fl0 = __bfloat162float(l0), fl1 = __bfloat162float(l1);
          hi2 = fmaf(fh0, fh0, fmaf(fh1, fh1, hi2));
          lo2 = fmaf(fl0, fl0, fmaf(fl1, fl1, lo2));
          hi[j] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
          lo[j] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
        }
        const int i0 = g * HALF + q * 8;  // first z index of this 8-group
        *reinterpret_cast<uint4*>(zs + zs_offset<R, KCAP>(t, i0 >> 3)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(zs + zs_offset<R, KCAP>(t, (R + i0) >> 3)) =
            make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
      znorm[g * kBT + t] = hi2;
      znorm[(2 + g) * kBT + t] = lo2;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(b.zsm_full);
    }

    // ---------------- pass 1: chunk maxima of z_hi . R2 -> top KL chunk keys -------------
    // warpgroup g owns columns 32 g .. 32 g + 31 of every 128-expert tile.
    uint32_t kl[KL];
#pragma unroll
    for (int i = 0; i < KL; ++i) kl[i] = 0u;
    for (int pt = 0; pt < p.p_count; ++pt) {
      if (!wait_bar(&b.d_full[ds], dph, b.abort_flag, a.status)) return;
      tc_fence_after();
      uint32_t v[32];
      tmem_ld_x32(tmem_base + lane_base + ds * 128 + g * 32, v);
      tmem_wait_ld();
      reg_fence<32>(v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&b.d_empty[ds]);
      if (++ds == C::ND) {
        ds = 0;
        dph ^= 1u;
      }
      if (lt == 0) {
        // first tile of this CTA: squared column norms of R2 (experts 8 cw .. 8 cw + 7 of the stage)
        int st;
        if (!r2_stage(pt, st)) return;
        const uint8_t* base = r2s + st * C::R2_STAGE;
        const int el = 8 * cw + (lane & 7);
        float acc = 0.f;
#pragma unroll 4
        for (int i = lane >> 3; i < R; i += 4) {
          const float w = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(base + r2_offset<R>(i, el)));
          acc = fmaf(w, w, acc);
        }
        acc += __shfl_xor_sync(0xffffffffu, acc, 8);
        acc += __shfl_xor_sync(0xffffffffu, acc, 16);
        colmax2 = fmaxf(colmax2, acc);
        r2_release(1);
      } else {
        r2_release(cw == 0 ? kConsumerWarps : 0);  // nobody reads R2 here: one warp arrives for all
      }
      const int c = pt * 4 + g;
      if (32 * c + 32 > a.M) {  // out-of-range experts at -infinity (Algorithm 1)
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (32 * c + j >= a.M) v[j] = 0xff800000u;
      }
      key_insert<KL>(kl, (ord_key(max32(v)) & ~low) | (uint32_t)c);
    }

    // ---------------- select: merge the lists, certified window, needed pairs --------------
    // two-round merge of the four partial lists: g2 -> g0 and g3 -> g1, then g1 -> g0
    if (g >= 2) {
#pragma unroll
      for (int i = 0; i < KL; ++i) lists[((g - 2) * KL + i) * kBT + t] = kl[i];
    }
    if (lt == 0) {
      colmax2 = fmaxf(colmax2, __shfl_xor_sync(0xffffffffu, colmax2, 1));
      colmax2 = fmaxf(colmax2, __shfl_xor_sync(0xffffffffu, colmax2, 2));
      colmax2 = fmaxf(colmax2, __shfl_xor_sync(0xffffffffu, colmax2, 4));
      if (lane == 0) cnorm[cw] = colmax2;
    }
    if (!consumer_sync(b, cph, a.status)) return;
    if (lt == 0 && ctid == 0) {
      float m = 0.f;
      for (int w = 0; w < kConsumerWarps; ++w) m = fmaxf(m, cnorm[w]);
      cnorm[kConsumerWarps] = sqrtf(m) * (1.f + 0x1p-20f);  // max column norm of R2, rounded up
    }
    if (g < 2) {
#pragma unroll
      for (int i = 0; i < KL; ++i) key_insert<KL>(kl, lists[(g * KL + i) * kBT + t]);
      if (g == 1) {  // each thread rewrites only its own column of slot 1
#pragma unroll
        for (int i = 0; i < KL; ++i) lists[(KL + i) * kBT + t] = kl[i];
      }
    }
    if (!consumer_sync(b, cph, a.status)) return;
    if (g == 0) {
#pragma unroll
      for (int i = 0; i < KL; ++i) key_insert<KL>(kl, lists[(KL + i) * kBT + t]);
      const bool active = n0 + t < a.N;
      // Certified window: values from z_hi differ from the z_hi + z_lo values by at most
      // eps = |z_lo| cmax (Cauchy-Schwarz) plus a bound on fp32 accumulation differences.
      const float cmax = cnorm[kConsumerWarps];
      const float zh = sqrtf(znorm[t] + znorm[kBT + t]);
      const float zl = sqrtf(znorm[2 * kBT + t] + znorm[3 * kBT + t]);
      const float eps = (zl * cmax) * (1.f + 0x1p-8f) + (float)R * 0x1p-20f * zh * cmax + 1e-30f;
      uint32_t kth = 0;
#pragma unroll
      for (int i = 0; i < KL; ++i)
        if (i == a.k - 1) kth = kl[i];
      int f = active ? 0 : 2;
      // The k chunks with the largest z_hi maxima (>= tlow) hold k elements whose exact logit
      // is >= tlow - eps, so the exact k-th logit is >= tlow - eps (the candidate cut), and an
      // element reaching it has a z_hi logit >= tlow - 2 eps (the chunk cut).
      float ccut = -INFINITY;                  // candidates: exact logit >= ccut
      uint32_t cut_key = 0u;                   // chunks whose key range reaches cut_key are needed
      if ((kth & ~low) >= kRealKey) {
        const float tlow = ord_inv(kth & ~low);  // <= the k-th largest z_hi chunk maximum
        ccut = __fsub_rd(tlow, eps);
        cut_key = ord_key(__fsub_rd(tlow, __fmul_ru(2.f, eps)));
        if ((kl[KL - 1] & ~low) >= kRealKey && (kl[KL - 1] | low) >= cut_key) f |= 1;  // list too short
      }
      int needed = 0;
      if (f == 0) {
#pragma unroll
        for (int i = 0; i < KL; ++i) {
          if ((kl[i] & ~low) >= kRealKey && (kl[i] | low) >= cut_key) {
            const uint32_t cid = kl[i] & low;
            const int rank = atomicAdd(&ccount[cid], 1);
            stage[i * kBT + t] = cid | ((uint32_t)rank << 16);  // until the bucket bases are known
            needed = i + 1;
          }
        }
      }
      thr[t] = ccut;
      flag[t] = f;
      nq[t] = (uint8_t)needed;
      poolcnt[t] = 0;
      if (t == 0 && g == 0) *fbcount = 0;
    }
    if (!consumer_sync(b, cph, a.status)) return;
    // exclusive prefix of the per-chunk pair counts (chunks 0 .. nchunks; the last is empty)
    {
      int vals[4], run = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = ctid * 4 + j;
        vals[j] = (i < p.nchunks) ? ccount[i] : 0;
        run += vals[j];
      }
      int incl = run;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += o;
      }
      if (lane == 31) scan[ctid >> 5] = incl;
      if (!consumer_sync(b, cph, a.status)) return;
      int before = incl - run;
      for (int w = 0; w < (ctid >> 5); ++w) before += scan[w];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = ctid * 4 + j;
        if (i <= p.nchunks) cbase[i] = before;
        if (i < p.nchunks) ccount[i] = 0;
        before += vals[j];
      }
      // the end of the last bucket (index nchunks lies past the 4 x 512 slots when nchunks == 2048)
      if (ctid == kConsumerThreads - 1) cbase[p.nchunks] = before;
    }
    if (!consumer_sync(b, cph, a.status)) return;
    if (g == 0) {
      const int needed = nq[t];
      const float cut = thr[t];
      for (int i = 0; i < needed; ++i) {
        const uint32_t st = stage[i * kBT + t];
        // {token | needed-chunk index << 8, candidate cut}
        pairs[cbase[st & 0xffffu] + (st >> 16)] = make_uint2((uint32_t)t | ((uint32_t)i << 8), __float_as_uint(cut));
      }
    }
    if (!consumer_sync(b, cph, a.status)) return;

    // ---------------- pass 2: candidates of the needed chunks (exact z_hi + z_lo logits) ----
    // Lane group sp of the transposed tile is chunk 4 pt + sp.  Tile pt belongs to
    // warpgroups 0-1 when pt is even, 2-3 when odd: the two warps of a lane group split the
    // pairs of their chunk (first and second half), so a tile is worked by eight warps and
    // two tiles at once.  Every warp waits for every tile and arrives once on its empty
    // barrier (the owners when done, the others at once): a buffer is refilled only after
    // all sixteen warps have seen its current phase, so no warp can fall two phases
    // behind, which a parity wait could not tell from the phase it waits for.
    for (int pt = 0; pt < p.p_count; ++pt) {
      if (!wait_bar(&b.d_full[ds], dph, b.abort_flag, a.status)) return;
      if ((pt & 1) == (g >> 1)) {
        tc_fence_after();
        const int c = pt * 4 + sp;
        if (c < p.nchunks) {
          const int e = 32 * c + lane;
          const bool e_ok = e < a.M;
          const uint32_t col0 = tmem_base + lane_base + ds * 128;
          const uint32_t lt_mask = (1u << lane) - 1u;
          const int c_lo = cbase[c], c_hi = cbase[c + 1], c_mid = (c_lo + c_hi + 1) >> 1;
          const int lo = (g & 1) ? c_mid : c_lo, hi = (g & 1) ? c_hi : c_mid;
          for (int pi = lo; pi < hi; pi += kPairBatch) {
            const int nb = hi - pi < kPairBatch ? hi - pi : kPairBatch;
            uint2 ent[kPairBatch];
            uint32_t val[kPairBatch];
#pragma unroll
            for (int q = 0; q < kPairBatch; ++q)
              if (q < nb) ent[q] = pairs[pi + q];  // {token | slot << 8, candidate cut}
#pragma unroll
            for (int q = 0; q < kPairBatch; ++q)
              if (q < nb) val[q] = tmem_ld_x1(col0 + (ent[q].x & 0xffu));
            tmem_wait_ld();
            reg_fence<kPairBatch>(val);
            // per pair: ballot the experts at or above the cut; the first one takes the
            // pair's slot, lane 0 records the count, any further ones go to the pool below
            uint32_t bal[kPairBatch];
            uint32_t extra = 0u;
#pragma unroll
            for (int q = 0; q < kPairBatch; ++q) {
              const bool take = q < nb && e_ok && __uint_as_float(val[q]) >= __uint_as_float(ent[q].y);
              bal[q] = __ballot_sync(0xffffffffu, take);
              const uint32_t tq = ent[q].x & 0xffu, iq = ent[q].x >> 8;
              const uint32_t before = bal[q] & lt_mask;
              if (take && before == 0u) cand[iq * kBT + tq] = make_uint2(val[q], (uint32_t)e);
              if (lane == 0 && q < nb) pc[tq * C::KLP + iq] = (uint8_t)__popc(bal[q]);
              extra |= bal[q] & (bal[q] - 1u);  // set iff the pair has two or more candidates
            }
            if (extra) {  // rare: more candidates than the pair's slot
#pragma unroll
              for (int q = 0; q < kPairBatch; ++q) {
                if (((bal[q] >> lane) & 1u) && (bal[q] & lt_mask)) {
                  const int tok = ent[q].x & 0xff;
                  const int ps = atomicAdd(&poolcnt[tok], 1);
                  if (ps < kPoolSlots) pool[ps * kBT + tok] = make_uint2(val[q], (uint32_t)e);
                }
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&b.d_empty[ds]);
        r2_release(kConsumerWarps / 8);  // the tile's eight warps stand for all sixteen
      } else {
        __syncwarp();
        if (lane == 0) mbar_arrive(&b.d_empty[ds]);
        r2_release(0);
      }
      if (++ds == C::ND) {
        ds = 0;
        dph ^= 1u;
      }
    }
    if (!consumer_sync(b, cph, a.status)) return;

    // ---------------- finalize: order, softmax, store, count ---------------------------
    // Four threads per token (one per warpgroup).  Every thread loads all of the token's
    // candidates (the slots of its needed chunks, then its pool entries); thread g ranks
    // candidates g, g + 4, ... in routing order (larger logit, then lower expert) and the
    // ones of rank < k go to the output staging at their rank, with exp(logit - max).
    {
      constexpr int NC = KL + kPoolSlots;
      int32_t* sidx = reinterpret_cast<int32_t*>(pairs);  // staging: [token][k], like the outputs
      float* sex = reinterpret_cast<float*>(sidx + kBT * a.k);
      float* slog = sex + kBT * a.k;
      const int f = flag[t];
      if ((f & 2) == 0) {
        const int jn = nq[t], np = poolcnt[t];
        uint32_t cnt[C::KLP / 4];
#pragma unroll
        for (int w = 0; w < C::KLP / 16; ++w) {
          const uint4 q4 = *reinterpret_cast<const uint4*>(pc + t * C::KLP + 16 * w);
          cnt[4 * w] = q4.x;
          cnt[4 * w + 1] = q4.y;
          cnt[4 * w + 2] = q4.z;
          cnt[4 * w + 3] = q4.w;
        }
        // -0 and +0 are equal in routing order: both take the key of +0.  Empty slots take
        // key 0, below every real value, so they never outrank a candidate.
        uint32_t o[NC], e[NC];
        int total = 0;
#pragma unroll
        for (int q = 0; q < NC; ++q) {
          bool has;
          uint2 cv = make_uint2(0u, 0u);
          if (q < KL) {
            const int nc = q < jn ? (int)((cnt[q >> 2] >> (8 * (q & 3))) & 0xffu) : 0;
            total += nc;
            has = nc > 0;
            if (has) cv = cand[q * kBT + t];
          } else {
            has = q - KL < np;
            if (has) cv = pool[(q - KL) * kBT + t];
          }
          o[q] = has ? ord_key(__uint_as_float(cv.x) + 0.f) : 0u;
          e[q] = cv.y;
        }
        const bool fb = (f & 1) || np > kPoolSlots || total < a.k;
        if (g == 0) {
          fbmark[t] = fb ? 1 : 0;
          if (fb) fblist[atomicAdd(fbcount, 1)] = (uint8_t)t;
        }
        if (!fb) {
          uint32_t top = 0u;
#pragma unroll
          for (int q = 0; q < NC; ++q) top = max(top, o[q]);
          const float vtop = ord_inv(top);
          for (int q = g; q < NC; q += 4) {
            uint2 cv = make_uint2(0u, 0u);
            bool has;
            if (q < KL) {
              has = q < jn && pc[t * C::KLP + q] != 0;
              if (has) cv = cand[q * kBT + t];
            } else {
              has = q - KL < np;
              if (has) cv = pool[(q - KL) * kBT + t];
            }
            if (!has) continue;
            const uint32_t om = ord_key(__uint_as_float(cv.x) + 0.f), em = cv.y;
            int rank = 0;
#pragma unroll
            for (int j = 0; j < NC; ++j) rank += (o[j] > om || (o[j] == om && e[j] < em)) ? 1 : 0;
            if (rank < a.k) {
              const float v = ord_inv(om);
              sidx[t * a.k + rank] = (int)em;
              sex[t * a.k + rank] = expf(v - vtop);
              slog[t * a.k + rank] = v;
              if (em < (uint32_t)a.M) atomicAdd(a.out_count + em, 1);
            }
          }
        }
      }
      if (!consumer_sync(b, cph, a.status)) return;
      // gates: each selected exp divided by its token's sum
      if (g == 0 && (f & 2) == 0 && !fbmark[t]) {
        float sum = 0.f;
        for (int j = 0; j < a.k; ++j) sum += sex[t * a.k + j];
        const float inv = 1.f / sum;
        for (int j = 0; j < a.k; ++j) sex[t * a.k + j] *= inv;
      }
      if (!consumer_sync(b, cph, a.status)) return;
      // the tile's outputs are contiguous: copy the staging out with coalesced stores
      const int rows = a.N - n0 < kBT ? (int)(a.N - n0) : kBT;
      const size_t ob = (size_t)n0 * a.k;
      for (int x = ctid; x < rows * a.k; x += kConsumerThreads) {
        if (fbmark[x / a.k]) continue;
        a.out_idx[ob + x] = sidx[x];
        a.out_gate[ob + x] = sex[x];
        if (a.out_logits) a.out_logits[ob + x] = slog[x];
      }
    }
    // fallback tokens, kFbBatch at a time: every consumer warp ranks its 256-expert blocks
    // (blocks cw, cw + 16, ...) for each token, then warp j merges the 16 partial lists of
    // the batch's token j and writes it
    for (int fb0 = 0, nfb = *fbcount; fb0 < nfb; fb0 += kFbBatch) {
      const int nb = nfb - fb0 < kFbBatch ? nfb - fb0 : kFbBatch;
      fallback_rank<R, KCAP>(a, zs, fblist + fb0, nb, part, cw, lane);
      if (!consumer_sync(b, cph, a.status)) return;
      if (cw < nb) fallback_merge<KCAP>(a, part + cw * kConsumerWarps * KCAP, n0 + fblist[fb0 + cw], lane);
      if (!consumer_sync(b, cph, a.status)) return;
    }
  }
}

// ---- kernel -----------------------------------------------------------------------------

template <int R, int KCAP>
__global__ void __launch_bounds__(kThreads, 1)
    fused_route_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmR1,
                       const __grid_constant__ CUtensorMap tmR2, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Bars b = bars_at(smem, p);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < p.x_stages; ++i) {
      mbar_init(&b.x_full[i], 1);
      mbar_init(&b.x_empty[i], 1);
    }
    const int nr2 = p.r2_resident ? p.p_count : p.r2_stages;
    for (int i = 0; i < nr2; ++i) {
      mbar_init(&b.r2_full[i], 1);
      mbar_init(&b.r2_empty[i], 1 + kConsumerWarps);  // the MMA commit and every consumer warp
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&b.zacc_full[i], 1);
      mbar_init(&b.zacc_empty[i], 8);
      mbar_init(&b.drain[i], 1);
    }
    for (int i = 0; i < 3; ++i) {
      mbar_init(&b.d_full[i], 1);
      mbar_init(&b.d_empty[i], kConsumerWarps);
    }
    mbar_init(b.zsm_full, 8);
    mbar_init(b.zsm_empty, 1);
    mbar_init(b.cbar, kConsumerWarps);
    *b.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmX);
    prefetch_tensormap(&tmR1);
    prefetch_tensormap(&tmR2);
  }
  if (warp == 1) {
    tmem_alloc(b.tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp >= 4) {  // clear the per-chunk pair counters
    int* ccount = reinterpret_cast<int*>(smem + p.off_ccount);
    for (int i = threadIdx.x - 128; i < p.nchunks; i += kConsumerThreads) ccount[i] = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *b.tmem_slot;

  if (warp == 0) {
    if (lane == 0) producer_x<R, KCAP>(p, b, smem, &tmX, &tmR1);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) mma_z<R, KCAP>(p, b, smem, tmem_base);
    __syncwarp();
  } else if (warp == 2) {
    if (lane == 0) mma_scores<R, KCAP>(p, b, smem, tmem_base);
    __syncwarp();
  } else if (warp == 3) {
    if (lane == 0) producer_r2<R, KCAP>(p, b, smem, &tmR2);
    __syncwarp();
  } else {
    consumers<R, KCAP>(p, b, smem, tmem_base);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ---- host side ----------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
              uint32_t box_outer, CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr uint32_t kSmemLimit = 227 * 1024;

uint32_t align_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

// Shared-memory plan; returns the total bytes (0 when nothing fits).
template <int R, int KCAP>
uint32_t plan(Params& p) {
  using C = Cfg<R, KCAP>;
  for (int xs = 4; xs >= 2; --xs) {
    for (int mode = 0; mode < 2; ++mode) {  // 0: R2 resident, 1: streamed
      const int r2s = mode == 0 ? p.p_count : 8;
      if (mode == 0 && p.p_count > 64) continue;
      for (int r2n = r2s; r2n >= 2 || (mode == 0 && r2n == r2s); --r2n) {
        uint32_t off = 0;
        p.off_x = off;
        off += xs * C::X_STAGE;
        p.off_r1 = off = align_up(off, 1024);
        off += xs * C::R1_STAGE;
        p.off_r2 = off = align_up(off, 1024);
        off += r2n * C::R2_STAGE;
        p.off_zs = off = align_up(off, 1024);
        off += C::ZS_BYTES;
        // candidate slots and the list exchange + pair staging share memory (disjoint lifetimes)
        // (and, after the finalize, the partial lists of the cooperative fallback)
        const uint32_t cand_bytes = kBT * C::KLP * C::S * 8, list_bytes = 3 * kBT * C::KL * 4;
        const uint32_t part_bytes = kFbBatch * kConsumerWarps * KCAP * 8;
        uint32_t shared_bytes = cand_bytes > list_bytes ? cand_bytes : list_bytes;
        if (part_bytes > shared_bytes) shared_bytes = part_bytes;
        p.off_cand = p.off_lists = off = align_up(off, 16);
        off += shared_bytes;
        p.off_thr = off;
        off += kBT * 4;
        p.off_flag = off;
        off += kBT * 4;
        p.off_pairs = off = align_up(off, 16);  // pass-2 pairs; in the finalize, the output staging
        {
          const uint32_t pair_bytes = kBT * C::KL * 8, staging_bytes = 3 * kBT * KCAP * 4;
          off += pair_bytes > staging_bytes ? pair_bytes : staging_bytes;
        }
        p.off_ccount = off;
        off += p.nchunks * 4;
        p.off_cbase = off;
        off += (p.nchunks + 1) * 4;
        p.off_scan = off = align_up(off, 16);
        off += kConsumerWarps * 4;
        p.off_znorm = off;           // per token: |z_hi|^2 and |z_lo|^2 partial sums of both halves
        off += 4 * kBT * 4;
        p.off_cnorm = off;           // per consumer warp: max squared column norm of R2; [16] = result
        off += (kConsumerWarps + 1) * 4;
        p.off_nq = off;
        off += kBT;
        p.off_fb = off = align_up(off, 4);  // fallback count, the tile's fallback tokens, per-token mark
        off += 4 + 2 * kBT;
        p.off_poolcnt = off = align_up(off, 4);
        off += kBT * 4;
        p.off_pool = off = align_up(off, 8);
        off += kBT * kPoolSlots * 8;
        p.off_pc = off = align_up(off, 16);
        off += kBT * C::KLP;
        p.off_bar = off = align_up(off, 8);
        off += kBarBytes;
        const uint32_t total = off + 1024;  // alignment slack of the dynamic base
        if (total <= kSmemLimit) {
          p.x_stages = xs;
          p.r2_stages = r2n;
          p.r2_resident = mode == 0;
          return total;
        }
        if (mode == 0) break;
      }
    }
  }
  return 0;
}

template <int R, int KCAP>
bool fill_params(const RouteArgs& a, Params& p, uint32_t& smem) {
  p.a = a;
  p.num_tiles = (int)((a.N + kBT - 1) / kBT);
  p.kb_count = (a.h + Cfg<R, KCAP>::BK - 1) / Cfg<R, KCAP>::BK;
  p.p_count = (a.M + kBE - 1) / kBE;
  p.nchunks = (a.M + 31) / 32;
  int bits = 1;  // chunk ids run up to 4 p_count - 1 (the padded last tile)
  while ((1 << bits) < 4 * p.p_count) ++bits;
  p.low_mask = (1u << bits) - 1u;
  smem = plan<R, KCAP>(p);
  return smem != 0;
}

template <int R, int KCAP>
cudaError_t launch(const RouteArgs& a) {
  using C = Cfg<R, KCAP>;
  Params p;
  uint32_t smem = 0;
  if (!fill_params<R, KCAP>(a, p, smem)) return cudaErrorInvalidConfiguration;
  CUtensorMap tmX, tmR1, tmR2;
  const CUtensorMapSwizzle r1sw = C::R1_ROW == 32   ? CU_TENSOR_MAP_SWIZZLE_32B
                                  : C::R1_ROW == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                    : CU_TENSOR_MAP_SWIZZLE_128B;
  const CUtensorMapSwizzle xsw = C::BK == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  if (!make_map(&tmX, a.X, (uint64_t)a.h, (uint64_t)a.N, C::BK, kBT, xsw) ||
      !make_map(&tmR1, a.R1, (uint64_t)R, (uint64_t)a.h, C::R1_BOX, C::BK, r1sw) ||
      !make_map(&tmR2, a.R2, (uint64_t)a.M, (uint64_t)R, 64, R, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  static int configured = 0;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(fused_route_kernel<R, KCAP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemLimit);
    if (e != cudaSuccess) return e;
    configured = 1;
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = p.num_tiles < sms ? p.num_tiles : sms;
  fused_route_kernel<R, KCAP><<<grid, kThreads, smem, a.stream>>>(tmX, tmR1, tmR2, p);
  return cudaGetLastError();
}

template <int R>
cudaError_t launch_r(const RouteArgs& a) {
  if (a.k <= 4) return launch<R, 4>(a);
  if (a.k <= 8) return launch<R, 8>(a);
  return launch<R, 16>(a);
}

template <int R>
bool supports_r(const RouteArgs& a) {
  Params p;
  uint32_t smem;
  if (a.k <= 4) return fill_params<R, 4>(a, p, smem);
  if (a.k <= 8) return fill_params<R, 8>(a, p, smem);
  return fill_params<R, 16>(a, p, smem);
}

}  // namespace tc

bool fused_tc_supports(const RouteArgs& a) {
  // 65536 experts = 2048 chunks: the pair-count scan covers 4 chunks per consumer thread
  if (a.M > 65536 || a.k > 16 || a.N < 1 || a.N > 0x7fffffffLL - tc::kBT) return false;
  if (!tc::encode_fn()) return false;
  switch (a.r) {
    case 16: return tc::supports_r<16>(a);
    case 32: return tc::supports_r<32>(a);
    case 64: return tc::supports_r<64>(a);
    case 128: return tc::supports_r<128>(a);
    default: return false;
  }
}

cudaError_t launch_fused_tc(const RouteArgs& a) {
  switch (a.r) {
    case 16: return tc::launch_r<16>(a);
    case 32: return tc::launch_r<32>(a);
    case 64: return tc::launch_r<64>(a);
    case 128: return tc::launch_r<128>(a);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace more

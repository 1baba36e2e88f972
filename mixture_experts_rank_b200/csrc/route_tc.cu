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
// How (one persistent CTA per SM, 128-token tiles, 20 warps, each with one role):
//   warp 0  TMA producer of the X (128 x BK bf16, swizzled) and R1 (BK x r) stages and of
//           the R2 tiles (r x 128 experts); R2 stays resident in shared memory when it
//           fits, else it is streamed from L2 once per sweep.  It polls both rings.
//   warp 1  MMA issuer for Z = X R1: M=128 tokens, N=r, K=16 steps over h, into a
//           double-buffered TMEM accumulator (the next tiles stream while the
//           current ones are routed, so HBM never waits on the top-k).
//   warp 2  MMA issuer of pass A: D[tok, exp] = z_hi R2 (K = r), 128 experts a job.
//   warp 3  MMA issuer of pass B: D[tok, exp] = [z_hi | z_lo] [R2 ; R2] (K = 2r, exact to
//           ~16 bits of z), 128 experts a job.
//   warps 4-11   group A (two warps per TMEM lane group): per tile
//     epilogue  Z from TMEM -> (z_hi, z_lo) bf16 pair -> shared memory (K-major),
//               plus |z_hi|, |z_lo| per token and (first tile) the largest column norm
//               of R2.
//     pass A    every 32-expert chunk of a token is reduced to the maximum of its z_hi
//               logits, packed into a 32-bit key (order-preserving value bits above the
//               chunk id); a branch-free sorted list keeps the best k keys per warp.
//     select    the two lists of a token are merged.  z_hi logits differ from the exact
//               ones by at most eps (|z_lo| times the largest R2 column norm, plus fp32
//               rounding), and the k chunks with the largest z_hi maxima (>= tlow) hold k
//               experts whose exact logit is >= tlow - eps, so the exact k-th logit is at
//               least the cut tlow - eps.  The cut of every token is handed to group B.
//   warps 12-19  group B (two warps per TMEM lane group): per tile
//     pass B    each warp reads its 64 columns of every exact tile, reduces each 8-expert
//               octet to its maximum, and stores the octets that reach the token's cut
//               (about k + 1 per token) whole in the token's octet slots, with predicated
//               shared-memory stores; the two warps of a lane group fill the slots from
//               opposite ends, each counting in a register.
//     finalize  one thread per token walks its stored octets and keeps the best k logits
//               that reach the cut as sorted 64-bit routing keys (larger logit, then lower
//               expert), writes them with the softmax gates to a shared-memory staging of
//               the outputs, which the tile writes with coalesced stores, and counts them.
//               A token whose octets overflowed the slots goes to an exact recomputation on
//               CUDA cores shared by the group.
// The logit MMAs run in sweeps over the expert tiles: each sweep streams R2 once and every
// R2 tile feeds pass B of tile t and pass A of tile t + 1 (with two z buffers; otherwise a
// sweep carries one pass), so group B works on tile t while group A works on tile t + 1.
// Every mbarrier wait is bounded (a few seconds); on expiry the kernel records
// MORE_DEVERR_WAIT_TIMEOUT in the library's device error word and every role unwinds.  A
// group's select or finalize is entered through a bounded barrier of its eight warps; inside
// it the warps synchronise with a named barrier and nothing waits on another role, so every
// warp that enters reaches every named barrier.
#include <cudaTypedefs.h>

#include <atomic>
#include <cfloat>

#include "more_internal.cuh"
#include "mbar_wait.cuh"
#include "sm100_ptx.cuh"
#include "warp_simt.cuh"

namespace more {
namespace tc {

using namespace sm100;

constexpr int kBT = 128;        // tokens per tile (MMA M of Z and pass A, N of pass B)
constexpr int kBE = 128;        // experts per logit tile
constexpr int kRoleWarps = 4;
#ifndef MORE_GROUP_B_WARPS
#define MORE_GROUP_B_WARPS 8
#endif
constexpr int kWarpsA = 8;                       // group A: two warps per TMEM lane group
constexpr int kWarpsB = MORE_GROUP_B_WARPS;      // group B: kWarpsB / 4 warps per TMEM lane group
constexpr int kThreadsA = kWarpsA * 32, kThreadsB = kWarpsB * 32;
constexpr int kWarpA0 = kRoleWarps, kWarpB0 = kRoleWarps + kWarpsA;
constexpr int kThreads = (kRoleWarps + kWarpsA + kWarpsB) * 32;
constexpr int kNamedBarA = 1, kNamedBarB = 2;    // bar.sync ids of the groups
static_assert(kWarpsB % 4 == 0, "group B covers the four TMEM lane groups evenly");
static_assert((kWarpsB & (kWarpsB - 1)) == 0, "fallback teams divide group B evenly");
static_assert(kWarpsB == 8, "pass B splits each 128-expert tile into two 64-column halves per lane group");
constexpr int kFbBatch = 8;     // fallback tokens ranked per round of the cooperative fallback
static_assert(kFbBatch <= kWarpsB, "one merging warp per fallback token of a batch");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kRealKey = 0x00800000u;  // ordered value of -FLT_MAX: keys below are not real chunks

// ---- parameters -----------------------------------------------------------------------

struct Params {
  RouteArgs a;
  int num_tiles;     // token tiles
  int kb_count;      // hidden blocks of kBK
  int p_count;       // expert tiles of kBE
  uint32_t low_mask; // chunk-id bits of a key
  int x_stages;
  int r2_stages;
  int r2_resident;   // every expert tile stays in shared memory
  int interleave;    // two z buffers: a sweep carries pass B of one tile and pass A of the next
  uint32_t off_x, off_r1, off_r2, off_zs;
  // group A only
  uint32_t off_lists, off_znorm, off_cnorm;
  // handed from group A to group B, two buffers each: the cut and flags of every token
  uint32_t off_cut, off_flag;
  // group B only
  uint32_t off_slots, off_ids, off_hcnt, off_stage, off_fb, off_part;
  int fb_groups;  // warps per fallback token: min(kWarpsB, 256-expert blocks rounded up to a power of two)
  uint32_t off_bar;
};

template <int R, int KCAP>
struct Cfg {
  static constexpr int KA = KCAP;                      // chunk keys kept per token and warp in pass A
  // octet slots of pass B: every 8-expert octet that holds an expert at or above the token's cut
  // is stored whole (its eight exact logits and its index), up to OCT per token; a token with
  // more goes to the exact fallback.  The warp of the low column half fills a token's slots from
  // the first up, the other from the last down, so neither needs the other's count.
  static constexpr int OCT = R >= 128 ? KCAP + 4 : (R >= 64 ? KCAP + 5 : KCAP + 6);
  // In the finalize the octet slots take the output staging and, after it, the fallback's
  // partial lists.
  static constexpr uint32_t STAGE_BYTES = (3 * kBT * KCAP * 4 + 15) / 16 * 16;
  static constexpr uint32_t PART_BYTES = kFbBatch * kWarpsB * KCAP * 8;
  static_assert(STAGE_BYTES + PART_BYTES <= OCT * kBT * 32, "staging and partial lists fit the octet slots");
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
  static constexpr int NBUF = (512 - 2 * ZCOLS) / 128 < 3 ? (512 - 2 * ZCOLS) / 128 : 3;
#ifndef MORE_PASS_A_BUFS
#define MORE_PASS_A_BUFS 1
#endif
  static constexpr int NA = MORE_PASS_A_BUFS < NBUF ? MORE_PASS_A_BUFS : 1;  // TMEM buffers of pass A jobs
  static constexpr int NB = NBUF - NA;                 // TMEM buffers of pass B jobs (longer MMAs)
  static constexpr int ZCOL0 = NBUF * 128;             // first TMEM column of the Z accumulators
  static constexpr uint32_t IDESC_Z = idesc_bf16_f32(128, R, 0, 1);    // A = X (K-major), B = R1 (MN-major)
  static constexpr uint32_t IDESC_P = idesc_bf16_f32(128, 128, 0, 1);  // A = z pair, B = R2 tile
  static_assert(NB >= 1, "TMEM holds at least one buffer per pass");
};

// Jobs of one sweep over the expert tiles: pass A of local tile ta and pass B of local
// tile tb (-1: none).  Interleaved: sweep q carries A(q) and B(q - 1), so T tiles take
// T + 1 sweeps; otherwise sweep 2j carries A(j) and sweep 2j + 1 carries B(j).
struct Sweep {
  int ta, tb;
};
__host__ __device__ __forceinline__ Sweep sweep_jobs(int q, int T, int interleave) {
  if (interleave) return Sweep{q < T ? q : -1, q >= 1 ? q - 1 : -1};
  return (q & 1) ? Sweep{-1, q >> 1} : Sweep{q >> 1, -1};
}
__host__ __device__ __forceinline__ int sweep_count(int T, int interleave) {
  return T == 0 ? 0 : (interleave ? T + 1 : 2 * T);
}
// z buffer of local tile j and its use count on that buffer.
__device__ __forceinline__ int zs_buf(int j, int interleave) { return interleave ? (j & 1) : 0; }
__device__ __forceinline__ int zs_use(int j, int interleave) { return interleave ? (j >> 1) : j; }

// Barrier block layout (uint64_t slots).
struct Bars {
  uint64_t* x_full;      // [8]
  uint64_t* x_empty;     // [8]
  uint64_t* r2_full;     // [64]
  uint64_t* r2_empty;    // [64]
  uint64_t* zacc_full;   // [2] Z accumulators
  uint64_t* zacc_empty;  // [2]
  uint64_t* zsm_full;    // [2] z buffers in shared memory
  uint64_t* zsm_empty;   // [2]
  uint64_t* a_full;      // [2] pass A TMEM buffers
  uint64_t* a_empty;     // [2]
  uint64_t* b_full;      // [2] pass B TMEM buffers
  uint64_t* b_empty;     // [2]
  uint64_t* pairs_full;  // [2] pair buffers (group A -> group B)
  uint64_t* pairs_empty; // [2]
  uint64_t* gbar;        // [2] bounded entry barriers of groups A and B
  uint64_t* drain;       // [3]
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
  r.zsm_empty = r.zsm_full + 2;
  r.a_full = r.zsm_empty + 2;
  r.a_empty = r.a_full + 2;
  r.b_full = r.a_empty + 2;
  r.b_empty = r.b_full + 2;
  r.pairs_full = r.b_empty + 2;
  r.pairs_empty = r.pairs_full + 2;
  r.gbar = r.pairs_empty + 2;
  r.drain = r.gbar + 2;
  r.tmem_slot = reinterpret_cast<uint32_t*>(r.drain + 3);
  r.abort_flag = reinterpret_cast<int*>(r.tmem_slot + 1);
  return r;
}
constexpr uint32_t kBarSlots = 16 + 128 + 2 * 12 + 3;  // up to and with drain
constexpr uint32_t kBarBytes = kBarSlots * 8 + 16;

// Bounded entry barrier of one group's warps (an mbarrier, so that a warp of the
// group that gave up elsewhere cannot leave the others waiting without limit).  `phase` is
// the calling thread's parity of the barrier, flipped at every use.
__device__ __forceinline__ bool group_enter(uint64_t* gbar, uint32_t& phase, volatile int* abort_flag,
                                            unsigned int* status) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(gbar);
  const bool ok = bounded_wait(gbar, phase, abort_flag, status);
  phase ^= 1u;
  return ok;
}

// Named barrier of one group's threads.  Used only between a group_enter and the end of the
// same phase, where no thread waits on anything else.
__device__ __forceinline__ void group_bar(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
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

// Byte offset of R2 element (row i, expert e_local of a 128-expert stage) in the
// MN-major 128B-swizzled stage written by TMA (two boxes of 64 experts x R rows).
template <int R>
__device__ __forceinline__ uint32_t r2_offset(int i, int e_local) {
  const int box = e_local >> 6, col = e_local & 63;
  return (uint32_t)(box * (64 * R * 2) + i * 128 + ((((col >> 3) ^ (i & 7))) << 4) + (col & 7) * 2);
}

// Number of 128-token tiles this CTA routes (tiles blockIdx.x, blockIdx.x + gridDim.x, ...).
__device__ __forceinline__ int local_tiles(const Params& p) {
  return (int)blockIdx.x < p.num_tiles ? (p.num_tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
}


// ---- role: TMA producer of X, R1 and R2 ---------------------------------------------
//
// One thread keeps both rings full: X and R1 stages in tile order, R2 tiles in sweep order
// (or, when R2 is resident, all of them once).  It polls the rings' empty barriers without
// blocking and backs off briefly when neither has room, so a slow ring never holds up the
// other.  It gives up like every bounded wait: after kWaitLimitNs without progress, or when
// another role has raised the abort flag.

template <int R, int KCAP>
__device__ void producer(const Params& p, const Bars& b, uint8_t* smem, const CUtensorMap* tmX,
                         const CUtensorMap* tmR1, const CUtensorMap* tmR2) {
  using C = Cfg<R, KCAP>;
  auto load_r2 = [&](int slot, int t) {
    uint8_t* dst = smem + p.off_r2 + slot * C::R2_STAGE;
    mbar_arrive_expect_tx(&b.r2_full[slot], C::R2_STAGE);
    tma_load_2d(dst, tmR2, &b.r2_full[slot], t * kBE, 0);
    tma_load_2d(dst + C::R2_BOX_BYTES, tmR2, &b.r2_full[slot], t * kBE + 64, 0);
  };
  if (p.r2_resident)
    for (int t = 0; t < p.p_count; ++t) load_r2(t, t);
  // X side: local tile xt, hidden block kb
  RingPos sx, sr;
  int xt = 0, kb = 0;
  const int T = local_tiles(p);
  // R2 side: stage t of sweep q
  int q = 0, rt = 0;
  const int nsw = p.r2_resident ? 0 : sweep_count(T, p.interleave);
  uint64_t idle_since = global_timer_ns();
  uint32_t polls = 0;
  while (xt < T || q < nsw) {
    bool progress = false;
    if (xt < T && mbar_test_wait(&b.x_empty[sx.i], sx.phase ^ 1u)) {
      const int tile = (int)blockIdx.x + xt * (int)gridDim.x;
      mbar_arrive_expect_tx(&b.x_full[sx.i], C::X_STAGE + C::R1_STAGE);
      tma_load_2d(smem + p.off_x + sx.i * C::X_STAGE, tmX, &b.x_full[sx.i], kb * C::BK, tile * kBT);
#pragma unroll
      for (int r = 0; r < C::R1_BOXES; ++r)
        tma_load_2d(smem + p.off_r1 + sx.i * C::R1_STAGE + r * C::R1_BOX_BYTES, tmR1, &b.x_full[sx.i], r * 64,
                    kb * C::BK);
      sx.next(p.x_stages);
      if (++kb == p.kb_count) {
        kb = 0;
        ++xt;
      }
      progress = true;
    }
    if (q < nsw && mbar_test_wait(&b.r2_empty[sr.i], sr.phase ^ 1u)) {
      load_r2(sr.i, rt);
      sr.next(p.r2_stages);
      if (++rt == p.p_count) {
        rt = 0;
        ++q;
      }
      progress = true;
    }
    if (progress) {
      polls = 0;
      continue;
    }
    __nanosleep(64);
    if ((++polls & 63u) == 0) {
      if (*reinterpret_cast<volatile int*>(b.abort_flag)) return;
      const uint64_t now = global_timer_ns();
      if (polls == 64) idle_since = now;
      if (now - idle_since > kWaitLimitNs) {
        atomicOr(p.a.status, MORE_DEVERR_WAIT_TIMEOUT);
        *reinterpret_cast<volatile int*>(b.abort_flag) = 1;
        return;
      }
    }
  }
}

// ---- role: MMA issuer of Z = X R1 ------------------------------------------------------

template <int R, int KCAP>
__device__ void mma_z(const Params& p, const Bars& b, uint8_t* smem, uint32_t tmem_base) {
  using C = Cfg<R, KCAP>;
  RingPos s;
  int lt = 0;
  const uint32_t x0 = smem_u32(smem + p.off_x), r10 = smem_u32(smem + p.off_r1);
  for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++lt) {
    const int buf = lt & 1;
    if (!bounded_wait(&b.zacc_empty[buf], ((lt >> 1) & 1) ^ 1u, b.abort_flag, p.a.status)) break;
    tc_fence_after();
    const uint32_t d = tmem_base + C::ZCOL0 + buf * C::ZCOLS;
    for (int kb = 0; kb < p.kb_count; ++kb) {
      if (!bounded_wait(&b.x_full[s.i], s.phase, b.abort_flag, p.a.status)) goto done;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < C::BK / 16; ++kk) {
        uint64_t ad = smem_desc(x0 + s.i * C::X_STAGE + kk * 32, 16, C::X_SBO, C::X_LAYOUT);
        uint64_t bd = smem_desc(r10 + s.i * C::R1_STAGE + kk * 16 * C::R1_ROW, C::R1_BOX_BYTES, 8 * C::R1_ROW,
                                C::R1_LAYOUT);
        mma_bf16(d, ad, bd, C::IDESC_Z, (kb | kk) != 0);
      }
      mma_commit(&b.x_empty[s.i]);
      s.next(p.x_stages);
    }
    mma_commit(&b.zacc_full[buf]);
  }
done:
  mma_commit(&b.drain[0]);
  bounded_wait(&b.drain[0], 0, b.abort_flag, p.a.status);
}

// ---- roles: MMA issuers of the logit passes ---------------------------------------------
//
// Both issuers walk every sweep's R2 tiles in order.  For each tile they release their
// share of the R2 stage: a commit when they issued MMAs that read it (it arrives when those
// MMAs complete), a plain arrival otherwise.  Group A reads the stages of the first sweep
// for the R2 column norms and arrives then; in later sweeps the pass A issuer arrives for it.

template <int R, int KCAP, bool PASS_B>
__device__ void mma_pass(const Params& p, const Bars& b, uint8_t* smem, uint32_t tmem_base) {
  using C = Cfg<R, KCAP>;
  RingPos rs, d;
  const int T = local_tiles(p), nsw = sweep_count(T, p.interleave);
  const uint32_t zs0 = smem_u32(smem + p.off_zs), r20 = smem_u32(smem + p.off_r2);
  uint64_t* full = PASS_B ? b.b_full : b.a_full;
  uint64_t* empty = PASS_B ? b.b_empty : b.a_empty;
  constexpr int NBUF = PASS_B ? C::NB : C::NA;
  constexpr int COL0 = PASS_B ? C::NA * 128 : 0;
  // pass A reads z_hi only (K = r); pass B reads z_hi | z_lo (K = 2r) for exact logits
  constexpr int KSTEPS = PASS_B ? C::RK / 16 : R / 16;
  for (int q = 0; q < nsw; ++q) {
    const Sweep sw = sweep_jobs(q, T, p.interleave);
    const int j = PASS_B ? sw.tb : sw.ta;
    const uint32_t zs = j >= 0 ? zs0 + zs_buf(j, p.interleave) * C::ZS_BYTES : 0u;
    for (int t = 0; t < p.p_count; ++t) {
      int st;
      if (p.r2_resident) {
        st = t;
        if (q == 0 && !bounded_wait(&b.r2_full[t], 0, b.abort_flag, p.a.status)) goto done;
      } else {
        st = rs.i;
        if (!bounded_wait(&b.r2_full[rs.i], rs.phase, b.abort_flag, p.a.status)) goto done;
      }
      if (j >= 0) {
        // the tile's z buffer is written by group A's epilogue
        if (t == 0 && !bounded_wait(&b.zsm_full[zs_buf(j, p.interleave)], zs_use(j, p.interleave) & 1, b.abort_flag,
                                p.a.status))
          goto done;
        if (!bounded_wait(&empty[d.i], d.phase ^ 1u, b.abort_flag, p.a.status)) goto done;
        tc_fence_after();
        const uint32_t dt = tmem_base + COL0 + d.i * 128;
        const uint32_t r2 = r20 + st * C::R2_STAGE;
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
          const uint64_t zd = smem_desc(zs + kk * 256, 128, C::ZS_SBO, kSwizzleNone);
          const uint64_t rd = smem_desc(r2 + (kk % (R / 16)) * 2048, C::R2_BOX_BYTES, 1024, kSwizzle128B);
          mma_bf16(dt, zd, rd, C::IDESC_P, kk != 0);
        }
        mma_commit(&full[d.i]);
        d.next(NBUF);
      }
      if (!p.r2_resident) {
        if (j >= 0)
          mma_commit(&b.r2_empty[rs.i]);
        else
          mbar_arrive(&b.r2_empty[rs.i]);
        if (!PASS_B && q > 0) mbar_arrive_count(&b.r2_empty[rs.i], kWarpsA);  // for group A
        rs.next(p.r2_stages);
      }
    }
    // tile tb's z buffer: its pass B MMAs are one of the two releases (group B's finalize is
    // the other)
    if (PASS_B && j >= 0) mma_commit(&b.zsm_empty[zs_buf(j, p.interleave)]);
  }
done:
  mma_commit(&b.drain[PASS_B ? 2 : 1]);
  bounded_wait(&b.drain[PASS_B ? 2 : 1], 0, b.abort_flag, p.a.status);
}

// ---- group A: epilogue, pass A, select ------------------------------------------------------

template <int R, int KCAP>
__device__ void group_a(const Params& p, const Bars& b, uint8_t* smem, uint32_t tmem_base) {
  using C = Cfg<R, KCAP>;
  constexpr int KL = C::KA;
  const RouteArgs& a = p.a;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int aw = warp - kWarpA0;        // 0..7
  const int sp = warp & 3;              // TMEM lane group: lanes 32 sp .. 32 sp + 31
  const int hh = aw >> 2;               // which of the lane group's two warps
  const int gt = aw * 32 + lane;        // 0..255
  const int t = sp * 32 + lane;         // token of this thread
  const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
  const uint32_t low = p.low_mask;
  uint8_t* zs0 = smem + p.off_zs;
  const uint8_t* r2s = smem + p.off_r2;
  uint32_t* lists = reinterpret_cast<uint32_t*>(smem + p.off_lists);  // merge exchange
  float* znorm = reinterpret_cast<float*>(smem + p.off_znorm);  // [hi h0 | hi h1 | lo h0 | lo h1][token]
  float* cnorm = reinterpret_cast<float*>(smem + p.off_cnorm);  // [8] per warp, [8] = result
  uint32_t gph = 0;
  RingPos ad, rs;
  float colmax2 = 0.f;  // this warp's largest squared R2 column norm (first tile)
  const int T = local_tiles(p);
  uint32_t kl[KL];

  for (int j = 0; j < T; ++j) {
    const int64_t n0 = ((int64_t)blockIdx.x + (int64_t)j * gridDim.x) * kBT;
    const bool first = j == 0;
    // ---------------- epilogue: Z from TMEM -> (z_hi, z_lo) -> shared memory ----------------
    {
      const int buf = j & 1;
      if (!bounded_wait(&b.zacc_full[buf], (j >> 1) & 1, b.abort_flag, a.status)) return;
      tc_fence_after();
      constexpr int HALF = R / 2;
      uint32_t zr[HALF];
      const uint32_t taddr = tmem_base + lane_base + C::ZCOL0 + buf * C::ZCOLS + hh * HALF;
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
      // the previous tile of this z buffer: its pass B MMAs and its finalize are done
      const int zb = zs_buf(j, p.interleave), u = zs_use(j, p.interleave);
      if (u > 0 && !bounded_wait(&b.zsm_empty[zb], (u - 1) & 1, b.abort_flag, a.status)) return;
      uint8_t* zs = zs0 + zb * C::ZS_BYTES;
      float hi2 = 0.f, lo2 = 0.f;
#pragma unroll
      for (int q = 0; q < HALF / 8; ++q) {
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          float z0 = __uint_as_float(zr[q * 8 + 2 * jj]), z1 = __uint_as_float(zr[q * 8 + 2 * jj + 1]);
          __nv_bfloat16 h0 = __float2bfloat16_rn(z0), h1 = __float2bfloat16_rn(z1);
          __nv_bfloat16 l0 = __float2bfloat16_rn(z0 - __bfloat162float(h0));
          __nv_bfloat16 l1 = __float2bfloat16_rn(z1 - __bfloat162float(h1));
          const float fh0 = __bfloat162float(h0), fh1 = __bfloat162float(h1);
          const float fl0 = __bfloat162float(l0), fl1 = __bfloat162float(l1);
          hi2 = fmaf(fh0, fh0, fmaf(fh1, fh1, hi2));
          lo2 = fmaf(fl0, fl0, fmaf(fl1, fl1, lo2));
          hi[jj] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
          lo[jj] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
        }
        const int i0 = hh * HALF + q * 8;  // first z index of this 8-group
        *reinterpret_cast<uint4*>(zs + zs_offset<R, KCAP>(t, i0 >> 3)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(zs + zs_offset<R, KCAP>(t, (R + i0) >> 3)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
      znorm[hh * kBT + t] = hi2;
      znorm[(2 + hh) * kBT + t] = lo2;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&b.zsm_full[zb]);
    }

    // ---------------- pass A: chunk maxima of z_hi . R2 -> top KL chunk keys -------------
    // warp hh of a lane group owns columns 64 hh .. 64 hh + 63 (chunks 4 pt + 2 hh, + 1)
#pragma unroll
    for (int i = 0; i < KL; ++i) kl[i] = 0u;
    for (int pt = 0; pt < p.p_count; ++pt) {
      if (!bounded_wait(&b.a_full[ad.i], ad.phase, b.abort_flag, a.status)) return;
      tc_fence_after();
      const uint32_t col = tmem_base + lane_base + ad.i * 128 + hh * 64;
      const int c0 = pt * 4 + 2 * hh;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t v[32];
        tmem_ld_x32(col + 32 * half, v);
        tmem_wait_ld();
        reg_fence<32>(v);
        if (half == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&b.a_empty[ad.i]);
        }
        const int c = c0 + half;
        if (32 * c + 32 > a.M) {  // out-of-range experts at -infinity (Algorithm 1)
#pragma unroll
          for (int jj = 0; jj < 32; ++jj)
            if (32 * c + jj >= a.M) v[jj] = 0xff800000u;
        }
        key_insert<KL>(kl, (ord_key(max32(v)) & ~low) | (uint32_t)c);
      }
      ad.next(C::NA);
      if (first) {
        // squared column norms of R2 (experts 16 aw .. 16 aw + 15 of the stage)
        int st;
        if (p.r2_resident) {
          st = pt;
          if (!bounded_wait(&b.r2_full[pt], 0, b.abort_flag, a.status)) return;
        } else {
          st = rs.i;
          if (!bounded_wait(&b.r2_full[rs.i], rs.phase, b.abort_flag, a.status)) return;
        }
        const uint8_t* base = r2s + st * C::R2_STAGE;
        const int el = 16 * aw + (lane & 15);
        float acc = 0.f;
#pragma unroll 4
        for (int i = lane >> 4; i < R; i += 2) {
          const float w = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(base + r2_offset<R>(i, el)));
          acc = fmaf(w, w, acc);
        }
        acc += __shfl_xor_sync(0xffffffffu, acc, 16);
        colmax2 = fmaxf(colmax2, acc);
        if (!p.r2_resident) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&b.r2_empty[rs.i]);
          rs.next(p.r2_stages);
        }
      }
    }

    // ---------------- select: merge the lists, the candidate cut -------------------------
    const int pb = j & 1, pu = j >> 1;  // hand-off buffer and its use count
    // the hand-off buffer's previous tile (j - 2) is finalized by group B
    if (pu > 0 && !bounded_wait(&b.pairs_empty[pb], (pu - 1) & 1, b.abort_flag, a.status)) return;
    float* cut = reinterpret_cast<float*>(smem + p.off_cut) + pb * kBT;
    uint8_t* flag = smem + p.off_flag + pb * kBT;
    if (hh == 1) {
#pragma unroll
      for (int i = 0; i < KL; ++i) lists[i * kBT + t] = kl[i];
    }
    if (first) {
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) colmax2 = fmaxf(colmax2, __shfl_xor_sync(0xffffffffu, colmax2, d));
      if (lane == 0) cnorm[aw] = colmax2;
    }
    if (!group_enter(&b.gbar[0], gph, b.abort_flag, a.status)) return;
    // from here to the hand-off nothing waits on another role
    if (hh == 0) {
#pragma unroll
      for (int i = 0; i < KL; ++i) key_insert<KL>(kl, lists[i * kBT + t]);
    }
    if (first && gt == 0) {
      float m = 0.f;
      for (int w = 0; w < kWarpsA; ++w) m = fmaxf(m, cnorm[w]);
      cnorm[kWarpsA] = sqrtf(m) * (1.f + 0x1p-20f);  // max column norm of R2, rounded up
    }
    group_bar(kNamedBarA, kThreadsA);  // the merge has read the exchanged lists; cnorm is final
    if (hh == 0) {
      const bool active = n0 + t < a.N;
      // z_hi logits differ from the z_hi + z_lo values by at most eps = |z_lo| cmax
      // (Cauchy-Schwarz) plus a bound on fp32 accumulation differences.
      const float cmax = cnorm[kWarpsA];
      const float zh = sqrtf(znorm[t] + znorm[kBT + t]);
      const float zl = sqrtf(znorm[2 * kBT + t] + znorm[3 * kBT + t]);
      const float eps = (zl * cmax) * (1.f + 0x1p-8f) + (float)R * 0x1p-20f * zh * cmax + 1e-30f;
      uint32_t kth = 0;
#pragma unroll
      for (int i = 0; i < KL; ++i)
        if (i == a.k - 1) kth = kl[i];
      // The k chunks with the largest z_hi maxima (>= tlow) hold k experts whose exact logit is
      // >= tlow - eps, so the exact k-th logit is >= tlow - eps: every top-k expert reaches the
      // cut.  With fewer than k real chunks every in-range expert is a candidate (the
      // out-of-range ones are at -infinity, below the lowest finite cut).
      float ccut = -FLT_MAX;
      if ((kth & ~low) >= kRealKey) ccut = __fsub_rd(ord_inv(kth & ~low), eps);
      cut[t] = active ? ccut : __int_as_float(0x7fffffff);  // NaN: no expert reaches it
      flag[t] = (uint8_t)(active ? 0 : 2);
    }
    group_bar(kNamedBarA, kThreadsA);  // the cuts are written; the exchange area may be reused
    if (gt == 0) mbar_arrive(&b.pairs_full[pb]);
  }
}

// ---- group B: pass B, finalize ------------------------------------------------------------

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

// The cooperative fallback's first step.  The group's warps form kWarpsB / G teams of G
// warps (G = p.fb_groups, a power of two no larger than the number of 256-expert blocks):
// team js takes tokens js, js + kWarpsB / G, ... of the nb tokens in tok, and warp g of the
// team ranks the blocks g, g + G, ... of each, writing its partial top-k to part.
template <int R, int KCAP>
__device__ __forceinline__ void fallback_rank(const RouteArgs& a, const uint8_t* zs, const uint8_t* tok, int nb,
                                              uint2* part, int G, int bw, int lane) {
  const int teams = kWarpsB / G, js = bw / G, g = bw % G;
  for (int j = js; j < nb; j += teams) {
    const int tf = tok[j];
    float zr[(R + 31) / 32];
#pragma unroll
    for (int q = 0; q < (R + 31) / 32; ++q)
      zr[q] = (32 * q + lane < R) ? zs_value<R, KCAP>(zs, tf, 32 * q + lane) : 0.f;
    TopList<KCAP> list;
    list.init();
    for (int eb = 256 * g; eb < a.M; eb += 256 * G) fallback_block<R, KCAP>(a, zr, eb, lane, list);
    float v;
    int e;
    warp_merge_topk<KCAP>(list, a.k, lane, v, e);
    if (lane < KCAP) part[(j * G + g) * KCAP + lane] = make_uint2(__float_as_uint(v), (uint32_t)e);
  }
}

// The second step: merge the G partial lists of one token (part: list-major, KCAP entries
// each, the first k valid) and write the token's outputs.
template <int KCAP>
__device__ __forceinline__ void fallback_merge(const RouteArgs& a, const uint2* part, int G, int64_t n, int lane) {
  TopList<KCAP> list;
  list.init();
  for (int q = lane; q < G * KCAP; q += 32) {
    const uint2 c = part[q];
    if ((q % KCAP) < a.k) list.insert_any(__uint_as_float(c.x), (int)c.y);
  }
  float v;
  int e;
  warp_merge_topk<KCAP>(list, a.k, lane, v, e);
  warp_write_selection(a, n, lane, v, e);
}

// Branch-free insertion of the 64-bit key x into the descending list kl[0..L).
template <int L>
__device__ __forceinline__ void key_insert64(uint64_t* kl, uint64_t x) {
#pragma unroll
  for (int i = L - 1; i > 0; --i) kl[i] = max(kl[i], min(kl[i - 1], x));
  kl[0] = max(kl[0], x);
}

// Routing-order key of (logit, expert): larger logit first, then lower expert; 0 is below
// every real key.  -0 and +0 are equal in routing order: both take the key of +0.
__device__ __forceinline__ uint64_t route_key(uint32_t logit_bits, uint32_t expert) {
  return ((uint64_t)ord_key(__uint_as_float(logit_bits) + 0.f) << 32) | (uint64_t)(~expert);
}

// Stores an octet of logits (32 bytes at dst) and its 16-bit index (at idst) in shared memory
// when pred is nonzero; predicated stores, no branch.
__device__ __forceinline__ void st_octet_if(uint32_t pred, uint32_t dst, const uint32_t* w, uint32_t idst,
                                            uint32_t id) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %0, 0;\n\t"
      "@p st.shared.v4.b32 [%1], {%2, %3, %4, %5};\n\t"
      "@p st.shared.v4.b32 [%1+16], {%6, %7, %8, %9};\n\t"
      "@p st.shared.u16 [%10], %11;\n\t}" ::"r"(pred),
      "r"(dst), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]), "r"(idst),
      "h"((unsigned short)id)
      : "memory");
}

template <int R, int KCAP>
__device__ void group_b(const Params& p, const Bars& b, uint8_t* smem, uint32_t tmem_base) {
  using C = Cfg<R, KCAP>;
  const RouteArgs& a = p.a;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bw = warp - kWarpB0;        // 0 .. kWarpsB - 1
  const int sp = warp & 3;              // TMEM lane group: lanes 32 sp .. 32 sp + 31
  const int hh = bw >> 2;               // which 64-column half of every tile
  const int gt = bw * 32 + lane;        // 0 .. kThreadsB - 1
  const int t = sp * 32 + lane;         // token of this thread
  const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
  uint8_t* zs0 = smem + p.off_zs;
  uint4* slots = reinterpret_cast<uint4*>(smem + p.off_slots);       // [slot][token][2]: eight logits
  uint16_t* ids = reinterpret_cast<uint16_t*>(smem + p.off_ids);     // [slot][token]: octet index
  int* hcnt = reinterpret_cast<int*>(smem + p.off_hcnt);             // [half][token]: octets found
  int32_t* sidx = reinterpret_cast<int32_t*>(smem + p.off_stage);    // [token][k]
  float* sex = reinterpret_cast<float*>(sidx + kBT * KCAP);
  float* slog = sex + kBT * KCAP;
  int* fbcount = reinterpret_cast<int*>(smem + p.off_fb);
  uint8_t* fblist = smem + p.off_fb + 4;
  uint8_t* fbmark = smem + p.off_fb + 4 + kBT;  // 1: the token's outputs come from the fallback
  uint2* part = reinterpret_cast<uint2*>(smem + p.off_part);
  uint32_t gph = 0;
  RingPos bd;
  const int T = local_tiles(p);

  for (int j = 0; j < T; ++j) {
    const int64_t n0 = ((int64_t)blockIdx.x + (int64_t)j * gridDim.x) * kBT;
    const int pb = j & 1, pu = j >> 1;
    if (!bounded_wait(&b.pairs_full[pb], pu & 1, b.abort_flag, a.status)) return;
    const float ccut = reinterpret_cast<const float*>(smem + p.off_cut)[pb * kBT + t];
    const bool active = (smem[p.off_flag + pb * kBT + t] & 2) == 0;

    // ---------------- pass B: octets of the token that reach its cut (exact logits) ----------
    // Warp hh of a lane group reads columns 64 hh .. 64 hh + 63 of every tile, reduces each
    // octet to its maximum and stores the octets that reach its lane's cut.
    int cnt = 0;  // octets of the lane's token that reach the cut in this warp's columns
    // shared-memory addresses of the lane's next octet slot and index; each stored octet moves
    // them one slot row up (warp 0) or down (warp 1)
    uint32_t sdst = smem_u32(slots + 2 * ((hh ? C::OCT - 1 : 0) * kBT + t));
    uint32_t idst = smem_u32(ids + (hh ? C::OCT - 1 : 0) * kBT + t);
    const int sstep = hh ? -kBT * 32 : kBT * 32, istep = hh ? -kBT * 2 : kBT * 2;
    for (int pt = 0; pt < p.p_count; ++pt) {
      if (!bounded_wait(&b.b_full[bd.i], bd.phase, b.abort_flag, a.status)) return;
      tc_fence_after();
      const uint32_t col = tmem_base + lane_base + (C::NA + bd.i) * 128 + hh * 64;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t v[32];
        tmem_ld_x32(col + 32 * half, v);
        tmem_wait_ld();
        reg_fence<32>(v);
        if (half == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&b.b_empty[bd.i]);
        }
        const int e0 = kBE * pt + 64 * hh + 32 * half;
        if (e0 + 32 > a.M) {  // out-of-range experts at -infinity (Algorithm 1): below every cut
#pragma unroll
          for (int jj = 0; jj < 32; ++jj)
            if (e0 + jj >= a.M) v[jj] = 0xff800000u;
        }
#pragma unroll
        for (int o = 0; o < 4; ++o) {
          const uint32_t* w = v + 8 * o;
          const float om = max3f(max3f(__uint_as_float(w[0]), __uint_as_float(w[1]), __uint_as_float(w[2])),
                                 max3f(__uint_as_float(w[3]), __uint_as_float(w[4]), __uint_as_float(w[5])),
                                 fmaxf(__uint_as_float(w[6]), __uint_as_float(w[7])));
          // rare per lane (about k + 1 octets of a token in all): predicated stores, no branch
          const int hit = om >= ccut ? 1 : 0;
          st_octet_if(hit & (cnt < C::OCT ? 1 : 0), sdst, w, idst, (uint32_t)((e0 >> 3) + o));
          sdst += (uint32_t)(hit * sstep);
          idst += (uint32_t)(hit * istep);
          cnt += hit;
        }
      }
      bd.next(C::NB);
    }

    hcnt[hh * kBT + t] = cnt;

    // ---------------- finalize: order, softmax, store, count ---------------------------
    // Thread 0 of a token (warp hh = 0) walks the token's stored octets, keeps the best k of
    // the logits that reach the cut as sorted 64-bit routing keys, and writes the token's
    // outputs to the staging with the softmax gates.
    if (!group_enter(&b.gbar[1], gph, b.abort_flag, a.status)) return;
    // from here to the hand-off nothing waits on another role
    uint64_t kl[KCAP];
#pragma unroll
    for (int i = 0; i < KCAP; ++i) kl[i] = 0ull;
    bool fb = false;
    if (hh == 0 && active) {
      const int c0 = hcnt[t], c1 = hcnt[kBT + t];
      fb = c0 + c1 > C::OCT;  // the two ends of the slots met: an octet was not stored
      if (!fb) {
        for (int q = 0; q < c0 + c1; ++q) {
          const int sl = q < c0 ? q : C::OCT - 1 - (q - c0);
          const uint4* src = slots + 2 * (sl * kBT + t);
          const uint4 q0 = src[0], q1 = src[1];
          uint32_t m = (uint32_t)(__uint_as_float(q0.x) >= ccut) | ((uint32_t)(__uint_as_float(q0.y) >= ccut) << 1) |
                       ((uint32_t)(__uint_as_float(q0.z) >= ccut) << 2) | ((uint32_t)(__uint_as_float(q0.w) >= ccut) << 3) |
                       ((uint32_t)(__uint_as_float(q1.x) >= ccut) << 4) | ((uint32_t)(__uint_as_float(q1.y) >= ccut) << 5) |
                       ((uint32_t)(__uint_as_float(q1.z) >= ccut) << 6) | ((uint32_t)(__uint_as_float(q1.w) >= ccut) << 7);
          const uint32_t eb = 8u * ids[sl * kBT + t];
          const uint32_t* sv = reinterpret_cast<const uint32_t*>(src);
          while (m) {  // the logits of the octet that reach the cut: usually one
            const int jj = __ffs(m) - 1;
            m &= m - 1u;
            key_insert64<KCAP>(kl, route_key(sv[jj], eb + (uint32_t)jj));
          }
        }
        uint64_t kth = 0ull;
#pragma unroll
        for (int i = 0; i < KCAP; ++i)
          if (i == a.k - 1) kth = kl[i];
        fb = kth == 0ull;  // fewer than k candidates
      }
      fbmark[t] = fb ? 1 : 0;
      if (fb) fblist[atomicAdd(fbcount, 1)] = (uint8_t)t;
    }
    group_bar(kNamedBarB, kThreadsB);  // every octet slot is read: the staging may overwrite them
    if (hh == 0 && active && !fb) {
      const float vtop = ord_inv((uint32_t)(kl[0] >> 32));
      float ex[KCAP], sum = 0.f;
#pragma unroll
      for (int i = 0; i < KCAP; ++i) {
        ex[i] = i < a.k ? expf(ord_inv((uint32_t)(kl[i] >> 32)) - vtop) : 0.f;
        sum += ex[i];
      }
      const float inv = 1.f / sum;
#pragma unroll
      for (int i = 0; i < KCAP; ++i) {
        if (i < a.k) {
          const uint32_t e = ~(uint32_t)kl[i];
          sidx[t * a.k + i] = (int)e;
          sex[t * a.k + i] = ex[i] * inv;
          slog[t * a.k + i] = ord_inv((uint32_t)(kl[i] >> 32));
          if (e < (uint32_t)a.M) atomicAdd(a.out_count + e, 1);
        }
      }
    }
    group_bar(kNamedBarB, kThreadsB);
    // the tile's outputs are contiguous: copy the staging out with coalesced stores
    const int rows = a.N - n0 < kBT ? (int)(a.N - n0) : kBT;
    const size_t ob = (size_t)n0 * a.k;
    for (int x = gt; x < rows * a.k; x += kThreadsB) {
      if (fbmark[x / a.k]) continue;
      a.out_idx[ob + x] = sidx[x];
      a.out_gate[ob + x] = sex[x];
      if (a.out_logits) a.out_logits[ob + x] = slog[x];
    }
    // fallback tokens, kFbBatch at a time: teams of p.fb_groups warps rank the batch's tokens
    // over their 256-expert blocks, then warp jj merges the partial lists of the batch's token
    // jj and writes it.  The partial lists lie past the staging, in the octet slots.
    const uint8_t* zs = zs0 + zs_buf(j, p.interleave) * C::ZS_BYTES;
    const int nfb = *fbcount;
    for (int fb0 = 0; fb0 < nfb; fb0 += kFbBatch) {
      const int nbt = nfb - fb0 < kFbBatch ? nfb - fb0 : kFbBatch;
      fallback_rank<R, KCAP>(a, zs, fblist + fb0, nbt, part, p.fb_groups, bw, lane);
      group_bar(kNamedBarB, kThreadsB);
      if (bw < nbt)
        fallback_merge<KCAP>(a, part + bw * p.fb_groups * KCAP, p.fb_groups, n0 + fblist[fb0 + bw], lane);
      group_bar(kNamedBarB, kThreadsB);
    }
    // every warp has read fbcount, the staging, the flags and the fallback lists: the next
    // tile's pass B may write the octet slots again
    group_bar(kNamedBarB, kThreadsB);
    if (gt == 0) {
      *fbcount = 0;
      mbar_arrive(&b.pairs_empty[pb]);
      mbar_arrive(&b.zsm_empty[zs_buf(j, p.interleave)]);  // the fallback is done with the z buffer
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
      // both logit issuers and group A's eight warps (the pass A issuer stands in for them
      // after the first sweep)
      mbar_init(&b.r2_empty[i], 2 + kWarpsA);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&b.zacc_full[i], 1);
      mbar_init(&b.zacc_empty[i], kWarpsA);
      mbar_init(&b.zsm_full[i], kWarpsA);
      mbar_init(&b.zsm_empty[i], 2);  // pass B MMAs done, finalize done
      mbar_init(&b.a_full[i], 1);
      mbar_init(&b.a_empty[i], kWarpsA);
      mbar_init(&b.b_full[i], 1);
      mbar_init(&b.b_empty[i], kWarpsB);
      mbar_init(&b.pairs_full[i], 1);
      mbar_init(&b.pairs_empty[i], 1);
      mbar_init(&b.gbar[i], i == 0 ? kWarpsA : kWarpsB);
    }
    for (int i = 0; i < 3; ++i) mbar_init(&b.drain[i], 1);
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
  if (threadIdx.x == kWarpB0 * 32) *reinterpret_cast<int*>(smem + p.off_fb) = 0;  // fallback count
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *b.tmem_slot;

  if (warp == 0) {
    if (lane == 0) producer<R, KCAP>(p, b, smem, &tmX, &tmR1, &tmR2);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) mma_z<R, KCAP>(p, b, smem, tmem_base);
    __syncwarp();
  } else if (warp == 2) {
    if (lane == 0) mma_pass<R, KCAP, false>(p, b, smem, tmem_base);
    __syncwarp();
  } else if (warp == 3) {
    if (lane == 0) mma_pass<R, KCAP, true>(p, b, smem, tmem_base);
    __syncwarp();
  } else if (warp < kWarpB0) {
    group_a<R, KCAP>(p, b, smem, tmem_base);
  } else {
    group_b<R, KCAP>(p, b, smem, tmem_base);
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

// Shared-memory layout for xs X stages, r2n R2 stages (all p_count when resident) and nz z
// buffers; returns the total bytes.
template <int R, int KCAP>
uint32_t layout(Params& p, int xs, int r2n, int nz) {
  using C = Cfg<R, KCAP>;
  uint32_t off = 0;
  p.off_x = off;
  off += xs * C::X_STAGE;
  p.off_r1 = off = align_up(off, 1024);
  off += xs * C::R1_STAGE;
  p.off_r2 = off = align_up(off, 1024);
  off += r2n * C::R2_STAGE;
  p.off_zs = off = align_up(off, 1024);
  off += nz * C::ZS_BYTES;
  // group A: list exchange
  p.off_lists = off = align_up(off, 16);
  off += C::KA * kBT * 4;
  p.off_znorm = off;  // per token: |z_hi|^2 and |z_lo|^2 partial sums of both halves
  off += 4 * kBT * 4;
  p.off_cnorm = off;  // per warp: max squared column norm of R2; [8] = the result
  off += (kWarpsA + 1) * 4;
  // group A -> group B, two buffers each: cut (fp32) and flags of every token
  p.off_cut = off = align_up(off, 16);
  off += 2 * kBT * 4;
  p.off_flag = off;
  off += 2 * kBT;
  // group B: octet slots, their indices and counts, the list exchange, fallback
  p.off_slots = off = align_up(off, 16);
  off += C::OCT * kBT * 32;
  p.off_ids = off;
  off += C::OCT * kBT * 2;
  p.off_hcnt = off = align_up(off, 16);
  off += 2 * kBT * 4;
  p.off_fb = off;  // fallback count, the tile's fallback tokens, per-token mark
  off += 4 + 2 * kBT;
  // the output staging and, after it, the fallback's partial lists reuse the octet slots: the
  // finalize has read them by then
  p.off_stage = p.off_slots;
  p.off_part = p.off_slots + C::STAGE_BYTES;
  p.off_bar = off = align_up(off, 8);
  off += kBarBytes;
  return off + 1024;  // alignment slack of the dynamic base
}

// Shared-memory plan; returns the total bytes (0 when nothing fits).  Preference order:
// R2 resident (no streaming at all); then two z buffers (one R2 sweep per tile) with at least
// 3 R2 stages; then one z buffer (two sweeps per tile) with at least 3 R2 stages; then 2 R2
// stages.  Within each, more X stages first, then more R2 stages.
template <int R, int KCAP>
uint32_t plan(Params& p) {
  struct Try {
    int nz, xs_min, r2_min;
  };
  if (p.p_count <= 64) {
    for (int nz = 2; nz >= 1; --nz)
      for (int xs = 4; xs >= 3; --xs) {
        const uint32_t total = layout<R, KCAP>(p, xs, p.p_count, nz);
        if (total <= kSmemLimit) {
          p.x_stages = xs;
          p.r2_stages = p.p_count;
          p.r2_resident = 1;
          p.interleave = nz == 2;
          return total;
        }
      }
  }
  const Try tries[] = {{2, 2, 3}, {1, 2, 3}, {1, 2, 2}, {2, 2, 2}};
  for (const Try& tr : tries) {
    for (int xs = 4; xs >= tr.xs_min; --xs) {
      for (int r2n = 8; r2n >= tr.r2_min; --r2n) {
        const uint32_t total = layout<R, KCAP>(p, xs, r2n, tr.nz);
        if (total <= kSmemLimit) {
          p.x_stages = xs;
          p.r2_stages = r2n;
          p.r2_resident = 0;
          p.interleave = tr.nz == 2;
          return total;
        }
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
  p.fb_groups = 1;
  while (p.fb_groups < kWarpsB && 256 * p.fb_groups < a.M) p.fb_groups *= 2;
  int bits = 1;  // chunk ids run up to 4 p_count - 1 (the padded last tile)
  while ((1 << bits) < 4 * p.p_count) ++bits;
  p.low_mask = (1u << bits) - 1u;
  smem = plan<R, KCAP>(p);
  return smem != 0;
}

// Raises the kernel's dynamic shared-memory limit once per device.
template <int R, int KCAP>
cudaError_t configure_once(int dev) {
  static std::atomic<int> done[64] = {};
  if (dev >= 0 && dev < 64 && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(fused_route_kernel<R, KCAP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemLimit);
  if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev].store(1, std::memory_order_release);
  return e;
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
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = configure_once<R, KCAP>(dev);
  if (e != cudaSuccess) return e;
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

bool fused_tc_fits(const RouteArgs& a) {
  // up to 65536 experts = 2048 chunks: the chunk id takes at most 11 low bits of a pass-A key
  if (a.M > 65536 || a.k > 16 || a.N < 1 || a.N > 0x7fffffffLL - tc::kBT) return false;
  switch (a.r) {
    case 16: return tc::supports_r<16>(a);
    case 32: return tc::supports_r<32>(a);
    case 64: return tc::supports_r<64>(a);
    case 128: return tc::supports_r<128>(a);
    default: return false;
  }
}

bool fused_tc_supports(const RouteArgs& a) { return fused_tc_fits(a) && tc::encode_fn() != nullptr; }

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

// Tensor-core kernels that compute every exact logit of a tile, with the fused kernel's tcgen05
// products ("MoRE: Scaling mixture of experts with hardware-aware low-rank routing"):
//   - the materialise-then-top-k comparison path, the unfused low-rank router of App. H.6
//     (Fig. 24): the logits are written to HBM and ranked by a second kernel;
//   - the training statistics of App. F, Algorithm 2 and eqs. (6)-(8): two sweeps per tile,
//     the first keeping each token's running maximum m and rescaled sum Z of exp(l - m), the
//     second adding exp(l - m) / Z into the per-expert column sums psum.
// The materialise path:
//   kernel 1 (persistent, one CTA per SM): z = X . R1 into TMEM, narrowed to the bf16 pair
//            z_hi | z_lo in shared memory; then for every 128-expert tile of R2 the exact
//            logits l = (z_hi + z_lo) . R2 (one K = 2r product) into TMEM, read back by
//            eight warps and written to the fp32 [N][M] score tensor with TMA tile stores;
//   kernel 2: one warp per row reads the scores back for the top-k (a running list filtered
//            by its k-th value) and the softmax.
// The products and their precision are those of the fused kernel, so both return the same
// selections up to the order of fp32 accumulation; what differs is the round trip of the
// N x M scores through HBM, which the fused kernel avoids.
#include <cudaTypedefs.h>

#include <atomic>

#include "more_internal.cuh"
#include "mbar_wait.cuh"
#include "sm100_ptx.cuh"

namespace more {
namespace mat {

using namespace sm100;

constexpr int kBT = 128;       // tokens per tile
constexpr int kBE = 128;       // experts per score tile
constexpr int kRoleWarps = 4;  // producer, Z issuer, score issuer, (idle: keeps warp % 4 = lane group)
constexpr int kEpiWarps = 8;   // two warps per TMEM lane group, 64 score columns each
constexpr int kThreads = (kRoleWarps + kEpiWarps) * 32;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kStgBytes = 32 * 32 * 4;  // one staged store box: 32 tokens x 32 experts fp32
constexpr uint32_t kSmemLimit = 227 * 1024;
constexpr int kMaxR2Stages = 64;

struct Params {
  RouteArgs a;
  int num_tiles, kb_count, p_count;
  int sweeps;  // logit sweeps per tile: 1 (materialise) or 2 (training statistics)
  int x_stages, r2_stages, r2_resident, nz, nstg;
  uint32_t off_x, off_r1, off_r2, off_zs, off_stg, off_stat, off_bar;
  float *out_m, *out_Z, *out_psum;  // training statistics
};

template <int R>
struct Cfg {
  static constexpr int BK = R >= 128 ? 32 : 64;        // hidden elements per X stage
  static constexpr uint32_t X_STAGE = kBT * BK * 2;
  static constexpr uint32_t X_LAYOUT = BK == 64 ? kSwizzle128B : kSwizzle64B;
  static constexpr uint32_t X_SBO = 8 * BK * 2;
  static constexpr int R1_BOX = R < 64 ? R : 64;
  static constexpr int R1_BOXES = R / R1_BOX;
  static constexpr uint32_t R1_BOX_BYTES = BK * R1_BOX * 2;
  static constexpr uint32_t R1_STAGE = R1_BOX_BYTES * R1_BOXES;
  static constexpr uint32_t R1_ROW = R1_BOX * 2;
  static constexpr uint32_t R1_LAYOUT = R1_ROW == 32 ? kSwizzle32B : (R1_ROW == 64 ? kSwizzle64B : kSwizzle128B);
  static constexpr uint32_t R2_BOX_BYTES = 64 * R * 2;  // 64 experts x R rows, MN-major, 128B swizzle
  static constexpr uint32_t R2_STAGE = 2 * R2_BOX_BYTES;
  static constexpr int RK = 2 * R;                       // z_hi | z_lo
  static constexpr uint32_t ZS_BYTES = kBT * RK * 2;     // K-major core matrices, no swizzle
  static constexpr uint32_t ZS_SBO = (RK / 8) * 128;
  static constexpr int ZCOLS = R < 32 ? 32 : R;
  static constexpr int NS = (512 - 2 * ZCOLS) / 128 < 3 ? (512 - 2 * ZCOLS) / 128 : 3;  // score buffers
  static constexpr int ZCOL0 = NS * 128;
  static constexpr uint32_t IDESC_Z = idesc_bf16_f32(128, R, 0, 1);   // A = X (K-major), B = R1 (MN-major)
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, 0, 1); // A = z pair, B = R2 tile
  static_assert(NS >= 2, "two score buffers at least");
};

struct Bars {
  uint64_t* x_full;      // [4]
  uint64_t* x_empty;     // [4]
  uint64_t* r2_full;     // [64]
  uint64_t* r2_empty;    // [64]
  uint64_t* zacc_full;   // [2]
  uint64_t* zacc_empty;  // [2]
  uint64_t* zsm_full;    // [2]
  uint64_t* zsm_empty;   // [2]
  uint64_t* s_full;      // [3]
  uint64_t* s_empty;     // [3]
  uint64_t* drain;       // [2]
  uint64_t* st_half;     // [1] training statistics: second-half (m, s) written
  uint64_t* st_tok;      // [1] training statistics: token (m, 1 / Z) written
  uint32_t* tmem_slot;
  int* abort_flag;
};
constexpr uint32_t kBarSlots = 8 + 2 * kMaxR2Stages + 8 + 6 + 2 + 2;
constexpr uint32_t kBarBytes = kBarSlots * 8 + 16;

__device__ __forceinline__ Bars bars_at(uint8_t* smem, const Params& p) {
  uint64_t* b = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  Bars r;
  r.x_full = b;
  r.x_empty = b + 4;
  r.r2_full = b + 8;
  r.r2_empty = r.r2_full + kMaxR2Stages;
  r.zacc_full = r.r2_empty + kMaxR2Stages;
  r.zacc_empty = r.zacc_full + 2;
  r.zsm_full = r.zacc_empty + 2;
  r.zsm_empty = r.zsm_full + 2;
  r.s_full = r.zsm_empty + 2;
  r.s_empty = r.s_full + 3;
  r.drain = r.s_empty + 3;
  r.st_half = r.drain + 2;
  r.st_tok = r.st_half + 1;
  r.tmem_slot = reinterpret_cast<uint32_t*>(r.st_tok + 1);
  r.abort_flag = reinterpret_cast<int*>(r.tmem_slot + 1);
  return r;
}

__device__ __forceinline__ int local_tiles(const Params& p) {
  return (int)blockIdx.x < p.num_tiles ? (p.num_tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
}

// Byte offset of the 16-byte core-matrix row (token t, K chunk c) in a z pair buffer.
template <int R>
__device__ __forceinline__ uint32_t zs_offset(int t, int c) {
  return (uint32_t)(((t >> 3) * (Cfg<R>::RK / 8) + c) * 128 + (t & 7) * 16);
}

// ---- role: TMA producer ------------------------------------------------------------------
// X and R1 stages in tile order; R2 tiles once per local tile (or all of R2 once, resident).
template <int R>
__device__ void producer(const Params& p, const Bars& b, uint8_t* smem, const CUtensorMap* tmX,
                         const CUtensorMap* tmR1, const CUtensorMap* tmR2) {
  using C = Cfg<R>;
  auto load_r2 = [&](int slot, int t) {
    uint8_t* dst = smem + p.off_r2 + slot * C::R2_STAGE;
    mbar_arrive_expect_tx(&b.r2_full[slot], C::R2_STAGE);
    tma_load_2d(dst, tmR2, &b.r2_full[slot], t * kBE, 0);
    tma_load_2d(dst + C::R2_BOX_BYTES, tmR2, &b.r2_full[slot], t * kBE + 64, 0);
  };
  if (p.r2_resident)
    for (int t = 0; t < p.p_count; ++t) load_r2(t, t);
  RingPos sx, sr;
  int xt = 0, kb = 0;
  const int T = local_tiles(p);
  int q = 0, rt = 0;
  const int nsw = p.r2_resident ? 0 : T * p.sweeps;
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

// ---- role: MMA issuer of Z = X R1 ----------------------------------------------------------
template <int R>
__device__ void mma_z(const Params& p, const Bars& b, uint8_t* smem, uint32_t tmem_base) {
  using C = Cfg<R>;
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
        const uint64_t ad = smem_desc(x0 + s.i * C::X_STAGE + kk * 32, 16, C::X_SBO, C::X_LAYOUT);
        const uint64_t bd = smem_desc(r10 + s.i * C::R1_STAGE + kk * 16 * C::R1_ROW, C::R1_BOX_BYTES,
                                      8 * C::R1_ROW, C::R1_LAYOUT);
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

// ---- role: MMA issuer of the score tiles ---------------------------------------------------
// Per local tile and 128-expert tile: l = z_hi . R2 + z_lo . R2 as one K = 2r product.
template <int R>
__device__ void mma_scores(const Params& p, const Bars& b, uint8_t* smem, uint32_t tmem_base) {
  using C = Cfg<R>;
  RingPos rs, d;
  const int T = local_tiles(p);
  const uint32_t zs0 = smem_u32(smem + p.off_zs), r20 = smem_u32(smem + p.off_r2);
  for (int j = 0; j < T; ++j) {
    const int zb = p.nz == 2 ? (j & 1) : 0, use = p.nz == 2 ? (j >> 1) : j;
    if (!bounded_wait(&b.zsm_full[zb], use & 1, b.abort_flag, p.a.status)) goto done;
    for (int sw = 0; sw < p.sweeps; ++sw) {
      const uint32_t zs = zs0 + zb * C::ZS_BYTES;
      for (int t = 0; t < p.p_count; ++t) {
        int st;
        if (p.r2_resident) {
          st = t;
          if (j == 0 && sw == 0 && !bounded_wait(&b.r2_full[t], 0, b.abort_flag, p.a.status)) goto done;
        } else {
          st = rs.i;
          if (!bounded_wait(&b.r2_full[rs.i], rs.phase, b.abort_flag, p.a.status)) goto done;
        }
        if (!bounded_wait(&b.s_empty[d.i], d.phase ^ 1u, b.abort_flag, p.a.status)) goto done;
        tc_fence_after();
        const uint32_t dt = tmem_base + d.i * 128;
        const uint32_t r2 = r20 + st * C::R2_STAGE;
#pragma unroll
        for (int kk = 0; kk < C::RK / 16; ++kk) {
          const uint64_t zd = smem_desc(zs + kk * 256, 128, C::ZS_SBO, kSwizzleNone);
          const uint64_t rd = smem_desc(r2 + (kk % (R / 16)) * 2048, C::R2_BOX_BYTES, 1024, kSwizzle128B);
          mma_bf16(dt, zd, rd, C::IDESC_S, kk != 0);
        }
        mma_commit(&b.s_full[d.i]);
        d.next(C::NS);
        if (!p.r2_resident) {
          mma_commit(&b.r2_empty[rs.i]);
          rs.next(p.r2_stages);
        }
      }
    }
    mma_commit(&b.zsm_empty[zb]);
  }
done:
  mma_commit(&b.drain[1]);
  bounded_wait(&b.drain[1], 0, b.abort_flag, p.a.status);
}

// z of local tile j from TMEM -> (z_hi, z_lo) bf16 -> the tile's z buffer in shared memory,
// R / 2 columns per epilogue warp.  False when a wait gave up.
template <int R>
__device__ bool z_to_smem(const Params& p, const Bars& b, uint8_t* smem, uint32_t tmem_base, int j) {
  using C = Cfg<R>;
  const RouteArgs& a = p.a;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hh = (warp - kRoleWarps) >> 2, sp = warp & 3, t = sp * 32 + lane;
  const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
  uint8_t* zs0 = smem + p.off_zs;
  const int buf = j & 1;
  if (!bounded_wait(&b.zacc_full[buf], (j >> 1) & 1, b.abort_flag, a.status)) return false;
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
  const int zb = p.nz == 2 ? (j & 1) : 0, use = p.nz == 2 ? (j >> 1) : j;
  if (use > 0 && !bounded_wait(&b.zsm_empty[zb], (use - 1) & 1, b.abort_flag, a.status)) return false;
  uint8_t* zs = zs0 + zb * C::ZS_BYTES;
#pragma unroll
  for (int q = 0; q < HALF / 8; ++q) {
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const float z0 = __uint_as_float(zr[q * 8 + 2 * jj]), z1 = __uint_as_float(zr[q * 8 + 2 * jj + 1]);
      const __nv_bfloat16 h0 = __float2bfloat16_rn(z0), h1 = __float2bfloat16_rn(z1);
      const __nv_bfloat16 l0 = __float2bfloat16_rn(z0 - __bfloat162float(h0));
      const __nv_bfloat16 l1 = __float2bfloat16_rn(z1 - __bfloat162float(h1));
      hi[jj] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
      lo[jj] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
    }
    const int i0 = hh * HALF + q * 8;
    *reinterpret_cast<uint4*>(zs + zs_offset<R>(t, i0 >> 3)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(zs + zs_offset<R>(t, (R + i0) >> 3)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) mbar_arrive(&b.zsm_full[zb]);
  return true;
}

// ---- epilogue warps: z pair to shared memory, score tiles to HBM ---------------------------
template <int R>
__device__ void epilogue(const Params& p, const Bars& b, uint8_t* smem, uint32_t tmem_base, const CUtensorMap* tmS) {
  using C = Cfg<R>;
  const RouteArgs& a = p.a;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ew = warp - kRoleWarps;  // 0..7
  const int sp = warp & 3;           // TMEM lane group
  const int hh = ew >> 2;            // which of the lane group's two warps
  const int t = sp * 32 + lane;
  const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
  uint8_t* stg0 = smem + p.off_stg + (uint32_t)ew * p.nstg * kStgBytes;
  int sc = 0;  // score boxes this warp has staged
  RingPos d;
  const int T = local_tiles(p);
  for (int j = 0; j < T; ++j) {
    const int64_t n0 = ((int64_t)blockIdx.x + (int64_t)j * gridDim.x) * kBT;
    if (!z_to_smem<R>(p, b, smem, tmem_base, j)) goto done;
    // score tiles: this warp's 32 tokens x 64 experts of each tile, as two 32 x 32 boxes
    const int row0 = (int)(n0 + sp * 32);
    const bool rows_in = n0 + sp * 32 < a.N;
    for (int pt = 0; pt < p.p_count; ++pt) {
      if (!bounded_wait(&b.s_full[d.i], d.phase, b.abort_flag, a.status)) goto done;
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
      d.next(C::NS);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int e0 = pt * kBE + hh * 64 + 32 * c;
        if (!rows_in || e0 >= a.M) continue;  // the box lies wholly outside the score tensor
        uint8_t* stg = stg0 + (uint32_t)(sc % p.nstg) * kStgBytes;
        // the store that last read this buffer is done reading it
        if (lane == 0) {
          if (p.nstg == 2)
            bulk_wait_group_read<1>();
          else
            bulk_wait_group_read<0>();
        }
        __syncwarp();
        // row `lane` of the box, 128B-swizzled: 16-byte chunk q sits at chunk q ^ (row & 7)
#pragma unroll
        for (int q = 0; q < 8; ++q)
          *reinterpret_cast<uint4*>(stg + lane * 128 + ((q ^ (lane & 7)) << 4)) =
              make_uint4(v[32 * c + 4 * q], v[32 * c + 4 * q + 1], v[32 * c + 4 * q + 2], v[32 * c + 4 * q + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(tmS, stg, e0, row0);
          bulk_commit_group();
        }
        ++sc;
      }
    }
  }
done:
  if (lane == 0) bulk_wait_group<0>();
  __syncwarp();
}

// ---- epilogue warps: training statistics (App. F, Algorithm 2, eqs. (6)-(8)) ----------------
// Thread (token t, half hh) covers experts hh * 64 .. hh * 64 + 63 of every tile.  Sweep 1 keeps
// its running maximum m and the sum s of exp(l - m), rescaled whenever m grows (eq. (8)).  The
// two halves of each token are then merged through shared memory into m_n and Z_n, which the
// hh = 0 thread writes out.  Sweep 2 adds exp(l - m_n) / Z_n of the warp's 32 tokens into each
// expert's column sum: a shuffle reduce-scatter leaves column q's sum on lane q, and one global
// atomic per column and warp adds it to psum.
template <int R>
__device__ void stats_epilogue(const Params& p, const Bars& b, uint8_t* smem, uint32_t tmem_base) {
  const RouteArgs& a = p.a;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ew = warp - kRoleWarps;
  const int sp = warp & 3, hh = ew >> 2, t = sp * 32 + lane;
  const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
  float2* stat = reinterpret_cast<float2*>(smem + p.off_stat);  // [kBT] second-half (m, s); [kBT] token (m, 1/Z)
  RingPos d;
  const int T = local_tiles(p);
  for (int j = 0; j < T; ++j) {
    const int64_t n0 = ((int64_t)blockIdx.x + (int64_t)j * gridDim.x) * kBT;
    if (!z_to_smem<R>(p, b, smem, tmem_base, j)) return;
    const bool tok_in = n0 + t < a.N;
    float m = -INFINITY, ssum = 0.f;
    for (int pt = 0; pt < p.p_count; ++pt) {  // sweep 1
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
      d.next(Cfg<R>::NS);
      const int e0 = pt * kBE + hh * 64;
      float tmax = -INFINITY;
#pragma unroll
      for (int q = 0; q < 64; ++q)
        if (e0 + q < a.M) tmax = fmaxf(tmax, __uint_as_float(v[q]));
      if (tmax > m) {
        ssum = m == -INFINITY ? 0.f : ssum * __expf(m - tmax);
        m = tmax;
      }
#pragma unroll
      for (int q = 0; q < 64; ++q)
        if (e0 + q < a.M) ssum += __expf(__uint_as_float(v[q]) - m);
    }
    // token t's halves: hh = 1 hands (m, s) over, hh = 0 merges and hands back (m_n, 1 / Z_n)
    float mn, invZ;
    if (hh == 1) {
      stat[t] = make_float2(m, ssum);
      __syncwarp();
      if (lane == 0) mbar_arrive(b.st_half);
      if (!bounded_wait(b.st_tok, j & 1, b.abort_flag, a.status)) return;
      const float2 tk = stat[kBT + t];
      mn = tk.x;
      invZ = tk.y;
    } else {
      if (!bounded_wait(b.st_half, j & 1, b.abort_flag, a.status)) return;
      const float2 o = stat[t];
      mn = fmaxf(m, o.x);
      const float Z = (m == -INFINITY ? 0.f : ssum * __expf(m - mn)) + (o.x == -INFINITY ? 0.f : o.y * __expf(o.x - mn));
      invZ = 1.f / Z;
      if (tok_in) {
        p.out_m[n0 + t] = mn;
        p.out_Z[n0 + t] = Z;
      }
      stat[kBT + t] = make_float2(mn, invZ);
      __syncwarp();
      if (lane == 0) mbar_arrive(b.st_tok);
    }
    for (int pt = 0; pt < p.p_count; ++pt) {  // sweep 2
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
      d.next(Cfg<R>::NS);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int e0 = pt * kBE + hh * 64 + 32 * c;
        if (e0 >= a.M) break;  // warp-uniform: no column of this group is an expert
        float x[32];
#pragma unroll
        for (int q = 0; q < 32; ++q)
          x[q] = (tok_in && e0 + q < a.M) ? __expf(__uint_as_float(v[32 * c + q]) - mn) * invZ : 0.f;
        // reduce-scatter over the warp: after the step with distance dd a lane keeps the half
        // of its columns selected by its own bit dd; lane q ends with column q's sum
#pragma unroll
        for (int dd = 16, w = 16; dd >= 1; dd >>= 1, w >>= 1) {
          const bool up = lane & dd;
#pragma unroll
          for (int q = 0; q < w; ++q) {
            const float send = up ? x[q] : x[q + w];
            x[q] = (up ? x[q + w] : x[q]) + __shfl_xor_sync(0xffffffffu, send, dd);
          }
        }
        if (e0 + lane < a.M) atomicAdd(p.out_psum + e0 + lane, x[0]);
      }
    }
  }
}

template <int R, bool STATS>
__global__ void __launch_bounds__(kThreads, 1)
    tc_logits_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmR1,
                     const __grid_constant__ CUtensorMap tmR2, const __grid_constant__ CUtensorMap tmS,
                     const Params p) {
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
      mbar_init(&b.r2_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&b.zacc_full[i], 1);
      mbar_init(&b.zacc_empty[i], kEpiWarps);
      mbar_init(&b.zsm_full[i], kEpiWarps);
      mbar_init(&b.zsm_empty[i], 1);
      mbar_init(&b.drain[i], 1);
    }
    for (int i = 0; i < 3; ++i) {
      mbar_init(&b.s_full[i], 1);
      mbar_init(&b.s_empty[i], kEpiWarps);
    }
    mbar_init(b.st_half, 4);  // the four hh = 1 warps
    mbar_init(b.st_tok, 4);   // the four hh = 0 warps
    *b.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmX);
    prefetch_tensormap(&tmR1);
    prefetch_tensormap(&tmR2);
    if (!STATS) prefetch_tensormap(&tmS);
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
    if (lane == 0) producer<R>(p, b, smem, &tmX, &tmR1, &tmR2);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) mma_z<R>(p, b, smem, tmem_base);
    __syncwarp();
  } else if (warp == 2) {
    if (lane == 0) mma_scores<R>(p, b, smem, tmem_base);
    __syncwarp();
  } else if (warp >= kRoleWarps) {
    if constexpr (STATS)
      stats_epilogue<R>(p, b, smem, tmem_base);
    else
      epilogue<R>(p, b, smem, tmem_base, &tmS);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ---- host side -----------------------------------------------------------------------------

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

bool make_map(CUtensorMap* m, CUtensorMapDataType type, uint32_t elem_bytes, const void* base, uint64_t inner,
              uint64_t outer, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * elem_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, type, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

uint32_t align_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

template <int R>
uint32_t layout(Params& p, int xs, int r2n, int nz, int nstg) {
  using C = Cfg<R>;
  uint32_t off = 0;
  p.off_x = off;
  off += xs * C::X_STAGE;
  p.off_r1 = off = align_up(off, 1024);
  off += xs * C::R1_STAGE;
  p.off_r2 = off = align_up(off, 1024);
  off += r2n * C::R2_STAGE;
  p.off_zs = off = align_up(off, 1024);
  off += nz * C::ZS_BYTES;
  p.off_stg = off = align_up(off, 1024);
  off += kEpiWarps * nstg * kStgBytes;
  p.off_stat = off = align_up(off, 16);  // training statistics: 2 x kBT (m, s) pairs
  off += p.sweeps == 2 ? 2 * kBT * 8 : 0;
  p.off_bar = off = align_up(off, 8);
  off += kBarBytes;
  return off + 1024;  // alignment slack of the dynamic base
}

// Shared-memory plan: R2 resident when it fits, else streamed; two z buffers and two
// staging boxes per warp first (none for the statistics, which store nothing per tile), then
// fewer; more X stages first.  0 when nothing fits.
template <int R>
uint32_t plan(Params& p) {
  const int nstg_max = p.sweeps == 2 ? 0 : 2, nstg_min = p.sweeps == 2 ? 0 : 1;
  auto take = [&](int xs, int r2n, int resident, int nz, int nstg) {
    const uint32_t total = layout<R>(p, xs, r2n, nz, nstg);
    if (total > kSmemLimit) return 0u;
    p.x_stages = xs;
    p.r2_stages = r2n;
    p.r2_resident = resident;
    p.nz = nz;
    p.nstg = nstg;
    return total;
  };
  if (p.p_count <= kMaxR2Stages)
    for (int xs = 4; xs >= 3; --xs)
      if (uint32_t s = take(xs, p.p_count, 1, 2, nstg_max)) return s;
  for (int nz = 2; nz >= 1; --nz)
    for (int nstg = nstg_max; nstg >= nstg_min; --nstg)
      for (int xs = 4; xs >= 2; --xs)
        for (int r2n = 4; r2n >= 2; --r2n)
          if (uint32_t s = take(xs, r2n, 0, nz, nstg)) return s;
  return 0;
}

template <int R>
bool fill_params(const RouteArgs& a, Params& p, uint32_t& smem, int sweeps) {
  p.a = a;
  p.sweeps = sweeps;
  p.out_m = p.out_Z = p.out_psum = nullptr;
  p.num_tiles = (int)((a.N + kBT - 1) / kBT);
  p.kb_count = (a.h + Cfg<R>::BK - 1) / Cfg<R>::BK;
  p.p_count = (a.M + kBE - 1) / kBE;
  smem = plan<R>(p);
  return smem != 0;
}

template <int R, bool STATS>
cudaError_t configure_once(int dev) {
  static std::atomic<int> done[64] = {};
  if (dev >= 0 && dev < 64 && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(tc_logits_kernel<R, STATS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemLimit);
  if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev].store(1, std::memory_order_release);
  return e;
}

// Materialised scores (stats == nullptr) or the training statistics (stats = {m, Z, psum}).
template <int R>
cudaError_t launch(const RouteArgs& a, float* scores, float* const* stats) {
  using C = Cfg<R>;
  Params p;
  uint32_t smem = 0;
  if (!fill_params<R>(a, p, smem, stats ? 2 : 1)) return cudaErrorInvalidConfiguration;
  if (stats) {
    p.out_m = stats[0];
    p.out_Z = stats[1];
    p.out_psum = stats[2];
  }
  CUtensorMap tmX, tmR1, tmR2, tmS;
  const CUtensorMapSwizzle r1sw = C::R1_ROW == 32   ? CU_TENSOR_MAP_SWIZZLE_32B
                                  : C::R1_ROW == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                    : CU_TENSOR_MAP_SWIZZLE_128B;
  const CUtensorMapSwizzle xsw = C::BK == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  constexpr CUtensorMapDataType bf16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, f32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  if (!make_map(&tmX, bf16, 2, a.X, (uint64_t)a.h, (uint64_t)a.N, C::BK, kBT, xsw) ||
      !make_map(&tmR1, bf16, 2, a.R1, (uint64_t)R, (uint64_t)a.h, C::R1_BOX, C::BK, r1sw) ||
      !make_map(&tmR2, bf16, 2, a.R2, (uint64_t)a.M, (uint64_t)R, 64, R, CU_TENSOR_MAP_SWIZZLE_128B) ||
      (!stats && !make_map(&tmS, f32, 4, scores, (uint64_t)a.M, (uint64_t)a.N, 32, 32, CU_TENSOR_MAP_SWIZZLE_128B)))
    return cudaErrorInvalidValue;
  if (stats) tmS = tmX;  // unused by the statistics
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = stats ? configure_once<R, true>(dev) : configure_once<R, false>(dev);
  if (e != cudaSuccess) return e;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = p.num_tiles < sms ? p.num_tiles : sms;
  if (stats)
    tc_logits_kernel<R, true><<<grid, kThreads, smem, a.stream>>>(tmX, tmR1, tmR2, tmS, p);
  else
    tc_logits_kernel<R, false><<<grid, kThreads, smem, a.stream>>>(tmX, tmR1, tmR2, tmS, p);
  return cudaGetLastError();
}

}  // namespace mat

namespace {
bool tc_logits_fits(const RouteArgs& a, int sweeps) {
  if (a.N < 1 || a.N > 0x7fffffffLL - mat::kBT || !mat::encode_fn()) return false;
  mat::Params p;
  uint32_t smem;
  switch (a.r) {
    case 16: return mat::fill_params<16>(a, p, smem, sweeps);
    case 32: return mat::fill_params<32>(a, p, smem, sweeps);
    case 64: return mat::fill_params<64>(a, p, smem, sweeps);
    case 128: return mat::fill_params<128>(a, p, smem, sweeps);
    default: return false;
  }
}

cudaError_t launch_tc_logits(const RouteArgs& a, float* scores, float* const* stats) {
  switch (a.r) {
    case 16: return mat::launch<16>(a, scores, stats);
    case 32: return mat::launch<32>(a, scores, stats);
    case 64: return mat::launch<64>(a, scores, stats);
    case 128: return mat::launch<128>(a, scores, stats);
    default: return cudaErrorInvalidValue;
  }
}
}  // namespace

bool unfused_tc_supports(const RouteArgs& a) { return tc_logits_fits(a, 1); }

bool train_stats_tc_supports(const RouteArgs& a) { return tc_logits_fits(a, 2); }

cudaError_t launch_train_stats_tc(const RouteArgs& a, float* out_m, float* out_Z, float* out_psum) {
  float* const stats[3] = {out_m, out_Z, out_psum};
  return launch_tc_logits(a, nullptr, stats);
}

cudaError_t launch_unfused_tc(const RouteArgs& a, void* scratch) {
  float* scores = unfused_scores_of(scratch, a.N, a.r);
  const cudaError_t e = launch_tc_logits(a, scores, nullptr);
  if (e != cudaSuccess) return e;
  return launch_threshold_topk(a, scores);
}

}  // namespace more

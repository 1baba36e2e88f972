// Backward of the low-rank router ("MoRE: Scaling mixture of experts with hardware-aware
// low-rank routing", App. F, F.2.2, Algorithm 3 and eqs. (10)-(12)), in fp32 on the CUDA cores.
//
// With z = X R1, l = z R2 and P = exp(l - m) / Z (m, Z saved by the training forward,
// Algorithm 2), the incoming gradients top_vals_bar (on the k selected logits of each token)
// and pbar (on psum) give
//   g_n     = sum_i pbar_i P_ni                                  (eq. (12))
//   ybar_ni = P_ni (pbar_i - g_n) + sum_j [top_idx_nj = i] top_vals_bar_nj
//   zbar    = ybar R2^T,   Xbar = zbar R1^T,   R1bar = X^T zbar,   R2bar = z^T ybar.
// Four kernels, deterministic (no atomics on the gradients):
//   1. token blocks, as Algorithm 3: z recomputed from X, sweep 1 over the expert tiles for g,
//      sweep 2 for zbar, then Xbar; z, zbar and g go to scratch;
//   2. expert tiles x token splits: ybar of the tile recomputed from z, g, m, Z (the same
//      arithmetic as kernel 1, so the same values), and the split's part of z^T ybar;
//   3. hidden tiles x token splits: the split's part of X^T zbar;
//   4. the splits' parts summed in a fixed order into R1bar and R2bar.
// Algorithm 3 adds the R1bar / R2bar contributions of every token block into one HBM copy;
// the splits here trade that for a fixed summation order.  Every global access checks its
// row and column against the array's extent; shared-memory tiles are zero-padded.
#include <algorithm>

#include <atomic>

#include "more_internal.cuh"

namespace more {
namespace {

constexpr int kBN = 32;       // tokens per block
constexpr int kBM = 64;       // experts per tile
constexpr int kHT = 64;       // hidden columns per tile
constexpr int kThreads = 256;
constexpr int kTargetCtas = 2 * 148;  // CTAs the split kernels aim for (two per SM)

static_assert(kThreads == kBN * 8, "token-major maps use thread (t = tid / 8, q = tid % 8)");
static_assert(kThreads == kBM * 4 && kThreads == kHT * 4, "column maps use (tid % 64, tid / 64)");

// z and zbar live in scratch as [N][RP] fp32 rows, r padded with zeros to RP.
int padded_r(int r) { return r <= 16 ? 16 : r <= 32 ? 32 : r <= 64 ? 64 : 128; }

struct BwdArgs {
  const __nv_bfloat16* X;   // [N][h]
  const __nv_bfloat16* R1;  // [h][r]
  const __nv_bfloat16* R2;  // [r][M]
  int64_t N;
  int h, r, M, k;
  const int32_t* idx;  // [N][k] or null (with tvb)
  const float* tvb;    // [N][k] or null
  const float* pbar;   // [M] or null (then m, Z unused)
  const float* m;      // [N]
  const float* Z;      // [N]
  float* Xbar;         // [N][h]
  float* g_out;        // [N] or null
  float* z;            // scratch [N][RP]
  float* zbar;         // scratch [N][RP]
  float* g;            // scratch [N]
  float* part1;        // scratch [S1][h][r]
  float* part2;        // scratch [S2][r][M]
  int S1, S2;
  unsigned int* status;
};

template <int RP>
struct Tiles {
  static constexpr int ZLD = RP + 1;   // row stride of z / zbar tiles
  static constexpr int R1LD = RP + 1;  // row stride of an R1 tile (kHT rows)
  static constexpr int TLD = kBM + 1;  // row stride of R2 tiles (RP rows) and ybar tiles (kBN rows)
  static constexpr int XLD = kHT + 1;  // row stride of X tiles (kBN rows)
  static constexpr int kZ = kBN * ZLD;
  static constexpr int kTok = 3 * kBN + kBM + 2 * kBN * MORE_KMAX;  // m, 1/Z, g, pbar tile, selections
  static constexpr int kPhase1 = kBN * XLD + kHT * R1LD;            // X tile + R1 tile
  static constexpr int kSweep = RP * TLD + kBN * TLD;               // R2 tile + ybar tile
  static constexpr int kUnion = kPhase1 > kSweep ? kPhase1 : kSweep;
  static constexpr int kTokenBlockFloats = 2 * kZ + kTok + kUnion;  // kernel 1
  static constexpr int kR2Floats = kZ + kTok + kSweep;              // kernel 2
  static constexpr int kR1Floats = kBN * XLD + kZ;                  // kernel 3
};

// Per-token staging shared by kernels 1 and 2: m, 1/Z, the token's selections (expert id,
// gradient; id -1 where absent or out of range) for tokens [n0, n0 + nb).
__device__ __forceinline__ void stage_tokens(const BwdArgs& a, int64_t n0, int nb, bool balance,
                                             bool flag_bad, float* tm, float* tzi, int* sidx,
                                             float* sval) {
  for (int i = threadIdx.x; i < kBN; i += kThreads) {
    const bool ok = i < nb && balance;
    tm[i] = ok ? a.m[n0 + i] : 0.f;
    tzi[i] = ok ? 1.f / a.Z[n0 + i] : 0.f;
  }
  for (int i = threadIdx.x; i < kBN * MORE_KMAX; i += kThreads) {
    const int tt = i / MORE_KMAX, s = i % MORE_KMAX;
    int e = -1;
    float v = 0.f;
    if (a.tvb && tt < nb && s < a.k) {
      const int64_t off = (n0 + tt) * a.k + s;
      e = a.idx[off];
      v = a.tvb[off];
      if ((unsigned)e >= (unsigned)a.M) {
        if (flag_bad) atomicOr(a.status, MORE_DEVERR_BAD_INPUT);
        e = -1;
        v = 0.f;
      }
    }
    sidx[i] = e;
    sval[i] = v;
  }
}

// R2 columns [m0, m0 + kBM) into r2t[c][e] (zero where c >= r or m0 + e >= M), pbar into pbt.
template <int RP>
__device__ __forceinline__ void stage_r2(const BwdArgs& a, int m0, float* r2t, float* pbt) {
  using T = Tiles<RP>;
  for (int i = threadIdx.x; i < RP * kBM; i += kThreads) {
    const int c = i / kBM, e = i % kBM;
    float v = 0.f;
    if (c < a.r && m0 + e < a.M) v = __bfloat162float(a.R2[(int64_t)c * a.M + m0 + e]);
    r2t[c * T::TLD + e] = v;
  }
  for (int i = threadIdx.x; i < kBM; i += kThreads) pbt[i] = (a.pbar && m0 + i < a.M) ? a.pbar[m0 + i] : 0.f;
}

// R1 rows [h0, h0 + kHT) into r1t[j][c] (zero where h0 + j >= h or c >= r).
template <int RP>
__device__ __forceinline__ void stage_r1(const BwdArgs& a, int h0, float* r1t) {
  using T = Tiles<RP>;
  for (int i = threadIdx.x; i < kHT * RP; i += kThreads) {
    const int j = i / RP, c = i % RP;
    float v = 0.f;
    if (h0 + j < a.h && c < a.r) v = __bfloat162float(a.R1[(int64_t)(h0 + j) * a.r + c]);
    r1t[j * T::R1LD + c] = v;
  }
}

// X rows [n0, n0 + nb), columns [h0, h0 + kHT) into xt[t][j] (zero outside).
template <int RP>
__device__ __forceinline__ void stage_x(const BwdArgs& a, int64_t n0, int nb, int h0, float* xt) {
  using T = Tiles<RP>;
  for (int i = threadIdx.x; i < kBN * kHT; i += kThreads) {
    const int tt = i / kHT, j = i % kHT;
    float v = 0.f;
    if (tt < nb && h0 + j < a.h) v = __bfloat162float(a.X[(n0 + tt) * a.h + h0 + j]);
    xt[tt * T::XLD + j] = v;
  }
}

// Logits of token t for experts q + 8 v of the staged tile (zero-padded z and R2).
template <int RP>
__device__ __forceinline__ void tile_logits(const float* zt, const float* r2t, int t, int q, float (&l)[8]) {
  using T = Tiles<RP>;
#pragma unroll
  for (int v = 0; v < 8; ++v) l[v] = 0.f;
#pragma unroll 4
  for (int c = 0; c < RP; ++c) {
    const float zc = zt[t * T::ZLD + c];
#pragma unroll
    for (int v = 0; v < 8; ++v) l[v] = fmaf(zc, r2t[c * T::TLD + q + 8 * v], l[v]);
  }
}

// Does any selection of the block fall in experts [m0, m0 + kBM)?  (Block-wide; every thread calls.)
__device__ __forceinline__ bool tile_selected(const int* sidx, int m0, int k) {
  int any = 0;
  for (int i = threadIdx.x; i < kBN * MORE_KMAX; i += kThreads) {
    const int d = sidx[i] - m0;
    any |= (i % MORE_KMAX < k && sidx[i] >= 0 && d >= 0 && d < kBM);
  }
  return __syncthreads_or(any) != 0;
}

// ybar of token t, experts q + 8 v of the tile at m0, into yt[t][.]: the softmax term where the
// balancing gradient is present, plus the token's selected-logit gradients.
template <int RP>
__device__ __forceinline__ void ybar_tile(const BwdArgs& a, const float* zt, const float* r2t, const float* pbt,
                                          const float* tm, const float* tzi, const float* tg, const int* sidx,
                                          const float* sval, float* yt, int t, int q, int nb, int m0,
                                          bool balance) {
  using T = Tiles<RP>;
  float y[8];
#pragma unroll
  for (int v = 0; v < 8; ++v) y[v] = 0.f;
  if (balance) {
    float l[8];
    tile_logits<RP>(zt, r2t, t, q, l);
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      const int e = q + 8 * v;
      if (t < nb && m0 + e < a.M) y[v] = expf(l[v] - tm[t]) * tzi[t] * (pbt[e] - tg[t]);
    }
  }
  for (int s = 0; s < a.k; ++s) {
    const int i = sidx[t * MORE_KMAX + s];
    const int d = i - m0;
    if (i >= 0 && d >= 0 && d < kBM) {
      const float val = sval[t * MORE_KMAX + s];
#pragma unroll
      for (int v = 0; v < 8; ++v)
        if (d == q + 8 * v) y[v] += val;
    }
  }
#pragma unroll
  for (int v = 0; v < 8; ++v) yt[t * T::TLD + q + 8 * v] = y[v];
}

// Kernel 1: one CTA per block of kBN tokens.
template <int RP>
__global__ void __launch_bounds__(kThreads) bwd_token_block_kernel(BwdArgs a) {
  using T = Tiles<RP>;
  extern __shared__ float4 smem4[];
  float* zt = reinterpret_cast<float*>(smem4);  // [kBN][ZLD]
  float* zbt = zt + T::kZ;                       // [kBN][ZLD]
  float* tm = zbt + T::kZ;                       // [kBN]
  float* tzi = tm + kBN;                         // [kBN]
  float* tg = tzi + kBN;                         // [kBN]
  float* pbt = tg + kBN;                         // [kBM]
  int* sidx = reinterpret_cast<int*>(pbt + kBM);  // [kBN][KMAX]
  float* sval = reinterpret_cast<float*>(sidx + kBN * MORE_KMAX);
  float* un = sval + kBN * MORE_KMAX;  // phase buffers
  float* xt = un;                      // phase 1: [kBN][XLD]
  float* r1t = un + kBN * T::XLD;      // phases 1 and 3: [kHT][R1LD]
  float* r2t = un;                     // sweeps: [RP][TLD]
  float* yt = un + RP * T::TLD;        // sweep 2: [kBN][TLD]
  static_assert(2 * T::kZ + T::kTok == 2 * T::kZ + 3 * kBN + kBM + 2 * kBN * MORE_KMAX, "layout");

  const int tid = threadIdx.x, t = tid >> 3, q = tid & 7;
  const int64_t n0 = (int64_t)blockIdx.x * kBN;
  const int nb = (int)(a.N - n0 < kBN ? a.N - n0 : kBN);
  const bool balance = a.pbar != nullptr;

  stage_tokens(a, n0, nb, balance, true, tm, tzi, sidx, sval);
  if (tid < kBN) tg[tid] = 0.f;

  // Phase 1: z = X_block R1 over hidden tiles; thread (t, q) owns columns q + 8 u.
  float acc[RP / 8];
#pragma unroll
  for (int u = 0; u < RP / 8; ++u) acc[u] = 0.f;
  for (int h0 = 0; h0 < a.h; h0 += kHT) {
    stage_x<RP>(a, n0, nb, h0, xt);
    stage_r1<RP>(a, h0, r1t);
    __syncthreads();
#pragma unroll 4
    for (int j = 0; j < kHT; ++j) {
      const float xv = xt[t * T::XLD + j];
#pragma unroll
      for (int u = 0; u < RP / 8; ++u) acc[u] = fmaf(xv, r1t[j * T::R1LD + q + 8 * u], acc[u]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < RP / 8; ++u) zt[t * T::ZLD + q + 8 * u] = acc[u];  // zero rows past nb
  if (t < nb) {
#pragma unroll
    for (int u = 0; u < RP / 8; ++u) a.z[(n0 + t) * RP + q + 8 * u] = acc[u];
  }
  __syncthreads();

  // Phase 2, sweep 1: g_n = sum_i pbar_i P_ni over all expert tiles.
  if (balance) {
    float gacc = 0.f;
    for (int m0 = 0; m0 < a.M; m0 += kBM) {
      stage_r2<RP>(a, m0, r2t, pbt);
      __syncthreads();
      float l[8];
      tile_logits<RP>(zt, r2t, t, q, l);
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        const int e = q + 8 * v;
        if (t < nb && m0 + e < a.M) gacc = fmaf(expf(l[v] - tm[t]) * tzi[t], pbt[e], gacc);
      }
      __syncthreads();
    }
    gacc += __shfl_xor_sync(0xffffffffu, gacc, 1);  // the 8 lanes of token t are lanes 8 (t % 4) + q
    gacc += __shfl_xor_sync(0xffffffffu, gacc, 2);
    gacc += __shfl_xor_sync(0xffffffffu, gacc, 4);
    if (q == 0) tg[t] = gacc;
    __syncthreads();
  }
  if (tid < nb) {
    a.g[n0 + tid] = tg[tid];
    if (a.g_out) a.g_out[n0 + tid] = tg[tid];
  }

  // Phase 2, sweep 2: ybar tile by tile, contracted into zbar; thread (t, q) owns columns q + 8 u.
  float zb[RP / 8];
#pragma unroll
  for (int u = 0; u < RP / 8; ++u) zb[u] = 0.f;
  for (int m0 = 0; m0 < a.M; m0 += kBM) {
    if (!balance && !tile_selected(sidx, m0, a.k)) continue;  // ybar is zero on this tile
    stage_r2<RP>(a, m0, r2t, pbt);
    __syncthreads();
    ybar_tile<RP>(a, zt, r2t, pbt, tm, tzi, tg, sidx, sval, yt, t, q, nb, m0, balance);
    __syncthreads();
#pragma unroll 4
    for (int e = 0; e < kBM; ++e) {
      const float yv = yt[t * T::TLD + e];
#pragma unroll
      for (int u = 0; u < RP / 8; ++u) zb[u] = fmaf(yv, r2t[(q + 8 * u) * T::TLD + e], zb[u]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < RP / 8; ++u) zbt[t * T::ZLD + q + 8 * u] = zb[u];
  if (t < nb) {
#pragma unroll
    for (int u = 0; u < RP / 8; ++u) a.zbar[(n0 + t) * RP + q + 8 * u] = zb[u];
  }
  __syncthreads();

  // Phase 3: Xbar_block = zbar R1^T over hidden tiles; thread (t, q) owns columns q + 8 w.
  for (int h0 = 0; h0 < a.h; h0 += kHT) {
    stage_r1<RP>(a, h0, r1t);
    __syncthreads();
    float xb[kHT / 8];
#pragma unroll
    for (int w = 0; w < kHT / 8; ++w) xb[w] = 0.f;
#pragma unroll 4
    for (int c = 0; c < RP; ++c) {
      const float zv = zbt[t * T::ZLD + c];
#pragma unroll
      for (int w = 0; w < kHT / 8; ++w) xb[w] = fmaf(zv, r1t[(q + 8 * w) * T::R1LD + c], xb[w]);
    }
    if (t < nb) {
#pragma unroll
      for (int w = 0; w < kHT / 8; ++w) {
        const int j = h0 + q + 8 * w;
        if (j < a.h) a.Xbar[(n0 + t) * a.h + j] = xb[w];
      }
    }
    __syncthreads();
  }
}

// Token range [b, end) of split s of S.
__device__ __forceinline__ void split_range(int64_t N, int S, int s, int64_t& b, int64_t& end) {
  const int64_t chunk = (N + S - 1) / S;
  b = (int64_t)s * chunk;
  end = b + chunk < N ? b + chunk : N;
}

// Kernel 2: CTA (expert tile blockIdx.x, split blockIdx.y); part2[s][c][m0 + e] = the split's
// sum over tokens of z_nc ybar_n,m0+e.  Thread owns expert e = tid % 64, columns tid / 64 + 4 u.
template <int RP>
__global__ void __launch_bounds__(kThreads) bwd_r2_kernel(BwdArgs a) {
  using T = Tiles<RP>;
  extern __shared__ float4 smem4[];
  float* zt = reinterpret_cast<float*>(smem4);  // [kBN][ZLD]
  float* tm = zt + T::kZ;
  float* tzi = tm + kBN;
  float* tg = tzi + kBN;
  float* pbt = tg + kBN;
  int* sidx = reinterpret_cast<int*>(pbt + kBM);
  float* sval = reinterpret_cast<float*>(sidx + kBN * MORE_KMAX);
  float* r2t = sval + kBN * MORE_KMAX;  // [RP][TLD]
  float* yt = r2t + RP * T::TLD;        // [kBN][TLD]

  const int tid = threadIdx.x, t = tid >> 3, q = tid & 7;
  const int e = tid % kBM, cg = tid / kBM;
  const int m0 = blockIdx.x * kBM, s = blockIdx.y;
  const bool balance = a.pbar != nullptr;
  int64_t b, end;
  split_range(a.N, a.S2, s, b, end);

  stage_r2<RP>(a, m0, r2t, pbt);
  float acc[RP / 4];
#pragma unroll
  for (int u = 0; u < RP / 4; ++u) acc[u] = 0.f;
  for (int64_t n0 = b; n0 < end; n0 += kBN) {
    const int nb = (int)(end - n0 < kBN ? end - n0 : kBN);
    __syncthreads();  // the previous block's tiles are no longer read
    stage_tokens(a, n0, nb, balance, false, tm, tzi, sidx, sval);
    for (int i = tid; i < kBN * RP; i += kThreads) {
      const int tt = i / RP, c = i % RP;
      zt[tt * T::ZLD + c] = tt < nb ? a.z[(n0 + tt) * RP + c] : 0.f;
    }
    if (tid < kBN) tg[tid] = tid < nb ? a.g[n0 + tid] : 0.f;
    if (!balance && !tile_selected(sidx, m0, a.k)) continue;  // (block-uniform) ybar is zero here
    __syncthreads();
    ybar_tile<RP>(a, zt, r2t, pbt, tm, tzi, tg, sidx, sval, yt, t, q, nb, m0, balance);
    __syncthreads();
#pragma unroll 4
    for (int tt = 0; tt < kBN; ++tt) {
      const float yv = yt[tt * T::TLD + e];
#pragma unroll
      for (int u = 0; u < RP / 4; ++u) acc[u] = fmaf(zt[tt * T::ZLD + cg + 4 * u], yv, acc[u]);
    }
  }
  if (m0 + e < a.M) {
#pragma unroll
    for (int u = 0; u < RP / 4; ++u) {
      const int c = cg + 4 * u;
      if (c < a.r) a.part2[((int64_t)s * a.r + c) * a.M + m0 + e] = acc[u];
    }
  }
}

// Kernel 3: CTA (hidden tile blockIdx.x, split blockIdx.y); part1[s][h0 + j][c] = the split's sum
// over tokens of X_n,h0+j zbar_nc.  Thread owns hidden column j = tid % 64, columns tid / 64 + 4 u.
template <int RP>
__global__ void __launch_bounds__(kThreads) bwd_r1_kernel(BwdArgs a) {
  using T = Tiles<RP>;
  extern __shared__ float4 smem4[];
  float* xt = reinterpret_cast<float*>(smem4);  // [kBN][XLD]
  float* zbt = xt + kBN * T::XLD;                // [kBN][ZLD]

  const int tid = threadIdx.x, j = tid % kHT, cg = tid / kHT;
  const int h0 = blockIdx.x * kHT, s = blockIdx.y;
  int64_t b, end;
  split_range(a.N, a.S1, s, b, end);

  float acc[RP / 4];
#pragma unroll
  for (int u = 0; u < RP / 4; ++u) acc[u] = 0.f;
  for (int64_t n0 = b; n0 < end; n0 += kBN) {
    const int nb = (int)(end - n0 < kBN ? end - n0 : kBN);
    __syncthreads();
    stage_x<RP>(a, n0, nb, h0, xt);
    for (int i = tid; i < kBN * RP; i += kThreads) {
      const int tt = i / RP, c = i % RP;
      zbt[tt * T::ZLD + c] = tt < nb ? a.zbar[(n0 + tt) * RP + c] : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int tt = 0; tt < kBN; ++tt) {
      const float xv = xt[tt * T::XLD + j];
#pragma unroll
      for (int u = 0; u < RP / 4; ++u) acc[u] = fmaf(xv, zbt[tt * T::ZLD + cg + 4 * u], acc[u]);
    }
  }
  if (h0 + j < a.h) {
#pragma unroll
    for (int u = 0; u < RP / 4; ++u) {
      const int c = cg + 4 * u;
      if (c < a.r) a.part1[((int64_t)s * a.h + h0 + j) * a.r + c] = acc[u];
    }
  }
}

// Kernel 4: out[i] = sum over s of part[s][i], s in increasing order.
__global__ void bwd_sum_parts_kernel(const float* __restrict__ part, int S, int64_t L, float* __restrict__ out) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < L; i += (int64_t)gridDim.x * blockDim.x) {
    float v = 0.f;
    for (int s = 0; s < S; ++s) v += part[(int64_t)s * L + i];
    out[i] = v;
  }
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Token splits of the two reduction kernels: enough CTAs for two per SM, at most one per block.
void split_counts(int64_t N, int h, int M, int& S1, int& S2) {
  const int64_t blocks = std::max<int64_t>(1, ceil_div(N, kBN));
  S1 = (int)std::min<int64_t>(blocks, std::max<int64_t>(1, ceil_div(kTargetCtas, ceil_div(h, kHT))));
  S2 = (int)std::min<int64_t>(blocks, std::max<int64_t>(1, ceil_div(kTargetCtas, ceil_div(M, kBM))));
}

struct ScratchLayout {
  int64_t z, zbar, g, part1, part2, total;  // float offsets
};

ScratchLayout scratch_layout(int64_t N, int h, int r, int M) {
  int S1, S2;
  split_counts(N, h, M, S1, S2);
  const int64_t RP = padded_r(r);
  ScratchLayout L;
  L.z = 0;
  L.zbar = L.z + N * RP;
  L.g = L.zbar + N * RP;
  L.part1 = L.g + ceil_div(N, 4) * 4;
  L.part2 = L.part1 + (int64_t)S1 * h * r;
  L.total = L.part2 + (int64_t)S2 * r * M;
  return L;
}

template <int RP>
cudaError_t launch_rp(BwdArgs a, cudaStream_t stream) {
  using T = Tiles<RP>;
  const size_t tok_bytes = sizeof(float) * T::kTokenBlockFloats;
  const size_t r2_bytes = sizeof(float) * T::kR2Floats;
  const size_t r1_bytes = sizeof(float) * T::kR1Floats;
  // shared-memory limits, set once per device (a call captured into a CUDA graph then only launches)
  static std::atomic<int> configured[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !configured[dev].load(std::memory_order_acquire)) {
    if ((e = cudaFuncSetAttribute(bwd_token_block_kernel<RP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)tok_bytes)) != cudaSuccess)
      return e;
    if ((e = cudaFuncSetAttribute(bwd_r2_kernel<RP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)r2_bytes)) != cudaSuccess)
      return e;
    if ((e = cudaFuncSetAttribute(bwd_r1_kernel<RP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)r1_bytes)) != cudaSuccess)
      return e;
    if (dev >= 0 && dev < 64) configured[dev].store(1, std::memory_order_release);
  }
  const unsigned blocks = (unsigned)ceil_div(a.N, kBN);
  bwd_token_block_kernel<RP><<<blocks, kThreads, tok_bytes, stream>>>(a);
  bwd_r2_kernel<RP><<<dim3((unsigned)ceil_div(a.M, kBM), (unsigned)a.S2), kThreads, r2_bytes, stream>>>(a);
  bwd_r1_kernel<RP><<<dim3((unsigned)ceil_div(a.h, kHT), (unsigned)a.S1), kThreads, r1_bytes, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

int64_t backward_scratch_bytes(int64_t N, int h, int r, int M) {
  return scratch_layout(N, h, r, M).total * (int64_t)sizeof(float);
}

cudaError_t launch_backward(const BackwardArgs& b) {
  cudaStream_t stream = b.stream;
  if (b.N == 0) {
    cudaError_t e = cudaMemsetAsync(b.R1bar, 0, sizeof(float) * (size_t)b.h * b.r, stream);
    if (e != cudaSuccess) return e;
    return cudaMemsetAsync(b.R2bar, 0, sizeof(float) * (size_t)b.r * b.M, stream);
  }
  const ScratchLayout L = scratch_layout(b.N, b.h, b.r, b.M);
  float* base = static_cast<float*>(b.scratch);
  BwdArgs a;
  a.X = b.X;
  a.R1 = b.R1;
  a.R2 = b.R2;
  a.N = b.N;
  a.h = b.h;
  a.r = b.r;
  a.M = b.M;
  a.k = b.k;
  a.idx = b.top_idx;
  a.tvb = b.top_vals_bar;
  a.pbar = b.pbar;
  a.m = b.m;
  a.Z = b.Z;
  a.Xbar = b.Xbar;
  a.g_out = b.g;
  a.z = base + L.z;
  a.zbar = base + L.zbar;
  a.g = base + L.g;
  a.part1 = base + L.part1;
  a.part2 = base + L.part2;
  split_counts(b.N, b.h, b.M, a.S1, a.S2);
  a.status = b.status;
  cudaError_t e;
  switch (padded_r(b.r)) {
    case 16:
      e = launch_rp<16>(a, stream);
      break;
    case 32:
      e = launch_rp<32>(a, stream);
      break;
    case 64:
      e = launch_rp<64>(a, stream);
      break;
    default:
      e = launch_rp<128>(a, stream);
      break;
  }
  if (e != cudaSuccess) return e;
  const int64_t L1 = (int64_t)b.h * b.r, L2 = (int64_t)b.r * b.M;
  bwd_sum_parts_kernel<<<(unsigned)std::min<int64_t>(ceil_div(L1, 256), 4 * 148), 256, 0, stream>>>(
      a.part1, a.S1, L1, b.R1bar);
  bwd_sum_parts_kernel<<<(unsigned)std::min<int64_t>(ceil_div(L2, 256), 4 * 148), 256, 0, stream>>>(
      a.part2, a.S2, L2, b.R2bar);
  return cudaGetLastError();
}

}  // namespace more

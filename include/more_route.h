/*
 * more_route.h - C ABI of the fused low-rank MoE router for NVIDIA B200 (sm_100a).
 *
 * The operation is the MoRE router of "MoRE: Scaling mixture of experts with
 * hardware-aware low-rank routing" (arXiv 2609.36301):
 *   §2 "MoRE layer":  g(x; R1, R2) = softmax(TopK(R1 R2 x)), the standard router
 *                     softmax(TopK(R x)) with R replaced by a rank-r product;
 *   App. F, eq. (5):  logits l = X R_2^T R_1^T, one B_N x B_M tile at a time;
 *   App. F, Algorithm 1 (inference, prefilling): z = X R_2^T accumulated in
 *                     fp32 and narrowed to bf16, one sweep over the experts with a
 *                     running top-k, out-of-range experts at -infinity, and the
 *                     (N, k) TopVals/TopIdxs written instead of the (N, M) logits;
 *   App. F, Fig. 12:  gate weights = softmax over the k selected logits;
 *   App. F, eq. (9):  f = bincount of TopIdxs (here: out_expert_count).
 *
 * Naming: R1 here is h x r (the paper's R_2 transposed) and R2 is r x M (the
 * paper's R_1 transposed), so z = x . R1 and l = z . R2.
 *
 * Conventions shared by every entry point:
 *   - All tensors are row-major and live in device memory owned by the caller.
 *     bf16 tensors are raw 16-bit patterns.  Nothing is retained after a call.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and never synchronise the host, except more_device_status.
 *   - Per token the k experts are returned in routing order: larger logit
 *     first, lower expert index first on equal logits (Algorithm 1 keeps the
 *     earlier expert on equal values).  out_logits[n][j] is the fp32 logit of
 *     expert out_idx[n][j]; out_gate[n][] is the softmax of those k logits.
 *   - Precision: z = x . R1 is accumulated in fp32 and carried into the second
 *     product as a pair of bf16 terms, z_hi = bf16(z) and z_lo = bf16(z - z_hi)
 *     (nearest even), so z keeps about 16 significant bits; l = (z_hi + z_lo) . R2
 *     is accumulated in fp32.  Algorithm 1 narrows z to a single bf16; that alone
 *     moves logits by up to about 1% of their RMS, the whole parity tolerance.
 *   - out_expert_count[e] is set (not accumulated) to the number of (token,
 *     slot) pairs of this call that name expert e; the call zeroes it first.
 *   - Inputs must be finite; results for NaN or infinite inputs are unspecified.
 *
 * Argument requirements (checked before anything is launched; a violation
 * returns an error and launches nothing):
 *   N >= 0; h >= 8 and h % 8 == 0; M >= 8 and M % 8 == 0; r % 16 == 0 and
 *   16 <= r <= 128; 1 <= k <= M; k <= MORE_KMAX; M <= MORE_MMAX;
 *   R1, R2 and out_expert_count non-NULL, and X, out_idx and out_gate non-NULL
 *   unless N == 0; every non-NULL pointer 16-byte aligned.  Violations of the shape limits that are
 *   not errors of meaning (k > MORE_KMAX, r outside 16..128 or not a multiple
 *   of 16, M > MORE_MMAX) return MORE_ERR_UNSUPPORTED; the rest return
 *   MORE_ERR_INVALID_ARG.
 */
#ifndef MORE_ROUTE_H
#define MORE_ROUTE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MORE_ROUTE_ABI_VERSION 1
#define MORE_KMAX 16
#define MORE_MMAX 262144

typedef enum more_status {
  MORE_OK = 0,
  MORE_ERR_INVALID_ARG = 1, /* null/misaligned pointer, impossible shape          */
  MORE_ERR_UNSUPPORTED = 2, /* legal request outside this library's limits        */
  MORE_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed        */
  MORE_ERR_DEVICE = 4       /* a kernel recorded an error (see more_device_status) */
} more_status;

/* Kernel variants of more_route_variant.  All compute the same function. */
typedef enum more_variant {
  MORE_VARIANT_AUTO = 0,     /* chosen per shape: see more_route_auto_variant                         */
  MORE_VARIANT_FUSED_TC = 1, /* persistent kernel: TMA-staged X, tcgen05 MMAs into TMEM             */
  MORE_VARIANT_SMALL_N = 2,  /* CUDA-core kernel, one CTA of 16 warps per token (decode batches)    */
  MORE_VARIANT_CLUSTER = 3   /* CUDA-core kernel, 8 tokens per cluster of 8 CTAs: experts split over
                                the cluster, partial top-k merged through distributed shared memory */
} more_variant;

/*
 * Route N tokens.  [MoRE §2 "MoRE layer"; App. F, Algorithm 1 and Fig. 12]
 *   X                bf16 [N][h]      token hidden vectors
 *   R1               bf16 [h][r]      first router factor
 *   R2               bf16 [r][M]      second router factor (one column per expert)
 *   out_idx          int32 [N][k]     selected experts, routing order
 *   out_gate         fp32 [N][k]      softmax over the k selected logits
 *   out_expert_count int32 [M]        selections per expert (zeroed, then counted)
 *   out_logits       fp32 [N][k]      selected logits, or NULL to skip
 * No N x M tensor is written: the logits exist only on chip.
 */
more_status more_route(const void* X, const void* R1, const void* R2, int64_t N, int h, int r, int M,
                       int k, int32_t* out_idx, float* out_gate, int32_t* out_expert_count,
                       float* out_logits, void* stream);

/*
 * The kernel AUTO runs for this shape (a more_variant value), or MORE_VARIANT_AUTO if the shape
 * fails the argument requirements.  The choice follows per-call times measured on a B200:
 *   - N <= 148: MORE_VARIANT_SMALL_N (one CTA per token, a single wave on a B200's 148 SMs),
 *     except where the weights one CTA would read, r * (h + M) values, reach 196608 with
 *     N <= 64 or 393216 at any N <= 148: there MORE_VARIANT_CLUSTER, which spreads them over
 *     eight SMs (at h = 2048, M = 4096: r = 32 with N <= 64, and r >= 64);
 *   - otherwise MORE_VARIANT_CLUSTER while its time, which grows with N, stays below the fused
 *     kernel's floor (the latency of one 128-token tile: Z over h, then two sweeps over the
 *     M / 128 expert tiles); MORE_VARIANT_FUSED_TC beyond.  At h = 2048, M = 4096 the switch
 *     falls near N = 1,440 (r = 32) and N = 1,920 (r = 16);
 *   - MORE_VARIANT_CLUSTER at any N > 148 for shapes the fused kernel's shared-memory plan
 *     cannot hold: r = 128 with k > 8 (any M), every r not in {16, 32, 64, 128}, and
 *     M > 65536.  Those shapes run on CUDA cores, far slower per token at prefill sizes than
 *     the fused kernel (r = 128, k = 16, M = 4096: about 0.26 us per token against 2.1 ns for
 *     the fused kernel at r = 32).
 * Host-only; makes no CUDA call.
 */
int more_route_auto_variant(int64_t N, int h, int r, int M, int k);

/* more_route with an explicit kernel variant (more_variant); same contract. */
more_status more_route_variant(const void* X, const void* R1, const void* R2, int64_t N, int h, int r,
                               int M, int k, int32_t* out_idx, float* out_gate,
                               int32_t* out_expert_count, float* out_logits, int variant,
                               void* stream);

/*
 * Materialise-then-top-k comparison path (the unfused router of MoRE App. H.6,
 * Fig. 24): z = X . R1 (as z_hi + z_lo, see Precision) is written to scratch as
 * fp32 [N][r], the full logits as fp32 [N][M], then a row-wise top-k and
 * softmax read them back.  Same
 * arguments and results as more_route, plus caller-owned device scratch of at
 * least more_route_unfused_scratch_bytes(N, r, M) bytes (16-byte aligned).
 * Too little scratch returns MORE_ERR_INVALID_ARG.
 */
size_t more_route_unfused_scratch_bytes(int64_t N, int r, int M);
more_status more_route_unfused(const void* X, const void* R1, const void* R2, int64_t N, int h, int r,
                               int M, int k, int32_t* out_idx, float* out_gate,
                               int32_t* out_expert_count, float* out_logits, void* scratch,
                               size_t scratch_bytes, void* stream);

/*
 * The materialise-then-top-k comparison on the tensor cores (MoRE App. H.6, Fig. 24, with
 * the fused kernel's products): z = X . R1 accumulated in TMEM and narrowed to the bf16
 * pair, then the exact logits of every 128-expert tile as one tcgen05 product of K = 2r,
 * written to the fp32 [N][M] scores in scratch by TMA tile stores; the row-wise top-k and
 * softmax of more_route_unfused read them back.  The scores differ from the fused kernel's
 * only in being written out, so the two calls time the HBM round trip of the N x M tensor.
 * Same arguments, scratch size (more_route_unfused_scratch_bytes; the z area is unused)
 * and results as more_route_unfused.  r must be 16, 32, 64 or 128, else
 * MORE_ERR_UNSUPPORTED.
 */
more_status more_route_unfused_tc(const void* X, const void* R1, const void* R2, int64_t N, int h, int r,
                                  int M, int k, int32_t* out_idx, float* out_gate,
                                  int32_t* out_expert_count, float* out_logits, void* scratch,
                                  size_t scratch_bytes, void* stream);

/*
 * more_route_unfused with no scratch argument: its scratch is a fixed array of
 * MORE_STATIC_SCRATCH_BYTES bytes inside the library, so the call allocates
 * nothing.  This entry point has no counterpart in the MoRE paper; it is for
 * callers that may not allocate device memory themselves, e.g. code running
 * under an external allocator or memory budget that forbids raw allocations,
 * or latency-critical paths where a cudaMalloc (which can synchronise the
 * device) is not acceptable.
 *   - Limit: a problem needing more than MORE_STATIC_SCRATCH_BYTES of scratch
 *     (more_route_unfused_scratch_bytes(N, r, M)) returns MORE_ERR_UNSUPPORTED.
 *   - The array exists once per device for as long as the library is loaded,
 *     on every device that loads it, whether or not this call is used.
 *   - The first call on a device looks up the array's device address (one
 *     cudaGetSymbolAddress with that device current); make that first call
 *     before starting any stream capture.  The address is kept for the life of
 *     the process: after a cudaDeviceReset of that device (which discards the
 *     library's module and the array with it) this entry point must not be
 *     called again in the same process.
 *   - All calls share the array and it keeps the last call's contents (every
 *     call overwrites the part it reads).  Calls that may overlap on the GPU
 *     (different streams, or different host threads without ordering) race on
 *     it and give wrong results; serialise them.
 * Arguments, validation and results are those of more_route_unfused.
 */
#define MORE_STATIC_SCRATCH_BYTES (32u << 20)
more_status more_route_unfused_static(const void* X, const void* R1, const void* R2, int64_t N, int h,
                                      int r, int M, int k, int32_t* out_idx, float* out_gate,
                                      int32_t* out_expert_count, float* out_logits, void* stream);

/*
 * The standard (full-rank) router, fused.  [MoRE App. H.3 "Fusing a standard MoE layer",
 * Figs. 20-22]  Per token x: the M logits x . W, the top-k in routing order, softmax gates over
 * the k and per-expert counts, with the same conventions and outputs as more_route.  W is
 * streamed past every 128-token tile one 128-expert tile (all h rows) at a time and the N x M
 * logits stay on chip.
 *   X  bf16 [N][h]   token hidden vectors
 *   W  bf16 [h][M]   router weight (one column per expert)
 * Logits are fp32 sums of the exact bf16 products (tensor cores), ranked as they are.
 * Requirements: those of more_route without r (h and M multiples of 8, 1 <= k <= M,
 * k <= MORE_KMAX, M <= MORE_MMAX, pointers 16-byte aligned; X, out_idx and out_gate may be
 * NULL only when N == 0).
 */
more_status more_route_fullrank(const void* X, const void* W, int64_t N, int h, int M, int k,
                                int32_t* out_idx, float* out_gate, int32_t* out_expert_count,
                                float* out_logits, void* stream);

/*
 * Self-test of the failure path.  Launches one bounded mbarrier wait that nothing completes, the
 * same bounded wait every persistent kernel of the library uses.  After its limit (4 s) the wait
 * gives up, records MORE_DEVERR_WAIT_TIMEOUT in the device error word and returns, leaving the
 * context usable.  *out_result (device int32, 4-byte aligned) is set to 2 when the wait gave up
 * (1 if it had completed).  Asynchronous on `stream`; read the outcome with more_device_status.
 * Returns MORE_ERR_INVALID_ARG for a NULL out_result.
 */
more_status more_selftest_wait_timeout(int32_t* out_result, void* stream);

/*
 * Synchronise `stream`, then return and clear the library's device error word
 * on the current device: MORE_OK if no kernel recorded an error since the last
 * call, MORE_ERR_DEVICE if one did (e.g. a bounded wait gave up), or
 * MORE_ERR_CUDA if synchronising failed.  `detail` (may be NULL) receives the
 * raw error word (an OR of the MORE_DEVERR_* bits).
 */
#define MORE_DEVERR_WAIT_TIMEOUT 0x1u  /* a bounded barrier wait ran out            */
#define MORE_DEVERR_BAD_CONFIG 0x2u    /* a kernel saw a configuration it rejects  */
#define MORE_DEVERR_BAD_INPUT 0x4u     /* an input value outside its range (skipped) */
more_status more_device_status(void* stream, uint32_t* detail);

/* Static description of a status code. */
const char* more_status_string(more_status status);

/*
 * Training forward of the router ("MoRE", App. F, Algorithm 2): everything more_route
 * returns, plus the statistics a load-balancing loss needs, computed over all M experts
 * (eqs. (6)-(8)):
 *   out_m[n]    = max_j l_nj                         fp32 [N], the token's largest logit
 *   out_Z[n]    = sum_j exp(l_nj - out_m[n])         fp32 [N], the softmax normalizer
 *                                                    relative to out_m (as Algorithm 2 keeps it)
 *   out_psum[i] = sum_n exp(l_ni - out_m[n]) / out_Z[n]
 *                                                    fp32 [M], the column sum of the full
 *                                                    softmax (eq. (7)); the call zeroes it first
 * The Switch loss of eq. (9) is then (M / N) sum_i f_i psum_i, with f_i = out_expert_count[i] / (N k).
 * The logits are those of more_route (z carried as the bf16 pair z_hi + z_lo, fp32
 * accumulation); the statistics use fp32 exp.  Requirements: as for more_route, plus
 * out_psum non-NULL, out_m and out_Z non-NULL unless N == 0, all three 16-byte aligned,
 * and M <= MORE_STATS_MMAX (else MORE_ERR_UNSUPPORTED).  Asynchronous on `stream`; runs
 * the routing kernel and then one statistics kernel; allocates nothing.
 */
#define MORE_STATS_MMAX 32768
more_status more_route_train(const void* X, const void* R1, const void* R2, int64_t N, int h, int r, int M,
                             int k, int32_t* out_idx, float* out_gate, int32_t* out_expert_count,
                             float* out_logits, float* out_m, float* out_Z, float* out_psum, void* stream);

/*
 * Dispatch bookkeeping after routing ("MoRE", App. E, Fig. 9, "Sort + Count"): the
 * (N, k) expert indices flattened to N*k slots s = n*k + j, stably sorted by expert, and
 * the per-expert offsets:
 *   out_offsets[e] = number of slots naming an expert below e     int32 [M + 1]
 *                    (out_offsets[M] = N*k)
 *   out_sorted[out_offsets[e] .. out_offsets[e + 1])               int32 [N*k]
 *                  = the slots naming expert e, in increasing order
 * idx: int32 [N][k] device, values in [0, M) (as more_route writes them; a value outside
 * is skipped and sets MORE_DEVERR_BAD_INPUT, and the offsets then count only valid slots).
 * scratch: device, 16-byte aligned, at least more_dispatch_scratch_bytes(N, k, M) bytes
 * (per-chunk histograms).  Requirements: N >= 0, 1 <= k <= MORE_KMAX, 1 <= M <= MORE_MMAX,
 * N*k < 2^31, out_offsets non-NULL, idx / out_sorted / scratch non-NULL unless N == 0, all
 * 16-byte aligned.  Asynchronous on `stream` (four kernels and a memset); allocates nothing.
 * The result does not depend on the launch configuration (a deterministic counting sort).
 */
size_t more_dispatch_scratch_bytes(int64_t N, int k, int M);
more_status more_dispatch(const int32_t* idx, int64_t N, int k, int M, int32_t* out_offsets,
                          int32_t* out_sorted, void* scratch, size_t scratch_bytes, void* stream);

/*
 * more_dispatch with an explicit kernel variant; same arguments, scratch and result.
 *   MORE_DISPATCH_GLOBAL: histograms of 2048-slot chunks in global memory;
 *   MORE_DISPATCH_SHARED: about two chunks per SM, each counted in a shared-memory histogram of
 *     M counters; requires M <= MORE_DISPATCH_SHARED_MMAX (else MORE_ERR_UNSUPPORTED).
 *   MORE_DISPATCH_AUTO:   the variant more_dispatch uses: SHARED when M <= MORE_DISPATCH_SHARED_MMAX
 *     (the faster of the two where both apply), GLOBAL otherwise.
 * Any other value returns MORE_ERR_INVALID_ARG.
 */
#define MORE_DISPATCH_SHARED_MMAX 32768
typedef enum more_dispatch_kernel {
  MORE_DISPATCH_AUTO = 0,
  MORE_DISPATCH_GLOBAL = 1,
  MORE_DISPATCH_SHARED = 2
} more_dispatch_kernel;
more_status more_dispatch_variant(const int32_t* idx, int64_t N, int k, int M, int32_t* out_offsets,
                                  int32_t* out_sorted, void* scratch, size_t scratch_bytes, int variant,
                                  void* stream);

/*
 * Backward of the router ("MoRE", App. F, F.2.2, Algorithm 3 and eqs. (10)-(12)), with z
 * recomputed from X (activation recompute), in fp32 on the CUDA cores.  With z = X R1,
 * l = z R2 (fp32) and P_ni = exp(l_ni - saved_m[n]) / saved_Z[n]:
 *   g_n      = sum_i pbar_i P_ni                                  (eq. (12))
 *   ybar_ni  = P_ni (pbar_i - g_n) + sum_j [top_idx[n][j] = i] top_vals_bar[n][j]
 *   out_Xbar  = ybar R2^T R1^T        fp32 [N][h]   (gradient with respect to X)
 *   out_R1bar = X^T (ybar R2^T)       fp32 [h][r]
 *   out_R2bar = z^T ybar              fp32 [r][M]
 *   out_g     = g                     fp32 [N]      (may be NULL)
 * Inputs (device):
 *   X, R1, R2       bf16 as for more_route;
 *   top_idx         int32 [N][k], the forward's selections (constants of the backward); a
 *                   value outside [0, M) is skipped and sets MORE_DEVERR_BAD_INPUT; a
 *                   repeated index receives each of its gradients;
 *   top_vals_bar    fp32 [N][k], the gradient on the selected logits; NULL for none (then
 *                   top_idx may be NULL);
 *   pbar            fp32 [M], the gradient on psum (the load-balancing term); NULL for none
 *                   (then g = 0 and saved_m / saved_Z are not read);
 *   saved_m, saved_Z  fp32 [N], as more_route_train returns them (Algorithm 2), required
 *                   when pbar is given and N > 0;
 *   scratch         at least more_route_backward_scratch_bytes(N, h, r, M) bytes (z, zbar, g
 *                   and per-split partial sums); its contents need no initialisation.
 * Every output is overwritten (not accumulated into).  Requirements: as for more_route
 * (h, M multiples of 8, r a multiple of 16 in [16, 128], 1 <= k <= MORE_KMAX, k <= M,
 * M <= MORE_MMAX, N < 2^31), out_R1bar and out_R2bar non-NULL, X / out_Xbar / scratch
 * non-NULL unless N == 0, every non-NULL pointer 16-byte aligned.  N == 0 zeroes out_R1bar
 * and out_R2bar.  Asynchronous on `stream` (five kernel launches); allocates nothing; the result
 * does not depend on the launch (fixed summation order, no atomics on the gradients).
 */
size_t more_route_backward_scratch_bytes(int64_t N, int h, int r, int M);
more_status more_route_backward(const void* X, const void* R1, const void* R2, int64_t N, int h, int r, int M,
                                int k, const int32_t* top_idx, const float* top_vals_bar, const float* pbar,
                                const float* saved_m, const float* saved_Z, float* out_Xbar, float* out_R1bar,
                                float* out_R2bar, float* out_g, void* scratch, size_t scratch_bytes,
                                void* stream);

/* MORE_ROUTE_ABI_VERSION of the built library. */
int more_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MORE_ROUTE_H */

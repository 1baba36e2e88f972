/*
 * Seeded synthetic inputs for the MoRE router: i.i.d. Gaussian tensors rounded
 * to bf16.  This module holds no routing arithmetic; it only draws numbers, so
 * both the CUDA path and the fp64 oracle can be fed bit-identical inputs.
 *
 * Generator (each step follows its published definition):
 *   - SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
 *     generators", OOPSLA 2014) used as a counter-based stream: draw i of a
 *     stream with key K is mix(K + (i + 1) * GAMMA), GAMMA = 0x9e3779b97f4a7c15.
 *   - uniform in (0, 1]: ((draw >> 11) + 1) * 2^-53.
 *   - Box–Muller (Box & Muller 1958): normal pair p uses draws 2p and 2p+1,
 *     rho = sqrt(-2 ln u1), theta = 2 pi u2; element 2p takes rho cos theta,
 *     element 2p+1 takes rho sin theta.
 *   - Stream key of (seed, tensor_id): mix(mix(seed) ^ (tensor_id + 1) * GAMMA).
 * Element (row, col) of a rows x cols tensor is normal number row * cols + col
 * of its stream, times sigma, in fp64.  With unit_rms_rows, each row is first
 * divided by its fp64 root-mean-square.  Rounding to bf16: fp64 -> fp32
 * (round to nearest), then fp32 -> bf16 (round to nearest, ties to even).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define SYN_GAMMA 0x9e3779b97f4a7c15ULL

static inline uint64_t syn_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
  return z ^ (z >> 31);
}

uint64_t synth_stream_key(uint64_t seed, uint64_t tensor_id) {
  return syn_mix(syn_mix(seed) ^ ((tensor_id + 1) * SYN_GAMMA));
}

static inline uint64_t syn_draw(uint64_t key, uint64_t i) {
  return syn_mix(key + (i + 1) * SYN_GAMMA);
}

static inline double syn_u01(uint64_t x) {
  return (double)((x >> 11) + 1) * 0x1.0p-53;
}

/* Normal number j of the stream with the given key. */
double synth_normal_at(uint64_t key, uint64_t j) {
  uint64_t p = j >> 1;
  double u1 = syn_u01(syn_draw(key, 2 * p));
  double u2 = syn_u01(syn_draw(key, 2 * p + 1));
  double rho = sqrt(-2.0 * log(u1));
  double theta = 2.0 * M_PI * u2;
  return (j & 1) ? rho * sin(theta) : rho * cos(theta);
}

uint16_t synth_f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7fffu + lsb;
  return (uint16_t)(u >> 16);
}

typedef struct {
  uint64_t key;
  int64_t row_begin, row_end; /* absolute rows of the conceptual tensor */
  int64_t out_row0;           /* first row written by the whole call */
  int64_t cols;
  double sigma;
  int unit_rms_rows;
  uint16_t* out;
} syn_job;

static void* syn_worker(void* arg) {
  syn_job* jb = (syn_job*)arg;
  double* row = (double*)malloc(sizeof(double) * (size_t)jb->cols);
  for (int64_t r = jb->row_begin; r < jb->row_end; ++r) {
    uint64_t base = (uint64_t)r * (uint64_t)jb->cols;
    /* draw whole pairs; the column count may be odd */
    for (int64_t c = 0; c < jb->cols; ++c) row[c] = synth_normal_at(jb->key, base + (uint64_t)c);
    double scale = jb->sigma;
    if (jb->unit_rms_rows) {
      double ss = 0.0;
      for (int64_t c = 0; c < jb->cols; ++c) ss += row[c] * row[c];
      double rms = sqrt(ss / (double)jb->cols);
      scale = jb->sigma / rms;
    }
    uint16_t* o = jb->out + (size_t)(r - jb->out_row0) * (size_t)jb->cols;
    for (int64_t c = 0; c < jb->cols; ++c) o[c] = synth_f32_to_bf16((float)(row[c] * scale));
  }
  free(row);
  return NULL;
}

/*
 * Fill out[0 .. n_rows*cols) with rows [row_begin, row_begin + n_rows) of the
 * tensor (seed, tensor_id) of width cols.  Returns 0 on success.
 */
int synth_normal_bf16(uint64_t seed, uint64_t tensor_id, int64_t row_begin, int64_t n_rows,
                      int64_t cols, double sigma, int unit_rms_rows, uint16_t* out, int nthreads) {
  if (n_rows < 0 || cols <= 0 || row_begin < 0 || (n_rows > 0 && !out)) return 1;
  if (n_rows == 0) return 0;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if ((int64_t)nthreads > n_rows) nthreads = (int)n_rows;
  uint64_t key = synth_stream_key(seed, tensor_id);
  pthread_t th[256];
  int joined[256];
  syn_job jobs[256];
  int64_t per = (n_rows + nthreads - 1) / nthreads;
  int started = 0;
  for (int t = 0; t < nthreads; ++t) {
    int64_t b = row_begin + (int64_t)t * per;
    int64_t e = b + per;
    if (e > row_begin + n_rows) e = row_begin + n_rows;
    if (b >= e) break;
    jobs[t] = (syn_job){key, b, e, row_begin, cols, sigma, unit_rms_rows, out};
    joined[t] = 0;
    if (pthread_create(&th[t], NULL, syn_worker, &jobs[t]) != 0) {
      syn_worker(&jobs[t]);
      joined[t] = 1;
    }
    started = t + 1;
  }
  for (int t = 0; t < started; ++t)
    if (!joined[t]) pthread_join(th[t], NULL);
  return 0;
}

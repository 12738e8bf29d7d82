/*
 * Seeded, counter-based synthetic input generator.
 *
 * This module draws random numbers and nothing else: it holds none of the
 * recurrence's arithmetic (no gates, no normalisation of keys as the method
 * does it, no state update).  Both the CUDA path's tests/bench and the CPU
 * oracle's tests take their inputs from here, so that any slice of a large
 * workload can be regenerated on the host without storing it.
 *
 * Generator (published methods, restated):
 *   - SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
 *     generators", OOPSLA 2014; constants as in Vigna's public-domain
 *     splitmix64.c) is used as a counter-based hash: word(c) = mix(base + c).
 *   - uniform in (0,1): ((word >> 11) + 0.5) * 2^-53.
 *   - standard normal by the Box-Muller transform (Box & Muller, 1958):
 *     z = sqrt(-2 ln u1) * cos(2 pi u2), with u1, u2 drawn from the two
 *     counters 2i and 2i+1 of the element's stream.
 *   - a uniformly random unit vector (Marsaglia/Muller): a vector of d
 *     standard normals divided by its Euclidean length (in double).
 *
 * Stream of tensor `tid` under `seed`: base = mix(mix(seed) + tid).
 * Element i of that stream is a pure function of (seed, tid, i).
 */
#include <math.h>
#include <stdint.h>
#include <pthread.h>
#include <stdlib.h>

static inline uint64_t sm64_mix(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ULL;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t stream_base(uint64_t seed, uint64_t tid) {
  return sm64_mix(sm64_mix(seed) + tid);
}

static inline double to_unit(uint64_t w) {
  return ((double)(w >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

static inline double normal_at(uint64_t base, uint64_t i) {
  const double two_pi = 6.283185307179586476925286766559;
  double u1 = to_unit(sm64_mix(base + 2 * i));
  double u2 = to_unit(sm64_mix(base + 2 * i + 1));
  return sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
}

uint64_t synth_mix(uint64_t x) { return sm64_mix(x); }

uint64_t synth_word(uint64_t seed, uint64_t tid, uint64_t c) {
  return sm64_mix(stream_base(seed, tid) + c);
}

double synth_normal_one(uint64_t seed, uint64_t tid, uint64_t i) {
  return normal_at(stream_base(seed, tid), i);
}

/* ---- threaded fills ---------------------------------------------------- */

typedef struct {
  uint64_t base;
  int64_t lo, hi;      /* element (or row) range [lo, hi) of this worker   */
  int64_t first;       /* global index of out[0]                           */
  int64_t d;           /* row length for unit rows                         */
  double mean, std;
  float *out;
  int kind;            /* 0 = normal, 1 = unit rows                        */
} job_t;

static void *run_job(void *p) {
  job_t *j = (job_t *)p;
  if (j->kind == 0) {
    for (int64_t e = j->lo; e < j->hi; ++e)
      j->out[e] = (float)(j->mean + j->std * normal_at(j->base, (uint64_t)(j->first + e)));
  } else {
    double *tmp = (double *)malloc(sizeof(double) * (size_t)j->d);
    for (int64_t r = j->lo; r < j->hi; ++r) {
      uint64_t row0 = (uint64_t)((j->first + r) * j->d);
      double ss = 0.0;
      for (int64_t c = 0; c < j->d; ++c) {
        tmp[c] = normal_at(j->base, row0 + (uint64_t)c);
        ss += tmp[c] * tmp[c];
      }
      double inv = ss > 0.0 ? 1.0 / sqrt(ss) : 0.0;
      for (int64_t c = 0; c < j->d; ++c) j->out[r * j->d + c] = (float)(tmp[c] * inv);
    }
    free(tmp);
  }
  return NULL;
}

static void run_threads(job_t proto, int64_t n, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (n < 4096) nthreads = 1;
  pthread_t th[256];
  job_t jobs[256];
  int64_t per = (n + nthreads - 1) / nthreads;
  int started = 0;
  for (int t = 0; t < nthreads; ++t) {
    jobs[t] = proto;
    jobs[t].lo = t * per;
    jobs[t].hi = (t + 1) * per < n ? (t + 1) * per : n;
    if (jobs[t].lo >= jobs[t].hi) break;
    if (t == 0) continue;
    pthread_create(&th[t], NULL, run_job, &jobs[t]);
    started = t;
  }
  if (jobs[0].lo < jobs[0].hi) run_job(&jobs[0]);
  for (int t = 1; t <= started; ++t) pthread_join(th[t], NULL);
}

/* out[e] = mean + std * N(0,1)[first + e], e in [0, count) */
void synth_fill_normal(uint64_t seed, uint64_t tid, int64_t first, int64_t count,
                       double mean, double std, float *out, int nthreads) {
  job_t j = {stream_base(seed, tid), 0, 0, first, 1, mean, std, out, 0};
  run_threads(j, count, nthreads);
}

/* rows [first_row, first_row + nrows) of unit vectors of length d; row r uses
 * the normals at stream indices r*d .. r*d + d - 1. */
void synth_fill_unit_rows(uint64_t seed, uint64_t tid, int64_t first_row, int64_t nrows,
                          int64_t d, float *out, int nthreads) {
  job_t j = {stream_base(seed, tid), 0, 0, first_row, d, 0.0, 1.0, out, 1};
  run_threads(j, nrows, nthreads);
}

/*
 * Seeded synthetic inputs for the tree-indexed sparse decode path.
 *
 * This module only draws numbers: it holds none of the method's arithmetic
 * (no means, no scores, no softmax).  Tests, the benchmark and the smoke
 * check all take their inputs from here, so the CUDA path and the fp64
 * oracle see the same bytes.
 *
 * Generator: counter-based.  Element c of stream s under seed S is
 *     u(S, s, c) = top 53 bits of mix64(key(S, s) + (c + 1) * GOLDEN) / 2^53
 * where mix64 is the splitmix64 output function (Steele, Lea, Flood,
 * "Fast splittable pseudorandom number generators", OOPSLA 2014).
 * Normals come from the Box-Muller transform on the pair (2j, 2j+1):
 *     r = sqrt(-2 ln(1 - u0)), th = 2 pi u1, z_{2j} = r cos th, z_{2j+1} = r sin th.
 * Counter-based drawing lets every thread fill its own slice independently,
 * and makes a tensor's values independent of how large it is allocated.
 *
 * Rounding to storage types is round-to-nearest-even from fp64 directly
 * (no double rounding through fp32 for bf16).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t stream) {
  return mix64(seed * GOLDEN + mix64(stream ^ 0x632BE59BD9B4E019ULL));
}

static inline double unit_u01(uint64_t key, uint64_t ctr) {
  uint64_t r = mix64(key + (ctr + 1ULL) * GOLDEN);
  return (double)(r >> 11) * (1.0 / 9007199254740992.0); /* [0, 1) */
}

static inline double normal_at(uint64_t key, uint64_t idx) {
  uint64_t j = idx >> 1;
  double u0 = unit_u01(key, 2 * j);
  double u1 = unit_u01(key, 2 * j + 1);
  double r = sqrt(-2.0 * log(1.0 - u0)); /* 1 - u0 in (0, 1] */
  double th = 6.283185307179586476925286766559 * u1;
  return (idx & 1) ? r * sin(th) : r * cos(th);
}

/* fp64 -> bf16 bits, round to nearest even, straight from the fp64 value. */
uint16_t synth_f64_to_bf16_bits(double x) {
  uint64_t b;
  memcpy(&b, &x, 8);
  uint64_t sign = b >> 63;
  uint64_t mag = b & 0x7FFFFFFFFFFFFFFFULL;
  if (mag >= 0x7FF0000000000000ULL) { /* inf / nan */
    if (mag > 0x7FF0000000000000ULL) return (uint16_t)((sign << 15) | 0x7FC0);
    return (uint16_t)((sign << 15) | 0x7F80);
  }
  /* Keep 7 explicit mantissa bits of the double (bits 45..51), RNE on the rest. */
  uint64_t keep = mag >> 45;
  uint64_t rem = mag & ((1ULL << 45) - 1);
  uint64_t half = 1ULL << 44;
  if (rem > half || (rem == half && (keep & 1))) keep++;
  uint64_t r = keep << 45;
  double y;
  memcpy(&y, &r, 8);
  float f = (float)y; /* exact: 8 significant bits, exponent range checked below */
  uint32_t fb;
  memcpy(&fb, &f, 4);
  if ((fb & 0xFFFF) != 0) {
    /* Value fell in the fp32 subnormal range and was rounded again; redo it
       with an fp32-level RNE on the original value (values this small never
       occur in the recipes, but keep the function total). */
    float g = (float)x;
    uint32_t gb;
    memcpy(&gb, &g, 4);
    uint32_t lsb = (gb >> 16) & 1;
    gb += 0x7FFF + lsb;
    return (uint16_t)(gb >> 16);
  }
  return (uint16_t)((sign << 15) | (fb >> 16));
}

typedef struct {
  uint64_t key, offset;
  int64_t begin, end;
  double mean, std;
  int kind; /* 0 f64, 1 f32, 2 bf16, 3 uniform f64 */
  void *out;
} job_t;

static void *run_job(void *p) {
  job_t *j = (job_t *)p;
  for (int64_t i = j->begin; i < j->end; ++i) {
    uint64_t c = j->offset + (uint64_t)i;
    double v;
    if (j->kind == 3) {
      v = unit_u01(j->key, c);
    } else {
      v = j->mean + j->std * normal_at(j->key, c);
    }
    switch (j->kind) {
      case 0:
      case 3: ((double *)j->out)[i] = v; break;
      case 1: ((float *)j->out)[i] = (float)v; break;
      default: ((uint16_t *)j->out)[i] = synth_f64_to_bf16_bits(v); break;
    }
  }
  return NULL;
}

static int fill(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, double mean, double std,
                int kind, void *out, int nthreads) {
  if (n <= 0) return 0;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if ((int64_t)nthreads > n / 65536 + 1) nthreads = (int)(n / 65536 + 1);
  uint64_t key = stream_key(seed, stream);
  pthread_t th[256];
  int started[256];
  job_t jobs[256];
  int64_t per = (n + nthreads - 1) / nthreads;
  for (int t = 0; t < nthreads; ++t) {
    jobs[t].key = key;
    jobs[t].offset = offset;
    jobs[t].begin = (int64_t)t * per < n ? (int64_t)t * per : n;
    jobs[t].end = jobs[t].begin + per < n ? jobs[t].begin + per : n;
    jobs[t].mean = mean;
    jobs[t].std = std;
    jobs[t].kind = kind;
    jobs[t].out = out;
    started[t] = 0;
  }
  for (int t = 1; t < nthreads; ++t)
    started[t] = pthread_create(&th[t], NULL, run_job, &jobs[t]) == 0;
  run_job(&jobs[0]);
  for (int t = 1; t < nthreads; ++t) {
    if (started[t]) pthread_join(th[t], NULL);
    else run_job(&jobs[t]);
  }
  return 0;
}

/* out[i] = mean + std * N(0,1) at counters offset + i, as fp64. */
int synth_normal_f64(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, double mean,
                     double std, double *out, int nthreads) {
  return fill(seed, stream, offset, n, mean, std, 0, out, nthreads);
}
/* Same values rounded RNE to fp32. */
int synth_normal_f32(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, double mean,
                     double std, float *out, int nthreads) {
  return fill(seed, stream, offset, n, mean, std, 1, out, nthreads);
}
/* Same values rounded RNE to bf16 (bit patterns). */
int synth_normal_bf16(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, double mean,
                      double std, uint16_t *out, int nthreads) {
  return fill(seed, stream, offset, n, mean, std, 2, out, nthreads);
}
/* Uniform [0,1) doubles at counters offset + i. */
int synth_uniform_f64(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, double *out,
                      int nthreads) {
  return fill(seed, stream, offset, n, 0.0, 1.0, 3, out, nthreads);
}

/* Round an fp64 array to bf16 bits / fp32 (RNE). */
void synth_round_bf16(const double *in, int64_t n, uint16_t *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = synth_f64_to_bf16_bits(in[i]);
}
void synth_round_f32(const double *in, int64_t n, float *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = (float)in[i];
}

/*
 * Keys with a low-rank positional drift, rows [0, rows) of one unit:
 *   out[t*d + k] = round( N(0,1)[counter offset + t*d + k]
 *                         + amp * sum_j A[k*r + j] * sin(2 pi t / P[j] + phi[j]) )
 * rounded RNE to bf16 (out_bf16 != NULL) or fp32 (out_f32).
 */
typedef struct {
  uint64_t key, offset;
  int64_t t0, t1, d, r;
  double amp;
  const double *A, *P, *phi;
  uint16_t *ob;
  float *of;
} drift_job_t;

static void *run_drift(void *p) {
  drift_job_t *j = (drift_job_t *)p;
  double f[64];
  for (int64_t t = j->t0; t < j->t1; ++t) {
    for (int64_t q = 0; q < j->r; ++q)
      f[q] = sin(6.283185307179586476925286766559 * (double)t / j->P[q] + j->phi[q]);
    for (int64_t k = 0; k < j->d; ++k) {
      double s = 0.0;
      for (int64_t q = 0; q < j->r; ++q) s += j->A[k * j->r + q] * f[q];
      double v = normal_at(j->key, j->offset + (uint64_t)(t * j->d + k)) + j->amp * s;
      if (j->ob) j->ob[t * j->d + k] = synth_f64_to_bf16_bits(v);
      else j->of[t * j->d + k] = (float)v;
    }
  }
  return NULL;
}

int synth_drift_keys(uint64_t seed, uint64_t stream, uint64_t offset, int64_t rows, int64_t d,
                     int64_t r, double amp, const double *A, const double *P, const double *phi,
                     uint16_t *out_bf16, float *out_f32, int nthreads) {
  if (rows <= 0) return 0;
  if (r > 64) return -1;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (nthreads > rows / 256 + 1) nthreads = (int)(rows / 256 + 1);
  pthread_t th[256];
  int started[256];
  drift_job_t jobs[256];
  int64_t per = (rows + nthreads - 1) / nthreads;
  for (int t = 0; t < nthreads; ++t) {
    drift_job_t *j = &jobs[t];
    j->key = stream_key(seed, stream);
    j->offset = offset;
    j->t0 = (int64_t)t * per < rows ? (int64_t)t * per : rows;
    j->t1 = j->t0 + per < rows ? j->t0 + per : rows;
    j->d = d;
    j->r = r;
    j->amp = amp;
    j->A = A;
    j->P = P;
    j->phi = phi;
    j->ob = out_bf16;
    j->of = out_f32;
    started[t] = 0;
  }
  for (int t = 1; t < nthreads; ++t) started[t] = pthread_create(&th[t], NULL, run_drift, &jobs[t]) == 0;
  run_drift(&jobs[0]);
  for (int t = 1; t < nthreads; ++t) {
    if (started[t]) pthread_join(th[t], NULL);
    else run_drift(&jobs[t]);
  }
  return 0;
}

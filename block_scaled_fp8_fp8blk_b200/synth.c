/*
 * Seeded synthetic inputs for the block-FP8 linear layer.
 *
 * This file only draws random numbers. It holds none of the layer's own
 * arithmetic (no FP8 or BF16 coding, no scaling, no matrix products): it
 * writes float32 values that the caller rounds to BF16 with a library
 * conversion. Both the CUDA path and the CPU oracle consume the same drawn
 * tensors, so this is the only code the two sides share.
 *
 * Generator: counter-based splitmix64 (Steele, Lea and Flood, "Fast
 * splittable pseudorandom number generators", OOPSLA 2014) keyed by
 * (seed, stream), mapped to uniforms on (0, 1) and to normals by the
 * Box-Muller transform (Box and Muller, 1958). Element i of a stream
 * depends only on (key, i), so results do not depend on the thread count.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>

#define SYNTH_GOLDEN 0x9E3779B97F4A7C15ULL

static uint64_t synth_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* Stream key for (seed, stream): mixed so nearby seeds decorrelate. */
uint64_t synth_key(uint64_t seed, uint64_t stream) {
  return synth_mix(seed * 16ULL + stream + SYNTH_GOLDEN);
}

/* Uniform draw number idx of a stream, in (0, 1), 53-bit resolution. */
static double synth_u01(uint64_t key, uint64_t idx) {
  uint64_t z = synth_mix(key + (idx + 1ULL) * SYNTH_GOLDEN);
  return ((double)(z >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

/* Standard normal number i of a stream: pairs of uniforms (2j, 2j+1) give
 * the cosine branch for even i and the sine branch for odd i. */
static double synth_n01(uint64_t key, uint64_t i) {
  uint64_t j = i >> 1;
  double u1 = synth_u01(key, 2 * j), u2 = synth_u01(key, 2 * j + 1);
  double r = sqrt(-2.0 * log(u1));
  double t = 6.283185307179586476925286766559 * u2;
  return (i & 1) ? r * sin(t) : r * cos(t);
}

void synth_uniform(uint64_t key, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = synth_u01(key, (uint64_t)i);
}

void synth_normal_vec(uint64_t key, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = synth_n01(key, (uint64_t)i);
}

typedef struct {
  uint64_t key;
  int64_t rows, cols, r0, r1;
  double stddev;
  const double* row_gain;
  const double* col_gain;
  float* out;
} synth_job;

static void* synth_matrix_worker(void* p) {
  const synth_job* j = (const synth_job*)p;
  for (int64_t r = j->r0; r < j->r1; ++r) {
    double g = j->stddev * (j->row_gain ? j->row_gain[r] : 1.0);
    float* o = j->out + r * j->cols;
    uint64_t base = (uint64_t)r * (uint64_t)j->cols;
    for (int64_t c = 0; c < j->cols; ++c) {
      double v = g * synth_n01(j->key, base + (uint64_t)c);
      if (j->col_gain) v *= j->col_gain[c];
      o[c] = (float)v;
    }
  }
  return 0;
}

/* out[r][c] = float(stddev * row_gain[r] * col_gain[c] * normal(key, r*cols+c)).
 * row_gain / col_gain may be NULL (all ones). Rows are split over nthreads. */
void synth_matrix(uint64_t key, int64_t rows, int64_t cols, double stddev,
                  const double* row_gain, const double* col_gain, float* out,
                  int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (rows < nthreads) nthreads = rows > 0 ? (int)rows : 1;
  pthread_t th[256];
  int joinable[256];
  synth_job jobs[256];
  int64_t per = (rows + nthreads - 1) / nthreads;
  int started = 0;
  for (int t = 0; t < nthreads; ++t) {
    int64_t r0 = t * per, r1 = r0 + per;
    if (r1 > rows) r1 = rows;
    if (r0 >= r1) break;
    synth_job jb = {key, rows, cols, r0, r1, stddev, row_gain, col_gain, out};
    jobs[t] = jb;
    joinable[t] = pthread_create(&th[t], 0, synth_matrix_worker, &jobs[t]) == 0;
    if (!joinable[t]) synth_matrix_worker(&jobs[t]);
    started = t + 1;
  }
  for (int t = 0; t < started; ++t)
    if (joinable[t]) pthread_join(th[t], 0);
}

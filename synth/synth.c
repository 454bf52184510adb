/*
 * Seeded synthetic inputs for the weight-only quantized linear.
 *
 * This file holds no arithmetic of the method itself (no quantizer, no
 * dequantizer, no dot product).  It only draws the dense fp32 weight matrix,
 * the bf16 activations and the bf16 bias that both the CPU oracle and the
 * CUDA path consume, so that the two sides see identical inputs.
 *
 * Random numbers
 *   uniform i of stream (seed, tensor_id):
 *       key  = (seed << 16) | tensor_id
 *       z    = SplitMix64 output i  = mix(key + (i + 1) * 0x9E3779B97F4A7C15)
 *       u    = ((z >> 11) + 0.5) * 2^-53            (strictly inside (0, 1))
 *   normal j: Box-Muller on the uniform pair (2*(j/2), 2*(j/2)+1),
 *       r = sqrt(-2 ln u1), theta = 2 pi u2, even j -> r cos theta,
 *       odd j -> r sin theta.
 *   Student-t(5) element e: normals 6e .. 6e+5, t = Z / sqrt(chi2 / 5) with
 *       Z = normal 6e and chi2 the sum of the squares of the other five.
 * Everything is drawn in fp64 and cast once at the end (fp32 round-to-nearest-
 * even for weights, bf16 round-to-nearest-even for activations and bias).
 *
 * Every element is a pure function of its index, so the loops are split
 * across threads without changing any value.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t tensor_id) {
  return (seed << 16) | (tensor_id & 0xFFFFULL);
}

static inline double uniform_at(uint64_t key, uint64_t i) {
  uint64_t z = mix64(key + (i + 1) * GOLDEN);
  return ((double)(z >> 11) + 0.5) * 0x1.0p-53;
}

static inline double normal_at(uint64_t key, uint64_t j) {
  uint64_t p = j >> 1;
  double u1 = uniform_at(key, 2 * p);
  double u2 = uniform_at(key, 2 * p + 1);
  double r = sqrt(-2.0 * log(u1));
  double th = 6.283185307179586476925286766559 * u2;
  return (j & 1) ? r * sin(th) : r * cos(th);
}

static inline double student5_at(uint64_t key, uint64_t e) {
  double z = normal_at(key, 6 * e);
  double chi2 = 0.0;
  for (int i = 1; i <= 5; ++i) {
    double n = normal_at(key, 6 * e + i);
    chi2 += n * n;
  }
  return z / sqrt(chi2 / 5.0);
}

/* fp64 -> bf16 bits, round to nearest even, one rounding.  The double is first
 * cut to fp32 with round-to-odd (truncate, then set the last bit when inexact);
 * fp32 keeps 16 more bits than bf16, so the final even rounding is exact. */
static inline uint16_t f64_to_bf16(double v) {
  if (isnan(v)) return 0x7FC0;
  float t = (float)v;
  if (isinf(t) && !isinf(v)) {
    /* overflowed fp32 by rounding: the value is beyond bf16's range too */
    return (uint16_t)(signbit(v) ? 0xFF80 : 0x7F80);
  }
  uint32_t b;
  memcpy(&b, &t, 4);
  if (!isinf(t) && (double)t != v) {
    if (fabs((double)t) > fabs(v)) b -= 1; /* step back toward zero */
    b |= 1u;                               /* sticky bit */
  }
  uint32_t lsb = (b >> 16) & 1u;
  uint32_t r = b + 0x7FFFu + lsb;
  return (uint16_t)(r >> 16);
}

/* Distinct positions drawn without replacement from [0, range): draw
 * uniform i = 0, 1, 2, ... of stream (seed, tensor_id), map it to
 * floor(u * range) and keep it when it was not drawn before. */
int synth_distinct_positions(uint64_t seed, uint64_t tensor_id, int64_t range,
                             int64_t count, int64_t* out) {
  if (range <= 0 || count < 0 || count > range) return 1;
  uint8_t* seen = (uint8_t*)calloc((size_t)((range + 7) / 8), 1);
  if (!seen) return 2;
  uint64_t key = stream_key(seed, tensor_id);
  int64_t got = 0;
  uint64_t i = 0;
  while (got < count) {
    double u = uniform_at(key, i++);
    int64_t p = (int64_t)(u * (double)range);
    if (p >= range) p = range - 1;
    if (!(seen[p >> 3] & (1u << (p & 7)))) {
      seen[p >> 3] |= (uint8_t)(1u << (p & 7));
      out[got++] = p;
    }
  }
  free(seen);
  return 0;
}

/* Dense weight W[N, K] as fp32.
 *   dist 0: sigma * N(0, 1);   dist 1: sigma * Student-t(5).
 *   outlier_count > 0: that many distinct positions (stream tensor_id 4)
 *   are multiplied by outlier_mult before the fp32 cast. */
int synth_weight_f32(uint64_t seed, int64_t N, int64_t K, int dist, double sigma,
                     int64_t outlier_count, double outlier_mult, float* out) {
  const uint64_t tid_w = 1, tid_out = 4;
  if (N <= 0 || K <= 0) return 1;
  uint64_t key = stream_key(seed, tid_w);
  int64_t total = N * K;
#pragma omp parallel for schedule(static)
  for (int64_t e = 0; e < total; ++e) {
    double v = dist == 1 ? student5_at(key, (uint64_t)e) : normal_at(key, (uint64_t)e);
    out[e] = (float)(sigma * v);
  }
  if (outlier_count > 0) {
    int64_t* pos = (int64_t*)malloc(sizeof(int64_t) * (size_t)outlier_count);
    if (!pos) return 2;
    int rc = synth_distinct_positions(seed, tid_out, total, outlier_count, pos);
    if (rc) { free(pos); return rc; }
    for (int64_t i = 0; i < outlier_count; ++i) {
      int64_t e = pos[i];
      double v = dist == 1 ? student5_at(key, (uint64_t)e) : normal_at(key, (uint64_t)e);
      out[e] = (float)(outlier_mult * sigma * v);
    }
    free(pos);
  }
  return 0;
}

/* Activations X[M, K] as bf16 bits: sigma * N(0, 1) (stream tensor_id 2).
 * channel_count > 0: that many distinct columns k (stream tensor_id 5) are
 * multiplied by channel_mult before the bf16 cast. */
int synth_act_bf16(uint64_t seed, int64_t M, int64_t K, double sigma,
                   int64_t channel_count, double channel_mult, uint16_t* out) {
  const uint64_t tid_x = 2, tid_ch = 5;
  if (M < 0 || K <= 0) return 1;
  uint64_t key = stream_key(seed, tid_x);
  double* mult = (double*)malloc(sizeof(double) * (size_t)K);
  if (!mult) return 2;
  for (int64_t k = 0; k < K; ++k) mult[k] = 1.0;
  if (channel_count > 0) {
    int64_t* pos = (int64_t*)malloc(sizeof(int64_t) * (size_t)channel_count);
    if (!pos) { free(mult); return 2; }
    int rc = synth_distinct_positions(seed, tid_ch, K, channel_count, pos);
    if (rc) { free(pos); free(mult); return rc; }
    for (int64_t i = 0; i < channel_count; ++i) mult[pos[i]] = channel_mult;
    free(pos);
  }
  int64_t total = M * K;
#pragma omp parallel for schedule(static)
  for (int64_t e = 0; e < total; ++e) {
    double v = sigma * normal_at(key, (uint64_t)e) * mult[e % K];
    out[e] = f64_to_bf16(v);
  }
  free(mult);
  return 0;
}

/* Bias[N] as bf16 bits: sigma * N(0, 1) (stream tensor_id 3). */
int synth_bias_bf16(uint64_t seed, int64_t N, double sigma, uint16_t* out) {
  const uint64_t tid_b = 3;
  if (N <= 0) return 1;
  uint64_t key = stream_key(seed, tid_b);
  for (int64_t n = 0; n < N; ++n) out[n] = f64_to_bf16(sigma * normal_at(key, (uint64_t)n));
  return 0;
}

/* Raw streams, exposed so that tests can check the generator itself. */
int synth_uniform_f64(uint64_t seed, uint64_t tensor_id, int64_t start, int64_t n, double* out) {
  uint64_t key = stream_key(seed, tensor_id);
  for (int64_t i = 0; i < n; ++i) out[i] = uniform_at(key, (uint64_t)(start + i));
  return 0;
}

int synth_normal_f64(uint64_t seed, uint64_t tensor_id, int64_t start, int64_t n, double* out) {
  uint64_t key = stream_key(seed, tensor_id);
  for (int64_t i = 0; i < n; ++i) out[i] = normal_at(key, (uint64_t)(start + i));
  return 0;
}

int synth_student5_f64(uint64_t seed, uint64_t tensor_id, int64_t start, int64_t n, double* out) {
  uint64_t key = stream_key(seed, tensor_id);
  for (int64_t i = 0; i < n; ++i) out[i] = student5_at(key, (uint64_t)(start + i));
  return 0;
}

uint64_t synth_splitmix64(uint64_t key, uint64_t i) { return mix64(key + (i + 1) * GOLDEN); }

int synth_f64_to_bf16(const double* in, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = f64_to_bf16(in[i]);
  return 0;
}

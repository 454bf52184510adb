/*
 * ORACLE - test infrastructure, not part of the library.
 *
 * A plain, slow CPU statement of what the weight-only quantized linear
 * computes:  Y[M,N] = X[M,K] . dequant(Wq)[N,K]^T + bias,  X/Y/bias in bf16.
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg may
 * load this file; the CUDA library never does, and the two share no code.
 *
 * Sources (the pages print no formula for any quantizer, so every format
 * below is the plainest reading the pages support; each reading is named):
 *  - piper-kernels README, "ConvRot INT8": group-wise INT8 weight, group 256,
 *    weight shape [out_features, in_features].
 *  - Mamba-2 paired-nibble state file, pack/dequant helpers: symmetric RTN
 *    with scale = amax/qmax, clamp to +-qmax, half-precision scales, element
 *    2i in the low nibble and 2i+1 in the high nibble, signed nibble
 *    v = n - 16*[n > 7].
 *  - auto-round-lib README, section 1 "Linear": INT4/INT8 weight-only GEMM,
 *    sym and asym (zero-point) variants, per-group scales along K.
 *  - OrbitQuant packed matmul card, "API"/"Inputs": uint8 row-major packed
 *    codebook indices, per-row norms (bf16 on CUDA), fp32 Lloyd-Max
 *    centroids [2**bits].
 *  - Petit README, "Features"/"Known limitations": NVFP4 weights, positive
 *    scales, no negative-zero codes.
 *  - NVFP4 itself: E2M1 values, one E4M3 scale per 16 consecutive K
 *    elements, one fp32 tensor scale (format definition).
 *  - Petit README, "Features": MXFP4 weights beside NVFP4.  MXFP4 itself
 *    (the OCP microscaling format definition): E2M1 values, one E8M0 scale
 *    (a power of two, 2^(e-127), e = 255 is NaN) per 32 consecutive K
 *    elements, no tensor scale.
 *  - auto-round-lib README, section 1 "Supported Data Types": INT1-INT8
 *    weights, sym / asym; the INT2 member here is symmetric like INT4/INT8.
 *  - auto-round-lib README, section 1 "Supported Data Types": FP8 (E4M3,
 *    E5M2) weights with an FP32 scale, BF16 / FP32 compute (QuantLinearFP8,
 *    the FP8 weight-only linear).
 *
 * Readings taken where the pages are silent:
 *  - rounding of w/s to an integer: round half to even;
 *  - a scale is rounded once to bf16 and w is divided by the stored scale;
 *  - an all-zero group / row / block gets scale 0 and code 0;
 *  - INT4 emits [-7, 7], INT8 emits [-127, 127], INT2 emits [-1, 1],
 *    INT3 emits [-3, 3]
 *    (qmax = 2^(bits-1) - 1 for every width; -2^(bits-1) decodes but is
 *    never written);
 *  - asym INT4: lo = min(0, min w), hi = max(0, max w), s = bf16((hi-lo)/15),
 *    z = clamp(rne(-lo/s), 0, 15), q = clamp(rne(w/s) + z, 0, 15),
 *    dq = (q - z) * s;
 *  - codebook: norm = bf16(||w_row||_2 / sqrt(K)), idx = argmin_j
 *    |w/norm - c_j| with ties to the lower j, dq = fp32(c[idx] * norm);
 *  - NVFP4: ts = fp32(amax / (6*448)), sb = E4M3_rne_satfinite(amax_b /
 *    (6*ts)), q = E2M1_rne_sat(w / (e4m3(sb)*ts)), -0 written as +0,
 *    dq = fp32(e2m1(q) * e4m3(sb) * ts);  the tensor scale multiplies.
 *  - MXFP4: the microscaling recipe: shared exponent = floor(log2(amax_b))
 *    - 2 (2 = the largest E2M1 exponent, since 6 = 1.5 * 2^2), clamped to
 *    [-127, 127]; e = shared exponent + 127; q = E2M1_rne_sat(w / 2^(e-127))
 *    (|w| / 2^(e-127) in [4, 8) at the block's largest element, so values
 *    above 6 saturate), -0 written as +0; an all-zero block gets e = 0 and
 *    codes 0; dq = fp32(e2m1(q) * 2^(e-127)) (exact).
 *  - FP8 E4M3: one fp32 scale per group of G along K (the grouping of the
 *    INT formats), s = fp32(amax_g / 448) (448 = the largest finite E4M3),
 *    q = E4M3_rne_satfinite(w / s) with the sign of w, -0 written as +0;
 *    an all-zero group gets s = 0 and codes 0; dq = fp32(e4m3(q) * s)
 *    (one rounding of the exact product).
 *  - FP8 E5M2: the same with 57344 (the largest finite E5M2) in place of 448
 *    and E5M2_rne_satfinite; dq = fp32(e5m2(q) * s).
 *  - Lloyd-Max: the 2**bits-level quantizer of N(0,1), computed by the
 *    classical fixed-point iteration (thresholds at midpoints, levels at
 *    conditional means) from a uniform start on [-3, 3], in fp64, then cast
 *    to fp32.
 *  - y = sum_k x*dq accumulated in fp64 in increasing k, plus bias, rounded
 *    once to bf16 (round to nearest even).
 *  - LoRA merge into an INT8 weight (piper-kernels README, Tensor.addmm_ on
 *    a ConvRot weight): weight = beta * weight + alpha * (mat1 @ mat2),
 *    requantized with the weight's unchanged scales.  Readings: w' =
 *    beta * dq + alpha * sum_r mat1[n, r] * mat2[r, k] in fp64 (increasing r,
 *    separate multiply and add); t = w' / s; nearest: q = rne(t); with a
 *    seed: q = floor(t) + [u < t - floor(t)], u = top 53 bits of SplitMix64
 *    output (n*K + k) for key = seed, times 2^-53 (the two adjacent codes,
 *    each with probability proportional to the distance to the other); q
 *    clamped to [-127, 127]; a zero scale keeps code 0.
 *  - Activation-quantized compute (auto-round-lib README, section 1: INT8
 *    compute with dynamic activation quantization, low-bit weights rescaled
 *    to INT8 and computed by an INT8 GEMM; the library does not implement it
 *    yet): per token m, s_x = fp32(amax_k |x| / 127), x_q = clamp(rne(x /
 *    s_x), -127, 127) (an all-zero row: s_x = 0, x_q = 0); with the INT4 /
 *    INT8 symmetric weights' integer codes q_w and bf16 group scales s_w,
 *    y = sum_g s_w[n,g] * s_x[m] * (integer sum_{k in g} q_w * x_q) in fp64
 *    over increasing g, plus bias, rounded once to bf16.
 *  - SwiGLU input (piper-kernels README, convrot_linear with
 *    input_activation="swiglu"): the input row holds [up | gate], K values
 *    each; the linear's activation is a = bf16(up * silu(gate)) with
 *    silu(g) = g / (1 + e^-g) in fp64, rounded once to bf16 (the page's
 *    materialized path: SwiGLU first, then the ordinary linear).
 *
 * Canonical (pre-pack) layouts, the input of the library's pack step:
 *   int4_sym : codes u8 [N, K/2] two's complement nibbles; scales bf16 [N, K/G]
 *   int4_asym: codes u8 [N, K/2] nibbles 0..15; scales bf16 [N, K/G];
 *              zeros u8 [N, K/G] (one per byte, 0..15)
 *   int8_sym : codes i8 [N, K]; scales bf16 [N, K/G]
 *   cb4      : codes u8 [N, K/2] indices; norms bf16 [N]; centroids f32 [16]
 *   nvfp4    : codes u8 [N, K/2] E2M1 nibbles; block scales u8 [N, K/16] E4M3;
 *              tensor scale f32 [1]
 *   mxfp4    : codes u8 [N, K/2] E2M1 nibbles; block scales u8 [N, K/32] E8M0
 *   fp8_e4m3 : codes u8 [N, K] E4M3; scales f32 [N, K/G]
 *   int2_sym : codes u8 [N, K/4] two's complement 2-bit fields, element 4i+j
 *              at bits 2j..2j+1 of byte i; scales bf16 [N, K/G]
 *   int3_sym : codes u8 [N, 3K/8] a little-endian bit stream per row, element
 *              k at bits 3k..3k+2 (two's complement); scales bf16 [N, K/G]
 *              (oracle only: the library has no INT3 kernels yet)
 *   fp8_e5m2 : codes u8 [N, K] E5M2; scales f32 [N, K/G]
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORC_INT4_SYM = 0, ORC_INT4_ASYM = 1, ORC_INT8_SYM = 2, ORC_CB4 = 3, ORC_NVFP4 = 4,
       ORC_MXFP4 = 5, ORC_FP8_E4M3 = 6, ORC_FP8_E5M2 = 7, ORC_INT2_SYM = 8,
       ORC_INT3_SYM = 9 };

/* ------------------------------------------------------------------ bf16 */
float orc_bf16_to_f32(uint16_t h) {
  uint32_t b = (uint32_t)h << 16;
  float f;
  memcpy(&f, &b, 4);
  return f;
}

/* Round a double to the nearest bf16 (ties to even).  bf16 keeps 8 significant
 * bits; below 2^-126 the spacing is fixed at 2^-133. */
uint16_t orc_f64_to_bf16(double v) {
  if (isnan(v)) return 0x7FC0;
  int neg = signbit(v) ? 1 : 0;
  double a = fabs(v);
  uint16_t sign = (uint16_t)(neg << 15);
  if (a == 0.0) return sign;
  if (isinf(a)) return (uint16_t)(sign | 0x7F80);
  int e;
  frexp(a, &e);           /* a = f * 2^e, f in [0.5, 1) */
  int E = e - 1;          /* a = 1.xxx * 2^E */
  if (E < -126) E = -126; /* subnormal spacing */
  double quantum = ldexp(1.0, E - 7);
  double r = nearbyint(a / quantum) * quantum;
  if (r >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80);
  float rf = (float)r; /* exact: r has at most 8 significant bits */
  uint32_t b;
  memcpy(&b, &rf, 4);
  return (uint16_t)(sign | (b >> 16));
}

/* ------------------------------------------------------------------ E2M1 */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double orc_e2m1_value(int code) {
  double m = E2M1_MAG[code & 7];
  return (code & 8) ? -m : m;
}

/* Nearest E2M1 code (ties to the even code), saturating at +-6; a result of
 * magnitude 0 is written as +0. */
int orc_e2m1_encode(double r) {
  int neg = r < 0.0;
  double a = fabs(r);
  int code = 7;
  for (int i = 0; i < 7; ++i) {
    double mid = 0.5 * (E2M1_MAG[i] + E2M1_MAG[i + 1]);
    if (a < mid) { code = i; break; }
    if (a == mid) { code = (i % 2 == 0) ? i : i + 1; break; }
  }
  if (code == 0) return 0;
  return code | (neg ? 8 : 0);
}

/* ------------------------------------------------------------------ E4M3 */
/* E4M3 (fn variant): 1 sign, 4 exponent (bias 7), 3 mantissa bits; exponent 0
 * is subnormal with spacing 2^-9; 0x7F / 0xFF are NaN; no infinity. */
double orc_e4m3_value(int code) {
  int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) v = ldexp((double)m, -9);
  else v = ldexp(1.0 + m / 8.0, e - 7);
  return s ? -v : v;
}

/* Nearest non-negative finite E4M3 code (ties to the even code), saturating
 * to 448 (0x7E).  d must be >= 0. */
int orc_e4m3_encode(double d) {
  if (!(d > 0.0)) return 0;
  if (d >= 448.0) return 0x7E;
  /* codes 0..126 are increasing in value */
  int lo = 0, hi = 126;
  while (hi - lo > 1) { /* invariant: value(lo) <= d < value(hi) */
    int mid = (lo + hi) / 2;
    if (orc_e4m3_value(mid) <= d) lo = mid; else hi = mid;
  }
  double vl = orc_e4m3_value(lo), vh = orc_e4m3_value(hi);
  double half = 0.5 * (vl + vh);
  if (d < half) return lo;
  if (d > half) return hi;
  return (lo % 2 == 0) ? lo : hi;
}

/* ------------------------------------------------------------------ E5M2 */
/* E5M2: 1 sign, 5 exponent (bias 15), 2 mantissa bits; exponent 0 is
 * subnormal with spacing 2^-16; exponent 31 is infinity (m = 0) or NaN. */
double orc_e5m2_value(int code) {
  int s = (code >> 7) & 1, e = (code >> 2) & 31, m = code & 3;
  double v;
  if (e == 31) v = m ? NAN : INFINITY;
  else if (e == 0) v = ldexp((double)m, -16);
  else v = ldexp(1.0 + m / 4.0, e - 15);
  return s ? -v : v;
}

/* Nearest non-negative finite E5M2 code (ties to the even code), saturating
 * to 57344 (0x7B).  d must be >= 0. */
int orc_e5m2_encode(double d) {
  if (!(d > 0.0)) return 0;
  if (d >= 57344.0) return 0x7B;
  int lo = 0, hi = 0x7B; /* codes 0..0x7B are finite and increasing */
  if (d >= orc_e5m2_value(hi)) return hi;
  while (hi - lo > 1) {  /* invariant: value(lo) <= d < value(hi) */
    int mid = (lo + hi) / 2;
    if (orc_e5m2_value(mid) <= d) lo = mid; else hi = mid;
  }
  double vl = orc_e5m2_value(lo), vh = orc_e5m2_value(hi);
  double half = 0.5 * (vl + vh);
  if (d < half) return lo;
  if (d > half) return hi;
  return (lo % 2 == 0) ? lo : hi;
}

/* ------------------------------------------------------------- nibbles */
static inline int get_nib(const uint8_t* row, int64_t k) {
  uint8_t b = row[k >> 1];
  return (k & 1) ? (b >> 4) : (b & 15);
}
static inline void put_nib(uint8_t* row, int64_t k, int v) {
  uint8_t* b = &row[k >> 1];
  if (k & 1) *b = (uint8_t)((*b & 0x0F) | ((v & 15) << 4));
  else *b = (uint8_t)((*b & 0xF0) | (v & 15));
}

/* ---------------------------------------------------------- quantizers */
int orc_quant_int_sym(const float* W, int64_t N, int64_t K, int G, int bits, void* codes,
                      uint16_t* scales) {
  if (N <= 0 || K <= 0 || G <= 0 || K % G || bits < 2 || bits > 8 || (bits > 4 && bits != 8))
    return 1;
  if ((bits == 2 && K % 4) || (bits == 3 && K % 8)) return 1;
  int qmax = (1 << (bits - 1)) - 1;
  int64_t ng = K / G;
  for (int64_t n = 0; n < N; ++n) {
    const float* w = W + n * K;
    uint8_t* row4 = (uint8_t*)codes + n * (K / 2);
    int8_t* row8 = (int8_t*)codes + n * K;
    uint8_t* row2 = (uint8_t*)codes + n * (K / 4);
    if (bits == 4) memset(row4, 0, (size_t)(K / 2));
    if (bits == 2) memset(row2, 0, (size_t)(K / 4));
    uint8_t* row3 = (uint8_t*)codes + n * (K / 8 * 3);
    if (bits == 3) memset(row3, 0, (size_t)(K / 8 * 3));
    for (int64_t j = 0; j < ng; ++j) {
      double amax = 0.0;
      for (int64_t k = j * G; k < (j + 1) * G; ++k) amax = fmax(amax, fabs((double)w[k]));
      uint16_t sb = orc_f64_to_bf16(amax / (double)qmax);
      scales[n * ng + j] = sb;
      double s = (double)orc_bf16_to_f32(sb);
      for (int64_t k = j * G; k < (j + 1) * G; ++k) {
        int q = 0;
        if (s != 0.0) {
          double r = nearbyint((double)w[k] / s);
          if (r > qmax) r = qmax;
          if (r < -qmax) r = -qmax;
          q = (int)r;
        }
        if (bits == 3) {
          for (int b = 0; b < 3; ++b)
            if ((q >> b) & 1) row3[(3 * k + b) >> 3] |= (uint8_t)(1u << ((3 * k + b) & 7));
        } else if (bits == 2) row2[k >> 2] |= (uint8_t)((q & 3) << (2 * (k & 3)));
        else if (bits == 4) put_nib(row4, k, q & 15);
        else row8[k] = (int8_t)q;
      }
    }
  }
  return 0;
}

int orc_quant_int4_asym(const float* W, int64_t N, int64_t K, int G, uint8_t* codes,
                        uint16_t* scales, uint8_t* zeros) {
  if (N <= 0 || K <= 0 || G <= 0 || K % G || K % 2) return 1;
  int64_t ng = K / G;
  for (int64_t n = 0; n < N; ++n) {
    const float* w = W + n * K;
    uint8_t* row = codes + n * (K / 2);
    memset(row, 0, (size_t)(K / 2));
    for (int64_t j = 0; j < ng; ++j) {
      double lo = 0.0, hi = 0.0;
      for (int64_t k = j * G; k < (j + 1) * G; ++k) {
        lo = fmin(lo, (double)w[k]);
        hi = fmax(hi, (double)w[k]);
      }
      uint16_t sb = orc_f64_to_bf16((hi - lo) / 15.0);
      scales[n * ng + j] = sb;
      double s = (double)orc_bf16_to_f32(sb);
      int z = 0;
      if (s != 0.0) {
        double zr = nearbyint(-lo / s);
        if (zr < 0) zr = 0;
        if (zr > 15) zr = 15;
        z = (int)zr;
      }
      zeros[n * ng + j] = (uint8_t)z;
      for (int64_t k = j * G; k < (j + 1) * G; ++k) {
        int q = 0;
        if (s != 0.0) {
          double r = nearbyint((double)w[k] / s) + z;
          if (r < 0) r = 0;
          if (r > 15) r = 15;
          q = (int)r;
        }
        put_nib(row, k, q);
      }
    }
  }
  return 0;
}

/* Standard normal mass on [a, b], taking the tail form that keeps precision. */
static double normal_mass(double a, double b) {
  const double r2 = 1.4142135623730950488016887242097;
  if (a >= 0.0) return 0.5 * (erfc(a / r2) - erfc(b / r2));
  if (b <= 0.0) return 0.5 * (erfc(-b / r2) - erfc(-a / r2));
  return 0.5 * (erf(b / r2) - erf(a / r2));
}
static double normal_pdf(double x) {
  if (isinf(x)) return 0.0;
  return exp(-0.5 * x * x) / 2.5066282746310005024157652848110;
}

/* Lloyd-Max quantizer of N(0,1) with L levels (L >= 2): alternate
 * thresholds t_i = (c_i + c_{i+1})/2 and levels
 * c_i = (pdf(t_{i-1}) - pdf(t_i)) / (Phi(t_i) - Phi(t_{i-1})), the mean of
 * N(0,1) restricted to the cell, until no level moves by 1e-14. */
int orc_lloyd_max_gaussian(int L, double* c64, float* c32, int* iters_out, double* mse_out) {
  if (L < 2 || L > 256) return 1;
  double* c = (double*)malloc(sizeof(double) * L);
  double* t = (double*)malloc(sizeof(double) * (L + 1));
  if (!c || !t) { free(c); free(t); return 2; }
  for (int i = 0; i < L; ++i) c[i] = -3.0 + 6.0 * i / (L - 1);
  int it = 0;
  for (; it < 1000000; ++it) {
    t[0] = -INFINITY;
    t[L] = INFINITY;
    for (int i = 1; i < L; ++i) t[i] = 0.5 * (c[i - 1] + c[i]);
    double moved = 0.0;
    for (int i = 0; i < L; ++i) {
      double p = normal_mass(t[i], t[i + 1]);
      double nc = (normal_pdf(t[i]) - normal_pdf(t[i + 1])) / p;
      moved = fmax(moved, fabs(nc - c[i]));
      c[i] = nc;
    }
    if (moved < 1e-14) { ++it; break; }
  }
  /* mean squared error of the final quantizer:
   * E[(Z - c_i)^2 ; cell i] = (1 + c_i^2) P_i - 2 c_i (pdf(a) - pdf(b))
   *                           + a pdf(a) - b pdf(b)                  */
  for (int i = 1; i < L; ++i) t[i] = 0.5 * (c[i - 1] + c[i]);
  double mse = 0.0;
  for (int i = 0; i < L; ++i) {
    double a = t[i], b = t[i + 1];
    double p = normal_mass(a, b);
    double pa = normal_pdf(a), pb = normal_pdf(b);
    double apa = isinf(a) ? 0.0 : a * pa, bpb = isinf(b) ? 0.0 : b * pb;
    mse += (1.0 + c[i] * c[i]) * p - 2.0 * c[i] * (pa - pb) + apa - bpb;
  }
  for (int i = 0; i < L; ++i) {
    if (c64) c64[i] = c[i];
    if (c32) c32[i] = (float)c[i];
  }
  if (iters_out) *iters_out = it;
  if (mse_out) *mse_out = mse;
  free(c);
  free(t);
  return 0;
}

int orc_quant_cb4(const float* W, int64_t N, int64_t K, const float* centroids, uint8_t* codes,
                  uint16_t* norms) {
  if (N <= 0 || K <= 0 || K % 2) return 1;
  for (int64_t n = 0; n < N; ++n) {
    const float* w = W + n * K;
    uint8_t* row = codes + n * (K / 2);
    memset(row, 0, (size_t)(K / 2));
    double ss = 0.0;
    for (int64_t k = 0; k < K; ++k) ss += (double)w[k] * (double)w[k];
    double norm64 = sqrt(ss) / sqrt((double)K);
    uint16_t nb = orc_f64_to_bf16(norm64);
    norms[n] = nb;
    double nd = (double)orc_bf16_to_f32(nb);
    for (int64_t k = 0; k < K; ++k) {
      int best = 0;
      if (nd != 0.0) {
        double r = (double)w[k] / nd;
        double bestd = fabs(r - (double)centroids[0]);
        for (int j = 1; j < 16; ++j) {
          double d = fabs(r - (double)centroids[j]);
          if (d < bestd) { bestd = d; best = j; }
        }
      }
      put_nib(row, k, best);
    }
  }
  return 0;
}

int orc_quant_nvfp4(const float* W, int64_t N, int64_t K, uint8_t* codes, uint8_t* bscales,
                    float* tscale) {
  if (N <= 0 || K <= 0 || K % 16) return 1;
  double amax = 0.0;
  for (int64_t e = 0; e < N * K; ++e) amax = fmax(amax, fabs((double)W[e]));
  float ts = (float)(amax / (6.0 * 448.0));
  *tscale = ts;
  int64_t nb = K / 16;
  for (int64_t n = 0; n < N; ++n) {
    const float* w = W + n * K;
    uint8_t* row = codes + n * (K / 2);
    memset(row, 0, (size_t)(K / 2));
    for (int64_t b = 0; b < nb; ++b) {
      double ab = 0.0;
      for (int64_t k = b * 16; k < b * 16 + 16; ++k) ab = fmax(ab, fabs((double)w[k]));
      int sb = 0;
      if (ts != 0.0f) sb = orc_e4m3_encode(ab / (6.0 * (double)ts));
      bscales[n * nb + b] = (uint8_t)sb;
      double d = orc_e4m3_value(sb) * (double)ts;
      for (int64_t k = b * 16; k < b * 16 + 16; ++k) {
        int q = 0;
        if (d != 0.0) q = orc_e2m1_encode((double)w[k] / d);
        put_nib(row, k, q);
      }
    }
  }
  return 0;
}

/* E8M0 (unsigned power-of-two scale): 2^(code - 127); code 255 is NaN. */
double orc_e8m0_value(int code) {
  if (code == 255) return NAN;
  return ldexp(1.0, code - 127);
}

int orc_quant_mxfp4(const float* W, int64_t N, int64_t K, uint8_t* codes, uint8_t* bscales) {
  if (N <= 0 || K <= 0 || K % 32) return 1;
  int64_t nb = K / 32;
  for (int64_t n = 0; n < N; ++n) {
    const float* w = W + n * K;
    uint8_t* row = codes + n * (K / 2);
    memset(row, 0, (size_t)(K / 2));
    for (int64_t b = 0; b < nb; ++b) {
      double ab = 0.0;
      for (int64_t k = b * 32; k < b * 32 + 32; ++k) ab = fmax(ab, fabs((double)w[k]));
      int e = 0;
      if (ab > 0.0) {
        int ex;
        frexp(ab, &ex);         /* ab = m * 2^ex, m in [0.5, 1): floor(log2 ab) = ex - 1 */
        int se = (ex - 1) - 2;  /* minus the largest E2M1 exponent */
        if (se < -127) se = -127;
        if (se > 127) se = 127;
        e = se + 127;
      }
      bscales[n * nb + b] = (uint8_t)e;
      if (ab > 0.0) {
        double d = orc_e8m0_value(e);
        for (int64_t k = b * 32; k < b * 32 + 32; ++k) put_nib(row, k, orc_e2m1_encode((double)w[k] / d));
      }
    }
  }
  return 0;
}

/* FP8 weights (E4M3 or E5M2), fp32 scale per group of G along K. */
static int quant_fp8(const float* W, int64_t N, int64_t K, int G, int e5m2, uint8_t* codes,
                     float* scales) {
  if (N <= 0 || K <= 0 || G <= 0 || K % G) return 1;
  const double fmax_code = e5m2 ? 57344.0 : 448.0;
  int64_t ng = K / G;
  for (int64_t n = 0; n < N; ++n) {
    const float* w = W + n * K;
    for (int64_t j = 0; j < ng; ++j) {
      double amax = 0.0;
      for (int64_t k = j * G; k < (j + 1) * G; ++k) amax = fmax(amax, fabs((double)w[k]));
      float sf = (float)(amax / fmax_code);
      scales[n * ng + j] = sf;
      double s = (double)sf;
      for (int64_t k = j * G; k < (j + 1) * G; ++k) {
        int q = 0;
        if (s != 0.0) {
          double r = (double)w[k] / s;
          q = e5m2 ? orc_e5m2_encode(fabs(r)) : orc_e4m3_encode(fabs(r));
          if (r < 0.0 && q != 0) q |= 0x80;
        }
        codes[n * K + k] = (uint8_t)q;
      }
    }
  }
  return 0;
}

int orc_quant_fp8_e4m3(const float* W, int64_t N, int64_t K, int G, uint8_t* codes,
                       float* scales) {
  return quant_fp8(W, N, K, G, 0, codes, scales);
}
int orc_quant_fp8_e5m2(const float* W, int64_t N, int64_t K, int G, uint8_t* codes,
                       float* scales) {
  return quant_fp8(W, N, K, G, 1, codes, scales);
}

/* ------------------------------------------------------------- dequant */
/* Exact dequantized value of element (n, k) from the canonical layout. */
static float dq_one(int fmt, int64_t K, int G, const void* codes, const void* scales,
                    const void* aux, int64_t n, int64_t k) {
  switch (fmt) {
    case ORC_INT4_SYM: {
      int nib = get_nib((const uint8_t*)codes + n * (K / 2), k);
      int v = nib > 7 ? nib - 16 : nib;
      float s = orc_bf16_to_f32(((const uint16_t*)scales)[n * (K / G) + k / G]);
      return (float)v * s;
    }
    case ORC_INT4_ASYM: {
      int q = get_nib((const uint8_t*)codes + n * (K / 2), k);
      int z = ((const uint8_t*)aux)[n * (K / G) + k / G];
      float s = orc_bf16_to_f32(((const uint16_t*)scales)[n * (K / G) + k / G]);
      return (float)(q - z) * s;
    }
    case ORC_INT3_SYM: {
      const uint8_t* row = (const uint8_t*)codes + n * (K / 8 * 3);
      int c = 0;
      for (int b = 0; b < 3; ++b) c |= ((row[(3 * k + b) >> 3] >> ((3 * k + b) & 7)) & 1) << b;
      int v = c > 3 ? c - 8 : c;
      float s = orc_bf16_to_f32(((const uint16_t*)scales)[n * (K / G) + k / G]);
      return (float)v * s;
    }
    case ORC_INT2_SYM: {
      int c = (((const uint8_t*)codes)[n * (K / 4) + k / 4] >> (2 * (k & 3))) & 3;
      int v = c > 1 ? c - 4 : c;
      float s = orc_bf16_to_f32(((const uint16_t*)scales)[n * (K / G) + k / G]);
      return (float)v * s;
    }
    case ORC_INT8_SYM: {
      int v = ((const int8_t*)codes)[n * K + k];
      float s = orc_bf16_to_f32(((const uint16_t*)scales)[n * (K / G) + k / G]);
      return (float)v * s;
    }
    case ORC_CB4: {
      int idx = get_nib((const uint8_t*)codes + n * (K / 2), k);
      double c = (double)((const float*)aux)[idx];
      double nr = (double)orc_bf16_to_f32(((const uint16_t*)scales)[n]);
      return (float)(c * nr);
    }
    case ORC_NVFP4: {
      int q = get_nib((const uint8_t*)codes + n * (K / 2), k);
      int sb = ((const uint8_t*)scales)[n * (K / 16) + k / 16];
      double ts = (double)((const float*)aux)[0];
      return (float)(orc_e2m1_value(q) * orc_e4m3_value(sb) * ts);
    }
    case ORC_MXFP4: {
      int q = get_nib((const uint8_t*)codes + n * (K / 2), k);
      int e = ((const uint8_t*)scales)[n * (K / 32) + k / 32];
      return (float)(orc_e2m1_value(q) * orc_e8m0_value(e));
    }
    case ORC_FP8_E4M3: {
      int q = ((const uint8_t*)codes)[n * K + k];
      double s = (double)((const float*)scales)[n * (K / G) + k / G];
      return (float)(orc_e4m3_value(q) * s);
    }
    case ORC_FP8_E5M2: {
      int q = ((const uint8_t*)codes)[n * K + k];
      double s = (double)((const float*)scales)[n * (K / G) + k / G];
      return (float)(orc_e5m2_value(q) * s);
    }
  }
  return NAN;
}

static int check_fmt(int fmt, int64_t N, int64_t K, int G) {
  if (N <= 0 || K <= 0) return 1;
  if (fmt < 0 || fmt > 9) return 1;
  const int bytes = fmt == ORC_INT8_SYM || fmt == ORC_FP8_E4M3 || fmt == ORC_FP8_E5M2;
  if ((fmt == ORC_INT4_SYM || fmt == ORC_INT4_ASYM || fmt == ORC_INT8_SYM ||
       fmt == ORC_FP8_E4M3 || fmt == ORC_FP8_E5M2 || fmt == ORC_INT2_SYM ||
       fmt == ORC_INT3_SYM) && (G <= 0 || K % G))
    return 1;
  if (fmt == ORC_INT2_SYM && K % 4) return 1;
  if (fmt == ORC_INT3_SYM && K % 8) return 1;
  if (!bytes && K % 2) return 1;
  if (fmt == ORC_NVFP4 && K % 16) return 1;
  if (fmt == ORC_MXFP4 && K % 32) return 1;
  return 0;
}

int orc_dequant(int fmt, int64_t N, int64_t K, int G, const void* codes, const void* scales,
                const void* aux, float* out) {
  if (check_fmt(fmt, N, K, G)) return 1;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) out[n * K + k] = dq_one(fmt, K, G, codes, scales, aux, n, k);
  return 0;
}

/* -------------------------------------------------------------- linear */
/* y[m,n] = sum_k x[m,k] * dq[n,k] (fp64, k increasing) + bias[n]; bf16 out.
 * Every product of a bf16 and an fp32 is exact in fp64. */
int orc_linear(const uint16_t* x, const float* dq, const uint16_t* bias, int64_t M, int64_t N,
               int64_t K, uint16_t* y, double* y64) {
  if (M < 0 || N <= 0 || K <= 0) return 1;
#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t n = 0; n < N; ++n) {
    const float* w = dq + n * K;
    for (int64_t m = 0; m < M; ++m) {
      const uint16_t* xr = x + m * K;
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) acc += (double)orc_bf16_to_f32(xr[k]) * (double)w[k];
      if (bias) acc += (double)orc_bf16_to_f32(bias[n]);
      if (y64) y64[m * N + n] = acc;
      if (y) y[m * N + n] = orc_f64_to_bf16(acc);
    }
  }
  return 0;
}

/* y[i] = bf16(v[i]) (round to nearest even) for n values: the rounding of a
 * full fp64 product computed elsewhere (a library fp64 matmul) to the output
 * type, with the same rounding as orc_linear. */
int orc_round_bf16_array(const double* v, int64_t n, uint16_t* y) {
  if (n < 0) return 1;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) y[i] = orc_f64_to_bf16(v[i]);
  return 0;
}

/* Per-token INT8 activation quantization: xq int8 [M, K], sx f32 [M]. */
int orc_quant_act_int8(const uint16_t* x, int64_t M, int64_t K, int8_t* xq, float* sx) {
  if (M < 0 || K <= 0) return 1;
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    double amax = 0.0;
    for (int64_t k = 0; k < K; ++k) amax = fmax(amax, fabs((double)orc_bf16_to_f32(x[m * K + k])));
    float s = (float)(amax / 127.0);
    sx[m] = s;
    for (int64_t k = 0; k < K; ++k) {
      double q = 0.0;
      if (s != 0.0f) {
        q = nearbyint((double)orc_bf16_to_f32(x[m * K + k]) / (double)s);
        if (q > 127.0) q = 127.0;
        if (q < -127.0) q = -127.0;
      }
      xq[m * K + k] = (int8_t)q;
    }
  }
  return 0;
}

/* y = sum over groups of s_w * s_x * (integer dot of codes), for the INT4 /
 * INT8 symmetric formats (canonical codes and bf16 group scales). */
int orc_linear_a8(int fmt, const void* codes, const uint16_t* scales, int64_t N, int64_t K, int G,
                  const int8_t* xq, const float* sx, const uint16_t* bias, int64_t M, uint16_t* y,
                  double* y64) {
  if ((fmt != ORC_INT4_SYM && fmt != ORC_INT8_SYM) || check_fmt(fmt, N, K, G) || M < 0) return 1;
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t n = 0; n < N; ++n)
    for (int64_t m = 0; m < M; ++m) {
      double acc = 0.0;
      for (int64_t g = 0; g < K / G; ++g) {
        int64_t isum = 0;
        for (int64_t k = g * G; k < (g + 1) * G; ++k) {
          int qw;
          if (fmt == ORC_INT8_SYM) {
            qw = ((const int8_t*)codes)[n * K + k];
          } else {
            int nib = get_nib((const uint8_t*)codes + n * (K / 2), k);
            qw = nib > 7 ? nib - 16 : nib;
          }
          isum += (int64_t)qw * (int64_t)xq[m * K + k];
        }
        acc += (double)orc_bf16_to_f32(scales[n * (K / G) + g]) * (double)sx[m] * (double)isum;
      }
      if (bias) acc = acc + (double)orc_bf16_to_f32(bias[n]);
      if (y64) y64[m * N + n] = acc;
      if (y) y[m * N + n] = orc_f64_to_bf16(acc);
    }
  return 0;
}

/* SwiGLU input: a[m, k] = bf16(up * silu(gate)), up = x2[m, k],
 * gate = x2[m, K + k]; x2 is bf16 [M, 2K]. */
double orc_silu(double g) { return g / (1.0 + exp(-g)); }

int orc_swiglu(const uint16_t* x2, int64_t M, int64_t K, uint16_t* a) {
  if (M < 0 || K <= 0) return 1;
  for (int64_t m = 0; m < M; ++m)
    for (int64_t k = 0; k < K; ++k) {
      double up = (double)orc_bf16_to_f32(x2[m * 2 * K + k]);
      double gate = (double)orc_bf16_to_f32(x2[m * 2 * K + K + k]);
      a[m * K + k] = orc_f64_to_bf16(up * orc_silu(gate));
    }
  return 0;
}

/* SplitMix64 (Vigna): output i of the counter-based stream keyed by `key`. */
static uint64_t orc_splitmix64(uint64_t key, uint64_t i) {
  uint64_t z = key + (i + 1) * 0x9E3779B97F4A7C15ULL;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* LoRA merge into INT8 codes (canonical int8 [N, K], bf16 scales [N, K/G]):
 * codes are rewritten in place; mat1 bf16 [N, R], mat2 bf16 [R, K]. */
int orc_addmm_requant_int8(int8_t* codes, const uint16_t* scales, int64_t N, int64_t K, int G,
                           const uint16_t* mat1, const uint16_t* mat2, int64_t R, double alpha,
                           double beta, int stochastic, uint64_t seed) {
  if (N <= 0 || K <= 0 || G <= 0 || K % G || R < 0) return 1;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) {
      double s = (double)orc_bf16_to_f32(scales[n * (K / G) + k / G]);
      if (s == 0.0) { codes[n * K + k] = 0; continue; }
      double dot = 0.0;
      for (int64_t r = 0; r < R; ++r) {
        double p = (double)orc_bf16_to_f32(mat1[n * R + r]) * (double)orc_bf16_to_f32(mat2[r * K + k]);
        dot = dot + p;
      }
      double wq = beta * ((double)codes[n * K + k] * s) + alpha * dot;
      double t = wq / s, q;
      if (stochastic) {
        double f = floor(t);
        double u = (double)(orc_splitmix64(seed, (uint64_t)(n * K + k)) >> 11) * 0x1p-53;
        q = f + (u < t - f ? 1.0 : 0.0);
      } else {
        q = nearbyint(t);
      }
      if (q > 127.0) q = 127.0;
      if (q < -127.0) q = -127.0;
      codes[n * K + k] = (int8_t)q;
    }
  return 0;
}

/* The same value for chosen (m, n) pairs only, dequantizing row n on the fly
 * from the canonical layout; for workloads too large for the full product. */
int orc_linear_sampled(int fmt, int64_t N, int64_t K, int G, const void* codes,
                       const void* scales, const void* aux, const uint16_t* x,
                       const uint16_t* bias, int64_t S, const int64_t* ms, const int64_t* ns,
                       uint16_t* y, double* y64) {
  if (check_fmt(fmt, N, K, G)) return 1;
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t i = 0; i < S; ++i) {
    int64_t m = ms[i], n = ns[i];
    const uint16_t* xr = x + m * K;
    double acc = 0.0;
    for (int64_t k = 0; k < K; ++k)
      acc += (double)orc_bf16_to_f32(xr[k]) *
             (double)dq_one(fmt, K, G, codes, scales, aux, n, k);
    if (bias) acc += (double)orc_bf16_to_f32(bias[n]);
    if (y64) y64[i] = acc;
    if (y) y[i] = orc_f64_to_bf16(acc);
  }
  return 0;
}

/* Threads that OpenMP uses for the parallel loops above. */
int orc_threads(void);
/* Threads the parallel loops use from now on (n >= 1). */
void orc_set_threads(int n);
#ifdef _OPENMP
#include <omp.h>
int orc_threads(void) { return omp_get_max_threads(); }
void orc_set_threads(int n) { omp_set_num_threads(n < 1 ? 1 : n); }
#else
int orc_threads(void) { return 1; }
void orc_set_threads(int n) { (void)n; }
#endif

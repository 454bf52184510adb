// Offline round-to-nearest quantizers (dense fp32 weight -> canonical codes).
//
// Every decision that turns a real number into a code is taken in fp64 with
// the same IEEE operations, in the same order, as the definitions in wq.h, so
// the codes are bit-identical to the CPU definitions.  Products and sums are
// written with explicit round-to-nearest intrinsics so that the compiler does
// not fuse them.  Sources: piper-kernels README "ConvRot INT8"
// (ConvRotInt8Tensor.from_hp(dense_weight, group_size=256)); the Mamba-2
// paired-nibble pack helper (scale = amax/qmax, round, clamp to +-qmax);
// OrbitQuant card "Inputs" (row norms, Lloyd-Max centroids); Petit README
// "Features" (NVFP4, MXFP4) and "Known limitations" (positive scales, no -0
// codes).
#include "wq_internal.cuh"

namespace wq {

namespace {

// fp64 -> bf16 bits, round to nearest even, via round-to-odd in fp32.
__device__ __forceinline__ uint16_t f64_to_bf16_rn(double v) {
  if (v != v) return 0x7FC0;
  float t = __double2float_rz(v);  // truncated toward zero
  uint32_t b = __float_as_uint(t);
  bool inexact = (double)t != v;
  if ((b & 0x7F800000u) == 0x7F800000u) return (uint16_t)(b >> 16);  // inf
  if (inexact) {
    // |v| beyond the largest finite fp32 truncates to FLT_MAX: treat as overflow
    if (fabs(v) > 3.4028234663852886e38) return (uint16_t)((b >> 16 & 0x8000u) | 0x7F80u);
    b |= 1u;  // sticky
  }
  uint32_t r = b + 0x7FFFu + ((b >> 16) & 1u);
  return (uint16_t)(r >> 16);
}

// nearest E4M3 code (sign clear), ties to even, saturating at 448
__device__ __forceinline__ uint32_t e4m3_encode_rn_satfinite(double d) {
  if (!(d > 0.0)) return 0u;
  if (d >= 448.0) return 0x7Eu;
  // quantum of the binade containing d (subnormal spacing 2^-9 below 2^-6)
  int e = ilogb(d);
  if (e < -6) e = -6;
  double q = ldexp(1.0, e - 3);
  double r = rint(d / q);  // exact division by a power of two
  double v = r * q;        // representable candidate (may equal 2^(e+1))
  // encode v: v >= 2^-6 normal, else subnormal
  if (v >= 448.0) return 0x7Eu;
  if (v < 0.015625) return (uint32_t)(v * 512.0);  // m in 0..8 (8 == 2^-6 encodes as 0x08)
  int ev = ilogb(v);
  uint32_t m = (uint32_t)((v / ldexp(1.0, ev) - 1.0) * 8.0);
  return ((uint32_t)(ev + 7) << 3) | m;
}

// nearest E5M2 code (sign clear), ties to even, saturating at 57344
__device__ __forceinline__ uint32_t e5m2_encode_rn_satfinite(double d) {
  if (!(d > 0.0)) return 0u;
  if (d >= 57344.0) return 0x7Bu;
  // quantum of the binade containing d (subnormal spacing 2^-16 below 2^-14)
  int e = ilogb(d);
  if (e < -14) e = -14;
  double q = ldexp(1.0, e - 2);
  double r = rint(d / q);  // exact division by a power of two
  double v = r * q;        // representable candidate (may equal 2^(e+1))
  if (v >= 57344.0) return 0x7Bu;
  if (v < 6.103515625e-05) return (uint32_t)(v * 65536.0);  // m in 0..4 (4 == 2^-14 encodes as 0x04)
  int ev = ilogb(v);
  uint32_t m = (uint32_t)((v / ldexp(1.0, ev) - 1.0) * 4.0);
  return ((uint32_t)(ev + 15) << 2) | m;
}

// nearest E2M1 code, ties to even, saturating at 6; zero is +0
__device__ __forceinline__ uint32_t e2m1_encode_rn_sat(double r) {
  double a = fabs(r);
  uint32_t c;
  // cell boundaries between {0, .5, 1, 1.5, 2, 3, 4, 6}; at a boundary the
  // code with an even index wins
  if (a <= 0.25) c = 0;
  else if (a < 0.75) c = 1;
  else if (a <= 1.25) c = 2;
  else if (a < 1.75) c = 3;
  else if (a <= 2.5) c = 4;
  else if (a < 3.5) c = 5;
  else if (a <= 5.0) c = 6;
  else c = 7;
  if (c == 0) return 0u;
  return c | (r < 0.0 ? 8u : 0u);
}

constexpr int kWarps = 8;

// One warp per (row, group): symmetric INT2 / INT4 / INT8.
__global__ void quant_sym_kernel(int bits, int64_t N, int64_t K, int G,
                                 const float* __restrict__ w, uint8_t* __restrict__ codes,
                                 uint16_t* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int64_t groups = K / G;
  const int qmax = (1 << (bits - 1)) - 1;
  for (int64_t item = blockIdx.x * (int64_t)kWarps + (threadIdx.x >> 5); item < N * groups;
       item += (int64_t)gridDim.x * kWarps) {
    int64_t n = item / groups, grp = item % groups;
    const float* wg = w + n * K + grp * G;
    double amax = 0.0;
    for (int i = lane; i < G; i += 32) amax = fmax(amax, fabs((double)wg[i]));
    for (int o = 16; o; o >>= 1) amax = fmax(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    uint16_t sb = f64_to_bf16_rn(__ddiv_rn(amax, (double)qmax));
    double s = (double)bf16_bits_to_f32(sb);
    if (lane == 0) scales[item] = sb;
    if (bits == 2) {
      for (int i = 4 * lane; i < G; i += 128) {
        uint32_t packed = 0;
        for (int j = 0; j < 4; ++j) {
          int q = 0;
          if (s != 0.0) q = max(-qmax, min(qmax, __double2int_rn(__ddiv_rn((double)wg[i + j], s))));
          packed |= (uint32_t)(q & 3) << (2 * j);
        }
        codes[n * (K / 4) + (grp * G + i) / 4] = (uint8_t)packed;
      }
    } else if (bits == 3) {
      // eight codes = three bytes of the row's bit stream (a group of G
      // starts on a byte: 3 G / 8 bytes per group)
      for (int i = 8 * lane; i < G; i += 256) {
        uint32_t packed = 0;
        for (int j = 0; j < 8; ++j) {
          int q = 0;
          if (s != 0.0) q = max(-qmax, min(qmax, __double2int_rn(__ddiv_rn((double)wg[i + j], s))));
          packed |= (uint32_t)(q & 7) << (3 * j);
        }
        uint8_t* dst = codes + n * (3 * K / 8) + 3 * ((grp * G + i) / 8);
        dst[0] = (uint8_t)packed;
        dst[1] = (uint8_t)(packed >> 8);
        dst[2] = (uint8_t)(packed >> 16);
      }
    } else if (bits == 4) {
      for (int i = 2 * lane; i < G; i += 64) {
        int q0 = 0, q1 = 0;
        if (s != 0.0) {
          q0 = max(-qmax, min(qmax, __double2int_rn(__ddiv_rn((double)wg[i], s))));
          q1 = max(-qmax, min(qmax, __double2int_rn(__ddiv_rn((double)wg[i + 1], s))));
        }
        codes[n * (K / 2) + (grp * G + i) / 2] = (uint8_t)((q0 & 15) | ((q1 & 15) << 4));
      }
    } else {
      for (int i = lane; i < G; i += 32) {
        int q = 0;
        if (s != 0.0) q = max(-qmax, min(qmax, __double2int_rn(__ddiv_rn((double)wg[i], s))));
        codes[n * K + grp * G + i] = (uint8_t)(int8_t)q;
      }
    }
  }
}

// One warp per (row, group): FP8 codes, fp32 scale = amax / (largest finite
// value: 448 for E4M3, 57344 for E5M2).
__global__ void quant_fp8_kernel(int64_t N, int64_t K, int G, bool e5m2,
                                 const float* __restrict__ w, uint8_t* __restrict__ codes,
                                 float* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int64_t groups = K / G;
  for (int64_t item = blockIdx.x * (int64_t)kWarps + (threadIdx.x >> 5); item < N * groups;
       item += (int64_t)gridDim.x * kWarps) {
    int64_t n = item / groups, grp = item % groups;
    const float* wg = w + n * K + grp * G;
    double amax = 0.0;
    for (int i = lane; i < G; i += 32) amax = fmax(amax, fabs((double)wg[i]));
    for (int o = 16; o; o >>= 1) amax = fmax(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float sf = __double2float_rn(__ddiv_rn(amax, e5m2 ? 57344.0 : 448.0));
    const double s = (double)sf;
    if (lane == 0) scales[item] = sf;
    for (int i = lane; i < G; i += 32) {
      uint32_t q = 0;
      if (s != 0.0) {
        const double r = __ddiv_rn((double)wg[i], s);
        q = e5m2 ? e5m2_encode_rn_satfinite(fabs(r)) : e4m3_encode_rn_satfinite(fabs(r));
        if (r < 0.0 && q != 0u) q |= 0x80u;
      }
      codes[n * K + grp * G + i] = (uint8_t)q;
    }
  }
}

// One warp per (row, group): asymmetric INT4 with a uint4 zero-point.
__global__ void quant_asym_kernel(int64_t N, int64_t K, int G, const float* __restrict__ w,
                                  uint8_t* __restrict__ codes, uint16_t* __restrict__ scales,
                                  uint8_t* __restrict__ zeros) {
  const int lane = threadIdx.x & 31;
  const int64_t groups = K / G;
  for (int64_t item = blockIdx.x * (int64_t)kWarps + (threadIdx.x >> 5); item < N * groups;
       item += (int64_t)gridDim.x * kWarps) {
    int64_t n = item / groups, grp = item % groups;
    const float* wg = w + n * K + grp * G;
    double lo = 0.0, hi = 0.0;
    for (int i = lane; i < G; i += 32) {
      lo = fmin(lo, (double)wg[i]);
      hi = fmax(hi, (double)wg[i]);
    }
    for (int o = 16; o; o >>= 1) {
      lo = fmin(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmax(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    uint16_t sb = f64_to_bf16_rn(__ddiv_rn(__dsub_rn(hi, lo), 15.0));
    double s = (double)bf16_bits_to_f32(sb);
    int z = 0;
    if (s != 0.0) z = max(0, min(15, __double2int_rn(__ddiv_rn(-lo, s))));
    if (lane == 0) {
      scales[item] = sb;
      zeros[item] = (uint8_t)z;
    }
    for (int i = 2 * lane; i < G; i += 64) {
      int q0 = 0, q1 = 0;
      if (s != 0.0) {
        q0 = max(0, min(15, __double2int_rn(__ddiv_rn((double)wg[i], s)) + z));
        q1 = max(0, min(15, __double2int_rn(__ddiv_rn((double)wg[i + 1], s)) + z));
      }
      codes[n * (K / 2) + (grp * G + i) / 2] = (uint8_t)(q0 | (q1 << 4));
    }
  }
}

// One thread per row: the row norm ||w||_2 / sqrt(K), summed in increasing k.
__global__ void cb4_norm_kernel(int64_t N, int64_t K, const float* __restrict__ w,
                                uint16_t* __restrict__ norms) {
  for (int64_t n = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; n < N;
       n += (int64_t)gridDim.x * blockDim.x) {
    const float* wr = w + n * K;
    double ss = 0.0;
    for (int64_t k = 0; k < K; ++k) {
      double v = (double)wr[k];
      ss = __dadd_rn(ss, __dmul_rn(v, v));
    }
    double nrm = __ddiv_rn(__dsqrt_rn(ss), __dsqrt_rn((double)K));
    norms[n] = f64_to_bf16_rn(nrm);
  }
}

// One thread per canonical byte: nearest centroid of w / norm, ties to the lower index.
__global__ void cb4_code_kernel(int64_t N, int64_t K, const float* __restrict__ w,
                                const uint16_t* __restrict__ norms,
                                const float* __restrict__ centroids, uint8_t* __restrict__ codes) {
  __shared__ double c[16];
  if (threadIdx.x < 16) c[threadIdx.x] = (double)centroids[threadIdx.x];
  __syncthreads();
  const int64_t total = N * K / 2;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    int64_t n = (2 * i) / K;
    double nd = (double)bf16_bits_to_f32(norms[n]);
    uint32_t out = 0;
    for (int h = 0; h < 2; ++h) {
      int best = 0;
      if (nd != 0.0) {
        double r = __ddiv_rn((double)w[2 * i + h], nd);
        double bd = fabs(__dsub_rn(r, c[0]));
        for (int j = 1; j < 16; ++j) {
          double d = fabs(__dsub_rn(r, c[j]));
          if (d < bd) { bd = d; best = j; }
        }
      }
      out |= (uint32_t)best << (4 * h);
    }
    codes[i] = (uint8_t)out;
  }
}

// NVFP4 pass 1: global max |w| into the tensor-scale slot (as float bits;
// non-negative floats order like their bit patterns).
__global__ void nvfp4_amax_kernel(int64_t total, const float* __restrict__ w,
                                  unsigned int* __restrict__ slot) {
  float m = 0.f;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x)
    m = fmaxf(m, fabsf(w[i]));
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(slot, __float_as_uint(m));
}

// NVFP4 pass 2: one warp per 16-element block (two lanes per byte of codes).
__global__ void nvfp4_code_kernel(int64_t N, int64_t K, const float* __restrict__ w,
                                  const unsigned int* __restrict__ amax_slot,
                                  uint8_t* __restrict__ codes, uint8_t* __restrict__ bscales) {
  const double amax = (double)__uint_as_float(*amax_slot);
  const float ts = __double2float_rn(__ddiv_rn(amax, 6.0 * 448.0));
  const int64_t blocks = N * (K / 16);
  const int lane = threadIdx.x & 31;
  // 2 blocks per warp: lanes 0..15 block bp, lanes 16..31 block bp+1; the
  // loop bound is uniform across the warp so that the shuffles see all lanes
  for (int64_t bp = (blockIdx.x * (int64_t)kWarps + (threadIdx.x >> 5)) * 2; bp < blocks;
       bp += (int64_t)gridDim.x * kWarps * 2) {
    const int64_t b = bp + (lane >> 4);
    bool valid = b < blocks;
    int li = lane & 15;
    float v = valid ? w[b * 16 + li] : 0.f;
    double ab = fabs((double)v);
    for (int o = 8; o; o >>= 1) ab = fmax(ab, __shfl_xor_sync(0xffffffffu, ab, o));
    uint32_t sb = 0;
    if (ts != 0.f) sb = e4m3_encode_rn_satfinite(__ddiv_rn(ab, 6.0 * (double)ts));
    double d = __dmul_rn((double)e4m3_to_f32(sb), (double)ts);
    uint32_t q = 0;
    if (d != 0.0) q = e2m1_encode_rn_sat(__ddiv_rn((double)v, d));
    uint32_t q_hi = __shfl_down_sync(0xffffffffu, q, 1);
    if (valid) {
      if ((li & 1) == 0) codes[b * 8 + li / 2] = (uint8_t)(q | (q_hi << 4));
      if (li == 0) bscales[b] = (uint8_t)sb;
    }
  }
}

// MXFP4: one warp per 32-element block (one lane per element).  The block
// exponent is floor(log2 amax) - 2 (frexp, exact), clamped to [-127, 127];
// codes are the nearest E2M1 (ties to even, saturating at 6) of w / 2^exp,
// the division exact; an all-zero block gets exponent code 0.
__global__ void mxfp4_code_kernel(int64_t N, int64_t K, const float* __restrict__ w,
                                  uint8_t* __restrict__ codes, uint8_t* __restrict__ bscales) {
  const int64_t blocks = N * (K / 32);
  const int lane = threadIdx.x & 31;
  for (int64_t b = blockIdx.x * (int64_t)kWarps + (threadIdx.x >> 5); b < blocks;
       b += (int64_t)gridDim.x * kWarps) {
    const float v = w[b * 32 + lane];
    double ab = fabs((double)v);
    for (int o = 16; o; o >>= 1) ab = fmax(ab, __shfl_xor_sync(0xffffffffu, ab, o));
    uint32_t e = 0, q = 0;
    if (ab > 0.0) {
      int ex;
      frexp(ab, &ex);
      int se = (ex - 1) - 2;
      se = se < -127 ? -127 : (se > 127 ? 127 : se);
      e = (uint32_t)(se + 127);
      q = e2m1_encode_rn_sat(ldexp((double)v, -se));
    }
    const uint32_t q_hi = __shfl_down_sync(0xffffffffu, q, 1);
    if ((lane & 1) == 0) codes[b * 16 + lane / 2] = (uint8_t)(q | (q_hi << 4));
    if (lane == 0) bscales[b] = (uint8_t)e;
  }
}

__global__ void nvfp4_tscale_kernel(float* slot) {
  double amax = (double)__uint_as_float(*(const unsigned int*)slot);
  *slot = __double2float_rn(__ddiv_rn(amax, 6.0 * 448.0));
}

inline unsigned blocks_for(int64_t items, int per_block) {
  int64_t b = (items + per_block - 1) / per_block;
  if (b > 65535LL * 32) b = 65535LL * 32;
  return (unsigned)(b < 1 ? 1 : b);
}

}  // namespace

cudaError_t launch_quantize(int f, int64_t N, int64_t K, int G, const float* w, void* codes,
                            void* scales, void* aux, cudaStream_t st) {
  switch (f) {
    case INT4_SYM:
    case INT8_SYM:
    case INT2_SYM:
    case INT3_SYM:
      quant_sym_kernel<<<blocks_for(N * (K / G), kWarps), kWarps * 32, 0, st>>>(
          code_bits(f), N, K, G, w, (uint8_t*)codes, (uint16_t*)scales);
      break;
    case FP8_E4M3:
    case FP8_E5M2:
      quant_fp8_kernel<<<blocks_for(N * (K / G), kWarps), kWarps * 32, 0, st>>>(
          N, K, G, f == FP8_E5M2, w, (uint8_t*)codes, (float*)scales);
      break;
    case INT4_ASYM:
      quant_asym_kernel<<<blocks_for(N * (K / G), kWarps), kWarps * 32, 0, st>>>(
          N, K, G, w, (uint8_t*)codes, (uint16_t*)scales, (uint8_t*)aux);
      break;
    case CB4:
      cb4_norm_kernel<<<blocks_for(N, 128), 128, 0, st>>>(N, K, w, (uint16_t*)scales);
      cb4_code_kernel<<<blocks_for(N * K / 2, 256), 256, 0, st>>>(
          N, K, w, (const uint16_t*)scales, (const float*)aux, (uint8_t*)codes);
      break;
    case NVFP4: {
      cudaError_t e = cudaMemsetAsync(aux, 0, 4, st);
      if (e != cudaSuccess) return e;
      nvfp4_amax_kernel<<<blocks_for(N * K, 256 * 16), 256, 0, st>>>(N * K, w,
                                                                      (unsigned int*)aux);
      nvfp4_code_kernel<<<blocks_for(N * (K / 16), kWarps * 2), kWarps * 32, 0, st>>>(
          N, K, w, (const unsigned int*)aux, (uint8_t*)codes, (uint8_t*)scales);
      nvfp4_tscale_kernel<<<1, 1, 0, st>>>((float*)aux);
      break;
    }
    case MXFP4:
      mxfp4_code_kernel<<<blocks_for(N * (K / 32), kWarps), kWarps * 32, 0, st>>>(
          N, K, w, (uint8_t*)codes, (uint8_t*)scales);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace wq

// In-place LoRA merge into packed INT8 weights (piper-kernels README,
// Tensor.addmm_ on a ConvRot weight): weight = beta * weight + alpha *
// (mat1 @ mat2), requantized with the weight's unchanged group scales, either
// to the nearest code or, with a rounding seed, to one of the two adjacent
// codes with probability proportional to the distance to the other.
//
// One thread per weight element.  Every step is fp64 with explicit
// round-to-nearest operations (no contraction) in a fixed order (the dot
// product over the rank in increasing r), so each code is decided exactly as
// the definition states.  The random draw for element (n, k) is output
// n*K + k of the SplitMix64 stream keyed by the seed (Vigna's counter-based
// generator), its top 53 bits scaled by 2^-53.
#include "wq_internal.cuh"

namespace wq {

namespace {

__device__ __forceinline__ uint64_t splitmix64(uint64_t key, uint64_t i) {
  uint64_t z = key + (i + 1) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__global__ void addmm_requant_int8_kernel(int64_t N, int64_t K, int G, uint8_t* __restrict__ pw,
                                          const uint16_t* __restrict__ ps,
                                          const uint16_t* __restrict__ mat1,
                                          const uint16_t* __restrict__ mat2, int64_t R,
                                          double alpha, double beta, int use_seed,
                                          uint64_t seed) {
  const int64_t total = N * K;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = i / K, k = i - n * K;
    int64_t off;
    int sh;
    packed_loc(INT8_SYM, n, k, K, &off, &sh);
    const double s = (double)bf16_bits_to_f32(ps[packed_scale_idx(n, k / G, K / G)]);
    if (s == 0.0) {
      pw[off] = 128u;  // code 0, offset-binary
      continue;
    }
    double dot = 0.0;
    for (int64_t r = 0; r < R; ++r) {
      const double p = __dmul_rn((double)bf16_bits_to_f32(mat1[n * R + r]),
                                 (double)bf16_bits_to_f32(mat2[r * K + k]));
      dot = __dadd_rn(dot, p);
    }
    const int q0 = (int)pw[off] - 128;
    const double w = __dadd_rn(__dmul_rn(beta, __dmul_rn((double)q0, s)), __dmul_rn(alpha, dot));
    const double t = __ddiv_rn(w, s);
    double q;
    if (use_seed) {
      const double f = floor(t);
      const double u = (double)(splitmix64(seed, (uint64_t)i) >> 11) * 0x1p-53;
      q = f + (u < __dsub_rn(t, f) ? 1.0 : 0.0);
    } else {
      q = rint(t);
    }
    q = fmin(127.0, fmax(-127.0, q));
    pw[off] = (uint8_t)((int)q + 128);
  }
}

}  // namespace

cudaError_t launch_addmm_requant_int8(int64_t N, int64_t K, int G, void* pw, const void* ps,
                                      const void* mat1, const void* mat2, int64_t R,
                                      double alpha, double beta, int use_seed, uint64_t seed,
                                      cudaStream_t st) {
  const int64_t total = N * K;
  int64_t blocks = (total + 255) / 256;
  const int64_t cap = 32LL * device_sm_count();
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  addmm_requant_int8_kernel<<<(unsigned)blocks, 256, 0, st>>>(
      N, K, G, (uint8_t*)pw, (const uint16_t*)ps, (const uint16_t*)mat1, (const uint16_t*)mat2,
      R, alpha, beta, use_seed, seed);
  return cudaGetLastError();
}

}  // namespace wq

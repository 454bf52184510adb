// Per-token INT8 activation quantization for the activation-quantized linear
// (auto-round-lib README section 1, "Key Features": INT8 compute with the
// activations quantized dynamically per token, weights in INT8).
//
//   s_x[m] = fp32(amax_k |x[m, k]| / 127)
//   x_q[m, k] = clamp(round_half_even(x[m, k] / s_x[m]), -127, 127)   (0 if s_x = 0)
//
// The quotient amax / 127 is taken in fp64 and rounded once to fp32, and each
// x / s_x in fp64 (IEEE division) before the rounding to an integer, so the
// codes are the ones this definition gives, decision for decision.  One
// thread block per token row: a maximum pass, then a quantize pass, both
// with 16-byte loads of eight bf16 values.
#include "wq_internal.cuh"

namespace wq {

namespace {

__global__ void __launch_bounds__(256) quant_act_int8_kernel(const uint4* __restrict__ x,
                                                            int64_t K8, uint2* __restrict__ xq,
                                                            float* __restrict__ sx) {
  __shared__ float red[8];
  __shared__ float s_row;
  const int64_t m = blockIdx.x;
  const uint4* row = x + m * K8;
  float amax = 0.f;
  for (int64_t i = threadIdx.x; i < K8; i += blockDim.x) {
    const uint4 v = __ldg(row + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      amax = fmaxf(amax, fabsf(__uint_as_float(w[j] << 16)));
      amax = fmaxf(amax, fabsf(__uint_as_float(w[j] & 0xFFFF0000u)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  if (threadIdx.x == 0) {
    float a = 0.f;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) a = fmaxf(a, red[i]);
    const float s = __double2float_rn((double)a / 127.0);
    s_row = s;
    sx[m] = s;
  }
  __syncthreads();
  const float s = s_row;
  const double sd = (double)s;
  for (int64_t i = threadIdx.x; i < K8; i += blockDim.x) {
    const uint4 v = __ldg(row + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t out[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t h = (j & 1) ? (w[j >> 1] & 0xFFFF0000u) : (w[j >> 1] << 16);
      int q = 0;
      if (s != 0.f) {
        q = __double2int_rn((double)__uint_as_float(h) / sd);
        q = q > 127 ? 127 : (q < -127 ? -127 : q);
      }
      out[j >> 2] |= ((uint32_t)q & 0xFFu) << (8 * (j & 3));
    }
    xq[m * K8 + i] = make_uint2(out[0], out[1]);
  }
}

}  // namespace

cudaError_t launch_quant_act_int8(const void* x, int64_t M, int64_t K, void* xq, float* sx,
                                  cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  quant_act_int8_kernel<<<(unsigned)M, 256, 0, st>>>((const uint4*)x, K / 8, (uint2*)xq, sx);
  return cudaGetLastError();
}

}  // namespace wq

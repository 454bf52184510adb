// SwiGLU input of the linear (piper-kernels README, convrot_linear with
// input_activation="swiglu"): rows of x2 hold [up | gate], K values each;
// the activation is a = bf16(up * silu(gate)), silu(g) = g / (1 + e^-g).
// The page's general path materializes this activation and then runs the
// ordinary linear; this kernel is that materialization for the prefill path
// (the decode kernel applies the same step to its staged X slice instead).
// Elementwise and HBM-bound: 16-byte loads of up and gate, one 16-byte store.
#include "wq_frag.cuh"
#include "wq_internal.cuh"

namespace wq {

namespace {

// The library's own scratch for the materialized activation of
// wq_linear_swiglu_static: a file-scope device array (one per device,
// reserved when the module loads), so that entry point allocates nothing.
static __device__ __align__(256) uint8_t g_swiglu_scratch[kSwigluStaticScratchBytes];

__global__ void __launch_bounds__(256) swiglu_kernel(const uint4* __restrict__ x2, int64_t M,
                                                     int64_t K8, uint4* __restrict__ a) {
  const int64_t total = M * K8;  // 16-byte chunks of the output
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t m = i / K8, c = i - m * K8;
    const uint4 u = __ldg(x2 + m * 2 * K8 + c);
    const uint4 g = __ldg(x2 + m * 2 * K8 + K8 + c);
    a[i] = make_uint4(swiglu_pair(u.x, g.x), swiglu_pair(u.y, g.y), swiglu_pair(u.z, g.z),
                      swiglu_pair(u.w, g.w));
  }
}

}  // namespace

cudaError_t static_swiglu_scratch(void** ptr, size_t* bytes) {
  *bytes = kSwigluStaticScratchBytes;
  return cudaGetSymbolAddress(ptr, g_swiglu_scratch);
}

cudaError_t launch_swiglu(const void* x2, int64_t M, int64_t K, void* a, cudaStream_t st) {
  const int64_t K8 = K / 8;
  const int64_t total = M * K8;
  int64_t blocks = (total + 255) / 256;
  const int64_t cap = 16LL * device_sm_count();  // a few waves, grid-stride beyond
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  swiglu_kernel<<<(unsigned)blocks, 256, 0, st>>>((const uint4*)x2, M, K8, (uint4*)a);
  return cudaGetLastError();
}

}  // namespace wq

// Prefill path (M > 16).  Placeholder that runs the decode kernel over
// 16-token slices of X; replaced by the tcgen05 kernel.
#include "wq_internal.cuh"

namespace wq {

cudaError_t launch_prefill(const LinearArgs& a) {
  for (int64_t m0 = 0; m0 < a.M; m0 += 16) {
    LinearArgs s = a;
    s.M = (a.M - m0) < 16 ? (a.M - m0) : 16;
    s.x = (const uint16_t*)a.x + m0 * a.K;
    s.out = (uint16_t*)a.out + m0 * a.N;
    cudaError_t e = launch_decode(s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace wq

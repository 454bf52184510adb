// Decode kernel instantiations for CB4, NVFP4 (the template is in
// wq_decode_kernel.cuh; split over several files so that they compile in
// parallel).
#include "wq_decode_kernel.cuh"

namespace wq {

cudaError_t launch_decode_k2(int fmt, const DecodeParams& p, int nt, int rt, int kw, int d,
                             int grid, cudaStream_t st) {
  switch (fmt) {
    case CB4: return launch_fmt<CB4>(p, nt, rt, kw, d, grid, st);
    case NVFP4: return launch_fmt<NVFP4>(p, nt, rt, kw, d, grid, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace wq

// Decode kernel instantiations for MXFP4, FP8_E4M3, FP8_E5M2 (the template is in
// wq_decode_kernel.cuh; split over several files so that they compile in
// parallel).
#include "wq_decode_kernel.cuh"

namespace wq {

cudaError_t launch_decode_k3(int fmt, const DecodeParams& p, int nt, int rt, int kw, int d,
                             int grid, cudaStream_t st) {
  switch (fmt) {
    case MXFP4: return launch_fmt<MXFP4>(p, nt, rt, kw, d, grid, st);
    case FP8_E4M3: return launch_fmt<FP8_E4M3>(p, nt, rt, kw, d, grid, st);
    case FP8_E5M2: return launch_fmt<FP8_E5M2>(p, nt, rt, kw, d, grid, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace wq

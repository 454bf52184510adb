// Decode kernel instantiations for INT4_SYM, INT4_ASYM (the template is in
// wq_decode_kernel.cuh; split over several files so that they compile in
// parallel).
#include "wq_decode_kernel.cuh"

namespace wq {

cudaError_t launch_decode_k0(int fmt, const DecodeParams& p, int nt, int rt, int kw, int d,
                             int grid, cudaStream_t st) {
  switch (fmt) {
    case INT4_SYM: return launch_fmt<INT4_SYM>(p, nt, rt, kw, d, grid, st);
    case INT4_ASYM: return launch_fmt<INT4_ASYM>(p, nt, rt, kw, d, grid, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace wq

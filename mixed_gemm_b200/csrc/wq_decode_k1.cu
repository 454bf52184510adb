// Decode kernel instantiations for INT8_SYM, INT2_SYM, INT3_SYM (the template is in
// wq_decode_kernel.cuh; split over several files so that they compile in
// parallel).
#include "wq_decode_kernel.cuh"

namespace wq {

cudaError_t launch_decode_k1(int fmt, const DecodeParams& p, int nt, int rt, int kw, int d,
                             int grid, cudaStream_t st) {
  switch (fmt) {
    case INT8_SYM: return launch_fmt<INT8_SYM>(p, nt, rt, kw, d, grid, st);
    case INT2_SYM: return launch_fmt<INT2_SYM>(p, nt, rt, kw, d, grid, st);
    case INT3_SYM: return launch_fmt<INT3_SYM>(p, nt, rt, kw, d, grid, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace wq

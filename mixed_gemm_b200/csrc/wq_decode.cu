// Decode path (M <= 16): stream the packed weight once from HBM.
//
// Work split.  A CTA owns RT row tiles (16 output features each) and a slice
// of K; a cluster of CS CTAs covers all of K for those rows; the KW warps of a
// CTA split the CTA's K slice again.  Every lane issues one 16-byte
// no-L1-allocate load per row tile and 512-byte block, which holds exactly its
// tensor-core A fragments for that block (layout in wq_internal.cuh), and one
// 16-byte load of the 8 matching activations per token row.  Codes become
// bf16 in registers (magic-number nibble conversion for INT4, fp32 magic for
// INT8, an integer-multiply bit construction for NVFP4, byte-permute table
// lookups for CB4: a bf16 high part and a bf16 remainder per centroid, two
// products) and feed mma.sync.m16n8k16 with the W rows as the 16-row
// operand and the (<= 16) tokens as the 8-column operand.  INT group scales
// are applied once per group to an fp32 group accumulator (so the bf16
// fragments are the exact integer codes); NVFP4 block scales are multiplied
// into the fragments (the product e2m1*e4m3 is exact in bf16); the CB4 row
// norm and the NVFP4 tensor scale are applied in the epilogue.  The weight
// stream and its scales are requested before griddepcontrol.wait
// (programmatic dependent launch); after it, thread 0 stages the X slice with
// one bulk copy (cp.async.bulk) per token row onto an mbarrier.  Partial sums
// are reduced across warps through shared memory and across the cluster
// through distributed shared memory (no global workspace), then rank 0
// applies fold + bias, rounds to bf16 and stores.
//
// Sources: OrbitQuant card "Benchmark" (skinny batches are decode-bound; the
// Metal path dispatches a skinny GEMV for up to four rows with decoded weight
// segments reused across the batch); Petit README "Techniques and
// performance" (batches below 16 are the small-batch regime, weights shuffled
// offline for cheap dequantization).
#include <mutex>

#include "wq_decode_kernel.cuh"

namespace wq {

// Error word of the decode kernel: bit 128 when the wait for its staged
// activation slice ran out (that CTA then stores nothing).
__device__ unsigned int g_wq_decode_error;

namespace {

std::mutex g_err_mutex;
unsigned* g_err_ptr[64];

// device address of the error word on the current device
cudaError_t decode_error_word(unsigned** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_err_mutex);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_wq_decode_error);
    if (e != cudaSuccess) return e;
    g_err_ptr[dev] = (unsigned*)p;
  }
  *ptr = g_err_ptr[dev];
  return cudaSuccess;
}

}  // namespace

cudaError_t read_decode_error(unsigned* value, bool clear) {
  cudaError_t e = cudaMemcpyFromSymbol(value, g_wq_decode_error, sizeof(unsigned));
  if (e != cudaSuccess || !clear) return e;
  unsigned z = 0;
  return cudaMemcpyToSymbol(g_wq_decode_error, &z, sizeof(unsigned));
}

cudaError_t launch_decode(const LinearArgs& a) {
  DecodeParams p;
  p.x = (const uint16_t*)a.x;
  p.w = (const uint4*)a.w;
  p.scales = a.scales;
  p.aux = a.aux;
  p.bias = (const uint16_t*)a.bias;
  p.out = (uint16_t*)a.out;
  p.N = (int)a.N;
  p.K = (int)a.K;
  p.G = a.G;
  // a grouped launch takes token chunks of up to 8 (mean rows per expert
  // <= 8) or 16 per CTA; Mc is the rows a CTA stages
  const int64_t Mc = a.offsets ? ((a.M + a.E - 1) / a.E <= 8 ? 8 : 16) : a.M;
  p.M = (int)Mc;
  p.offsets = a.offsets;
  p.E = a.offsets ? a.E : 1;
  p.T = (int)a.M;
  size_t wbytes = 0, sbytes = 0, abytes = 0;
  wq_packed_sizes(a.fmt, a.N, a.K, a.G, &wbytes, &sbytes, &abytes);
  p.w_stride = a.offsets ? (int64_t)wbytes : 0;
  p.scale_stride = a.offsets ? a.scale_stride : 0;
  p.aux_stride = a.offsets ? a.aux_stride : 0;
  const int nt = Mc <= 8 ? 1 : 2;
  const int64_t tiles = a.N / 16;
  // Launch shape, from a sweep of row tiles per CTA, warps per CTA, cluster
  // size and ring depth over the 4096^2 INT4, 3072^2 codebook, 8192^2 FP8
  // and 28672 x 8192 NVFP4 layers at M = 1..16 (graph replay, weights past
  // L2): eight warps per CTA, two row tiles per CTA, K split over a cluster
  // of at least two CTAs and enough of them to keep each CTA's staged
  // activation slice near 64 KB (one 8-warp CTA per SM would otherwise be
  // all that fits at M = 16, K = 8192), and a ring of eight blocks per row
  // tile at M <= 8 (more weight bytes in flight; at M > 8 the second token
  // tile's accumulators make the deeper ring spill).  Against the previous
  // heuristic (about four 4-warp CTAs per SM) this measured 5-38% faster on
  // every shape of the sweep.
  int rt = (tiles % 2 == 0) ? 2 : 1;
#ifdef WQ_TUNING
  if (const char* e = getenv("WQ_DECODE_RT")) rt = atoi(e);
#endif
  const int64_t rowgroups = tiles / rt;
  const int kb = block_k(a.fmt);
  const int64_t nblk = a.K / kb;
  // short K: fewer warps, each with some blocks.  A grouped launch has many
  // small (expert, chunk) tiles and no weight prefetch ahead of the
  // dependency wait: four warps and no K split (measured on 64 experts of
  // 2048 x 2048 with 512 routed rows: 83 us against 202 with the dense shape)
  int kw = (nblk >= 16 && !a.offsets) ? 8 : 4;
#ifdef WQ_TUNING
  if (const char* e = getenv("WQ_DECODE_KW")) kw = atoi(e) == 8 ? 8 : 4;
#endif
  const int64_t x_bytes_all = Mc * a.K * 2 * (a.swiglu ? 2 : 1);
  int64_t cs = (x_bytes_all + 65535) / 65536;
  if (cs < 2) cs = a.offsets ? 1 : 2;
  if (cs > 8) cs = 8;
  if (cs > nblk / kw) cs = nblk / kw;  // keep every warp busy
  if (cs < 1) cs = 1;
#ifdef WQ_TUNING
  if (const char* e = getenv("WQ_DECODE_CS")) cs = atoi(e);
#endif
  // weight ring depth per row tile (two instantiated: 4 and 8)
  int d = (nt == 1 && rt <= 2 && !a.offsets) ? 8 : 4;
#ifdef WQ_TUNING
  if (const char* e = getenv("WQ_DECODE_D")) d = atoi(e) == 8 ? 8 : 4;
#endif
  const int64_t max_blocks = (nblk + cs - 1) / cs;
  const int64_t stride = ((max_blocks * kb * 2 + 127) / 128) * 128 + 64;
  // K too large for the staged activation slice (the SwiGLU input stages up
  // and gate): nothing launched, the caller takes the prefill path
  if (stride * Mc * (a.swiglu ? 2 : 1) > 200 * 1024) return cudaErrorNotSupported;
  p.cs = (int)cs;
  p.xs_stride = (int)stride;
  p.xs_bytes = (int)(stride * Mc);
  // staged side data per row tile: a K range of max_blocks*kb may touch one
  // more group than it spans
  p.gshift = 0;
  if (is_grouped_fmt(a.fmt)) {
    while ((1 << p.gshift) < a.G) ++p.gshift;
    p.side_rows = (int)((max_blocks * kb + a.G - 1) / a.G + 1);
    p.side_bytes = rt * p.side_rows * (a.fmt == INT4_ASYM ? 40 : is_fp8(a.fmt) ? 64 : 32);
  } else if (a.fmt == NVFP4 || a.fmt == MXFP4) {
    p.side_rows = (int)(max_blocks * kb / (a.fmt == NVFP4 ? 16 : 32));
    p.side_bytes = rt * p.side_rows * 16 + 1024;  // block scales + code table
  } else {
    p.side_rows = 0;
    p.side_bytes = 0;
  }
  p.side_bytes = (p.side_bytes + 15) & ~15;
  const int64_t warp_partials = (int64_t)kw * rt * nt * 4 * 32 * 4;
  p.swiglu = a.swiglu ? 1 : 0;
#ifdef WQ_FAULT_TEST
  p.fault_skip_x = getenv("WQ_FAULT_DECODE_SKIP_X") ? atoi(getenv("WQ_FAULT_DECODE_SKIP_X")) : 0;
#endif
  int64_t region = (int64_t)p.xs_bytes * (a.swiglu ? 2 : 1) + p.side_bytes;
  if (region < warp_partials) region = warp_partials;
  p.red_off = (int)((region + 15) & ~15LL);
  p.bar_off = (int)(p.red_off + cs * rt * nt * 4 * 32 * 4);
  // the X-slice barrier (8 bytes) and, grouped, the schedule entry after it
  if (p.bar_off + 32 > 227 * 1024) return cudaErrorNotSupported;
  const int grid = (int)(rowgroups * cs);
  // grouped: an upper bound on the schedule's chunks (ceil(T / Mc) + E)
  const int64_t ytiles = a.offsets ? (a.M + Mc - 1) / Mc + a.E : 1;
  if (ytiles > 65535) return cudaErrorNotSupported;
  p.ytiles = (int)ytiles;
  unsigned* err = nullptr;
  cudaError_t e = decode_error_word(&err);
  if (e != cudaSuccess) return e;
  p.err = err;
  switch (a.fmt) {
    case INT4_SYM:
    case INT4_ASYM: return launch_decode_k0(a.fmt, p, nt, rt, kw, d, grid, a.stream);
    case INT8_SYM:
    case INT2_SYM:
    case INT3_SYM: return launch_decode_k1(a.fmt, p, nt, rt, kw, d, grid, a.stream);
    case CB4:
    case NVFP4: return launch_decode_k2(a.fmt, p, nt, rt, kw, d, grid, a.stream);
    case MXFP4:
    case FP8_E4M3:
    case FP8_E5M2: return launch_decode_k3(a.fmt, p, nt, rt, kw, d, grid, a.stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace wq

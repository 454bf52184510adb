// C ABI: argument checks, dispatch and the host-side helpers declared in
// include/wq.h.  Every check runs on the host before anything is launched;
// nothing here allocates device memory.
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "wq_internal.cuh"

namespace wq {

cudaError_t launch_addmm_requant_int8(int64_t N, int64_t K, int G, void* pw, const void* ps,
                                      const void* mat1, const void* mat2, int64_t R,
                                      double alpha, double beta, int use_seed, uint64_t seed,
                                      cudaStream_t st);

namespace {

bool aligned(const void* p, uintptr_t a) { return ((uintptr_t)p % a) == 0; }

// [p, p + pb) and [q, q + qb) intersect (a NULL pointer intersects nothing)
bool overlap(const void* p, int64_t pb, const void* q, int64_t qb) {
  if (!p || !q) return false;
  const uintptr_t p0 = (uintptr_t)p, q0 = (uintptr_t)q;
  return p0 < q0 + (uintptr_t)qb && q0 < p0 + (uintptr_t)pb;
}

// Shape / format checks shared by every entry point.
int check_shape(int f, int64_t N, int64_t K, int G) {
  if (f < INT4_SYM || f > INT3_SYM) return WQ_ERR_INVALID_ARG;
  if (N <= 0 || K <= 0) return WQ_ERR_INVALID_ARG;
  if (N % 16 || K % 64) return WQ_ERR_INVALID_ARG;
  if (N > (1LL << 30) || K > (1LL << 24) || N * K > (1LL << 40)) return WQ_ERR_INVALID_ARG;
  if (is_grouped_fmt(f)) {
    if (G != 32 && G != 64 && G != 128 && G != 256) return WQ_ERR_INVALID_ARG;
    if (K % G) return WQ_ERR_INVALID_ARG;
  } else if (f == NVFP4) {
    if (G != 0 && G != 16) return WQ_ERR_INVALID_ARG;
  } else if (f == MXFP4) {
    if (G != 0 && G != 32) return WQ_ERR_INVALID_ARG;
  }
  return WQ_OK;
}

int effective_group(int f, int G) {
  return f == NVFP4 ? 16 : f == MXFP4 ? 32 : (f == CB4 ? 0 : G);
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? WQ_OK : WQ_ERR_CUDA; }

// Checks shared by the linear entry points; x holds x_cols bf16 values per row.
int check_linear(const void* x, int64_t x_cols, const void* pw, const void* scales,
                 const void* aux, const void* bias, int64_t M, int64_t N, int64_t K, int f,
                 int& G, void* out) {
  int st = check_shape(f, N, K, G);
  if (st) return st;
  if (M < 0 || M > (1LL << 24)) return WQ_ERR_INVALID_ARG;
  G = effective_group(f, G);
  bool need_aux = f == INT4_ASYM || f == CB4 || f == NVFP4;
  if (!x || !pw || !scales || !out || (need_aux && !aux)) return WQ_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(pw, 16) || !aligned(scales, 16) || !aligned(out, 16) ||
      (bias && !aligned(bias, 16)) || (aux && !aligned(aux, (f == INT4_ASYM) ? 16 : 4)))
    return WQ_ERR_ALIGNMENT;
  // the output must not overlap an input
  size_t wb = 0, sb = 0, ab = 0;
  wq_packed_sizes(f, N, K, G, &wb, &sb, &ab);
  if (M > 0 && (overlap(out, M * N * 2, x, M * x_cols * 2) || overlap(out, M * N * 2, pw, wb) ||
                overlap(out, M * N * 2, scales, sb) || overlap(out, M * N * 2, aux, ab) ||
                overlap(out, M * N * 2, bias, N * 2)))
    return WQ_ERR_INVALID_ARG;
  return WQ_OK;
}

std::mutex g_sm_mutex;
int g_sm_count[64];
bool g_sm_known[64];

// A word of device memory that only the stream fence below writes.
__device__ unsigned g_wq_stream_fence;
std::mutex g_fence_mutex;
void* g_fence_ptr[64];

// Kernel attributes are per device: one entry per (device, kernel) that has
// been given the larger shared-memory limit; a failed attempt is not cached.
std::mutex g_attr_mutex;
struct AttrEntry {
  int dev;
  const void* fn;
};
AttrEntry g_attr_done[1024];
int g_attr_count = 0;

}  // namespace

cudaError_t end_weight_write(cudaStream_t st) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  void* p = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_fence_mutex);
    if (!g_fence_ptr[dev]) {
      e = cudaGetSymbolAddress(&g_fence_ptr[dev], g_wq_stream_fence);
      if (e != cudaSuccess) {
        g_fence_ptr[dev] = nullptr;
        return e;
      }
    }
    p = g_fence_ptr[dev];
  }
  return cudaMemsetAsync(p, 0, sizeof(unsigned), st);
}

cudaError_t ensure_max_dynamic_smem(const void* fn, int bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(g_attr_mutex);
  for (int i = 0; i < g_attr_count; ++i)
    if (g_attr_done[i].dev == dev && g_attr_done[i].fn == fn) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  if (g_attr_count < 1024) g_attr_done[g_attr_count++] = AttrEntry{dev, fn};
  return cudaSuccess;
}

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  std::lock_guard<std::mutex> lk(g_sm_mutex);
  if (dev >= 0 && dev < 64 && g_sm_known[dev]) return g_sm_count[dev];
  int n = 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n = 148;
  if (dev >= 0 && dev < 64) {
    g_sm_count[dev] = n;
    g_sm_known[dev] = true;
  }
  return n;
}

}  // namespace wq

using namespace wq;

extern "C" {

const char* wq_status_string(int s) {
  switch (s) {
    case WQ_OK: return "ok";
    case WQ_ERR_INVALID_ARG: return "invalid argument";
    case WQ_ERR_UNSUPPORTED: return "unsupported";
    case WQ_ERR_ALIGNMENT: return "misaligned pointer";
    case WQ_ERR_CUDA: return "CUDA error";
    case WQ_ERR_DEVICE_CHECK: return "device-side check failed";
  }
  return "unknown status";
}

int wq_canonical_sizes(int f, int64_t N, int64_t K, int G, size_t* cb, size_t* sb, size_t* ab) {
  int st = check_shape(f, N, K, G);
  if (st) return st;
  G = effective_group(f, G);
  size_t c = 0, s = 0, a = 0;
  switch (f) {
    case INT4_SYM: c = N * K / 2; s = 2 * N * (K / G); break;
    case INT4_ASYM: c = N * K / 2; s = 2 * N * (K / G); a = N * (K / G); break;
    case INT8_SYM: c = N * K; s = 2 * N * (K / G); break;
    case INT2_SYM: c = N * K / 4; s = 2 * N * (K / G); break;
    case INT3_SYM: c = N * K * 3 / 8; s = 2 * N * (K / G); break;
    case FP8_E4M3:
    case FP8_E5M2: c = N * K; s = 4 * N * (K / G); break;
    case CB4: c = N * K / 2; s = 2 * N; a = 64; break;
    case NVFP4: c = N * K / 2; s = N * (K / 16); a = 4; break;
    case MXFP4: c = N * K / 2; s = N * (K / 32); a = 0; break;
  }
  if (cb) *cb = c;
  if (sb) *sb = s;
  if (ab) *ab = a;
  return WQ_OK;
}

int wq_packed_sizes(int f, int64_t N, int64_t K, int G, size_t* wb, size_t* sb, size_t* ab) {
  int st = wq_canonical_sizes(f, N, K, G, wb, sb, ab);
  if (st) return st;
  if (f == INT4_ASYM && ab) *ab = N * (K / G) / 2;
  return WQ_OK;
}

int wq_pack(int f, int64_t N, int64_t K, int G, const void* codes, const void* scales,
            const void* aux, void* pw, void* ps, void* pa, void* stream) {
  int st = check_shape(f, N, K, G);
  if (st) return st;
  G = effective_group(f, G);
  bool need_aux = f == INT4_ASYM || f == CB4 || f == NVFP4;
  if (!codes || !scales || !pw || !ps || (need_aux && (!aux || !pa))) return WQ_ERR_INVALID_ARG;
  cudaError_t e = launch_pack(f, N, K, G, codes, scales, aux, pw, ps, pa, (cudaStream_t)stream);
  if (e == cudaSuccess) e = end_weight_write((cudaStream_t)stream);
  return cuda_status(e);
}

int wq_unpack(int f, int64_t N, int64_t K, int G, const void* pw, const void* ps, const void* pa,
              void* codes, void* scales, void* aux, void* stream) {
  int st = check_shape(f, N, K, G);
  if (st) return st;
  G = effective_group(f, G);
  bool need_aux = f == INT4_ASYM || f == CB4 || f == NVFP4;
  if (!codes || !scales || !pw || !ps || (need_aux && (!aux || !pa))) return WQ_ERR_INVALID_ARG;
  return cuda_status(launch_unpack(f, N, K, G, pw, ps, pa, codes, scales, aux, (cudaStream_t)stream));
}

int wq_dequant(int f, int64_t N, int64_t K, int G, const void* pw, const void* ps, const void* pa,
               float* out, void* stream) {
  int st = check_shape(f, N, K, G);
  if (st) return st;
  G = effective_group(f, G);
  bool need_aux = f == INT4_ASYM || f == CB4 || f == NVFP4;
  if (!pw || !ps || !out || (need_aux && !pa)) return WQ_ERR_INVALID_ARG;
  return cuda_status(launch_dequant(f, N, K, G, pw, ps, pa, out, (cudaStream_t)stream));
}

int wq_quantize(int f, int64_t N, int64_t K, int G, const float* w, void* codes, void* scales,
                void* aux, void* stream) {
  int st = check_shape(f, N, K, G);
  if (st) return st;
  G = effective_group(f, G);
  bool need_aux = f == INT4_ASYM || f == CB4 || f == NVFP4;
  if (!w || !codes || !scales || (need_aux && !aux)) return WQ_ERR_INVALID_ARG;
  if (!aligned(w, 4) || (aux && !aligned(aux, 4))) return WQ_ERR_ALIGNMENT;
  cudaError_t e = launch_quantize(f, N, K, G, w, codes, scales, aux, (cudaStream_t)stream);
  if (e == cudaSuccess) e = end_weight_write((cudaStream_t)stream);
  return cuda_status(e);
}

int wq_linear(const void* x, const void* pw, const void* scales, const void* aux, const void* bias,
              int64_t M, int64_t N, int64_t K, int f, int G, void* out, void* stream) {
  int st = check_linear(x, K, pw, scales, aux, bias, M, N, K, f, G, out);
  if (st) return st;
  if (M == 0) return WQ_OK;
  LinearArgs a;
  a.x = x;
  a.w = pw;
  a.scales = scales;
  a.aux = aux;
  a.bias = bias;
  a.out = out;
  a.M = M;
  a.N = N;
  a.K = K;
  a.fmt = f;
  a.G = G;
  a.stream = (cudaStream_t)stream;
  cudaError_t e;
  if (M <= 16) {
    e = launch_decode(a);
    if (e == cudaErrorNotSupported) e = launch_prefill(a);  // K too long to stage
  } else {
    e = launch_prefill(a);
  }
  return cuda_status(e);
}

int wq_linear_grouped(const void* x, const void* const* pw, const void* const* scales,
                      const void* const* aux, const void* const* bias, const int64_t* offsets,
                      int64_t E, int64_t N, int64_t K, int f, int G, void* out, void* stream) {
  if (!offsets || !pw || !scales || E <= 0 || E > (1 << 20)) return WQ_ERR_INVALID_ARG;
  if (offsets[0] != 0) return WQ_ERR_INVALID_ARG;
  for (int64_t e = 0; e < E; ++e)
    if (offsets[e + 1] < offsets[e]) return WQ_ERR_INVALID_ARG;
  const int64_t T = offsets[E];
  // every expert's arguments are checked before anything is launched
  for (int64_t e = 0; e < E; ++e) {
    const int64_t m = offsets[e + 1] - offsets[e];
    int g = G;
    int st = check_linear(x, K, pw[e], scales[e], aux ? aux[e] : nullptr, bias ? bias[e] : nullptr,
                          T, N, K, f, g, out);
    if (st) return st;
    if (m < 0) return WQ_ERR_INVALID_ARG;
  }
  for (int64_t e = 0; e < E; ++e) {
    const int64_t m0 = offsets[e], m = offsets[e + 1] - m0;
    if (m == 0) continue;
    const uint16_t* xe = (const uint16_t*)x + m0 * K;
    uint16_t* ye = (uint16_t*)out + m0 * N;
    int st = wq_linear(xe, pw[e], scales[e], aux ? aux[e] : nullptr, bias ? bias[e] : nullptr, m,
                       N, K, f, G, ye, stream);
    if (st) return st;
  }
  return WQ_OK;
}

int wq_linear_grouped_dev(const void* x, const void* pw, const void* scales, const void* aux,
                          const void* bias, const int64_t* offsets, int64_t E, int64_t T,
                          int64_t N, int64_t K, int f, int G, void* out, void* stream) {
  int st = check_shape(f, N, K, G);
  if (st) return st;
  G = effective_group(f, G);
  if (E <= 0 || E > (1 << 20) || T < 0 || T > (1LL << 24)) return WQ_ERR_INVALID_ARG;
  const bool need_aux = f == INT4_ASYM || f == CB4 || f == NVFP4;
  if (!x || !pw || !scales || !out || !offsets || (need_aux && !aux)) return WQ_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(pw, 16) || !aligned(scales, 16) || !aligned(out, 16) ||
      !aligned(offsets, 8) || (bias && !aligned(bias, 16)) ||
      (aux && !aligned(aux, (f == INT4_ASYM) ? 16 : 4)))
    return WQ_ERR_ALIGNMENT;
  size_t wb = 0, sb = 0, ab = 0;
  wq_packed_sizes(f, N, K, G, &wb, &sb, &ab);
  const int64_t ob = T * N * 2;
  if (T > 0 && (overlap(out, ob, x, T * K * 2) || overlap(out, ob, pw, E * (int64_t)wb) ||
                overlap(out, ob, scales, E * (int64_t)sb) ||
                overlap(out, ob, aux, E * (int64_t)ab) || overlap(out, ob, bias, E * N * 2) ||
                overlap(out, ob, offsets, (E + 1) * 8)))
    return WQ_ERR_INVALID_ARG;
  if (T == 0) return WQ_OK;
  LinearArgs a;
  a.x = x;
  a.w = pw;
  a.scales = scales;
  a.aux = aux;
  a.bias = bias;
  a.out = out;
  a.M = T;
  a.N = N;
  a.K = K;
  a.fmt = f;
  a.G = G;
  a.stream = (cudaStream_t)stream;
  a.offsets = offsets;
  a.E = (int)E;
  a.scale_stride = (int64_t)sb;
  a.aux_stride = (int64_t)ab;
  // decode-like routing (at most 16 rows per expert on average): the decode
  // kernel over (expert, chunk of 8 or 16 rows) tiles; otherwise, or for a K
  // too long for its staged slice, the tcgen05 kernel's grouped mode
  cudaError_t e = cudaErrorNotSupported;
  if ((T + E - 1) / E <= 16) e = launch_decode(a);
  if (e == cudaErrorNotSupported) e = launch_prefill_grouped(a);
  return e == cudaErrorNotSupported ? WQ_ERR_UNSUPPORTED : cuda_status(e);
}

int wq_linear_swiglu(const void* x2, const void* pw, const void* scales, const void* aux,
                     const void* bias, int64_t M, int64_t N, int64_t K, int f, int G,
                     void* workspace, size_t workspace_bytes, void* out, void* stream) {
  int st = check_linear(x2, 2 * K, pw, scales, aux, bias, M, N, K, f, G, out);
  if (st) return st;
  const bool decode = M <= 16;
  // the materialized activation [M, K] bf16 lives in the caller's workspace
  auto check_ws = [&]() -> int {
    if (!workspace || workspace_bytes < (size_t)(M * K * 2)) return WQ_ERR_INVALID_ARG;
    if (!aligned(workspace, 16)) return WQ_ERR_ALIGNMENT;
    size_t wb = 0, sb = 0, ab = 0;
    wq_packed_sizes(f, N, K, G, &wb, &sb, &ab);
    const int64_t w = M * K * 2;
    if (overlap(workspace, w, x2, M * 2 * K * 2) || overlap(workspace, w, out, M * N * 2) ||
        overlap(workspace, w, pw, wb) || overlap(workspace, w, scales, sb) ||
        overlap(workspace, w, aux, ab) || overlap(workspace, w, bias, N * 2))
      return WQ_ERR_INVALID_ARG;
    return WQ_OK;
  };
  if (!decode && (st = check_ws()) != WQ_OK) return st;
  if (M == 0) return WQ_OK;
  LinearArgs a;
  a.x = x2;
  a.w = pw;
  a.scales = scales;
  a.aux = aux;
  a.bias = bias;
  a.out = out;
  a.M = M;
  a.N = N;
  a.K = K;
  a.fmt = f;
  a.G = G;
  a.stream = (cudaStream_t)stream;
  if (decode) {
    a.swiglu = true;
    cudaError_t e = launch_decode(a);
    if (e != cudaErrorNotSupported) return cuda_status(e);
    // K too long to stage both halves: materialize, if a workspace was given
    a.swiglu = false;
    if (!workspace) return WQ_ERR_UNSUPPORTED;
    if ((st = check_ws()) != WQ_OK) return st;
  }
  cudaError_t e = launch_swiglu(x2, M, K, workspace, a.stream);
  if (e != cudaSuccess) return cuda_status(e);
  a.x = workspace;
  return cuda_status(launch_prefill(a));
}

int wq_linear_swiglu_static(const void* x2, const void* pw, const void* scales, const void* aux,
                            const void* bias, int64_t M, int64_t N, int64_t K, int f, int G,
                            void* out, void* stream) {
  int st = check_linear(x2, 2 * K, pw, scales, aux, bias, M, N, K, f, G, out);
  if (st) return st;
  const bool fits = (uint64_t)M * (uint64_t)K * 2u <= kSwigluStaticScratchBytes;
  if (M <= 16 && !fits)  // the decode path needs no scratch unless K is very long
    return wq_linear_swiglu(x2, pw, scales, aux, bias, M, N, K, f, G, nullptr, 0, out, stream);
  if (!fits) return WQ_ERR_UNSUPPORTED;
  void* ws = nullptr;
  size_t ws_bytes = 0;
  if (static_swiglu_scratch(&ws, &ws_bytes) != cudaSuccess) return WQ_ERR_CUDA;
  return wq_linear_swiglu(x2, pw, scales, aux, bias, M, N, K, f, G, ws, ws_bytes, out, stream);
}

int wq_linear_a8_workspace_size(int64_t M, int64_t K, size_t* bytes) {
  if (!bytes || M < 0 || M > (1LL << 24) || K <= 0 || K > (1LL << 24)) return WQ_ERR_INVALID_ARG;
  *bytes = (size_t)(((M * K + 255) & ~255LL) + 4 * M);
  return WQ_OK;
}

int wq_quantize_act_int8(const void* x, int64_t M, int64_t K, void* xq, void* sx, void* stream) {
  if (M < 0 || M > (1LL << 24) || K <= 0 || K > (1LL << 24) || K % 8) return WQ_ERR_INVALID_ARG;
  if (M == 0) return WQ_OK;
  if (!x || !xq || !sx) return WQ_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(xq, 16) || !aligned(sx, 4)) return WQ_ERR_ALIGNMENT;
  if (overlap(xq, M * K, x, M * K * 2) || overlap(sx, M * 4, x, M * K * 2) ||
      overlap(sx, M * 4, xq, M * K))
    return WQ_ERR_INVALID_ARG;
  return cuda_status(launch_quant_act_int8(x, M, K, xq, (float*)sx, (cudaStream_t)stream));
}

int wq_linear_a8(const void* x, const void* pw, const void* scales, const void* bias, int64_t M,
                 int64_t N, int64_t K, int f, int G, void* workspace, size_t workspace_bytes,
                 void* out, void* stream) {
  int st = check_linear(x, K, pw, scales, nullptr, bias, M, N, K, f, G, out);
  if (st) return st;
  if ((f != INT8_SYM && f != INT4_SYM) || K % 128) return WQ_ERR_UNSUPPORTED;
  size_t need = 0;
  if ((st = wq_linear_a8_workspace_size(M, K, &need)) != WQ_OK) return st;
  if (M == 0) return WQ_OK;
  if (!workspace || workspace_bytes < need) return WQ_ERR_INVALID_ARG;
  if (!aligned(workspace, 16)) return WQ_ERR_ALIGNMENT;
  size_t wb = 0, sb = 0, ab = 0;
  wq_packed_sizes(f, N, K, G, &wb, &sb, &ab);
  const int64_t w = (int64_t)need;
  if (overlap(workspace, w, x, M * K * 2) || overlap(workspace, w, out, M * N * 2) ||
      overlap(workspace, w, pw, wb) || overlap(workspace, w, scales, sb) ||
      overlap(workspace, w, bias, N * 2))
    return WQ_ERR_INVALID_ARG;
  uint8_t* xq = (uint8_t*)workspace;
  float* sx = (float*)(xq + ((M * K + 255) & ~255LL));
  cudaError_t e = launch_quant_act_int8(x, M, K, xq, sx, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_status(e);
  LinearArgs a;
  a.x = xq;
  a.w = pw;
  a.scales = scales;
  a.aux = sx;
  a.bias = bias;
  a.out = out;
  a.M = M;
  a.N = N;
  a.K = K;
  a.fmt = f;
  a.G = G;
  a.stream = (cudaStream_t)stream;
  return cuda_status(launch_prefill_a8(a));
}

int wq_addmm_requant(int f, int64_t N, int64_t K, int G, void* pw, const void* ps,
                     const void* mat1, const void* mat2, int64_t rank, double alpha, double beta,
                     int use_seed, uint64_t seed, void* stream) {
  int st = check_shape(f, N, K, G);
  if (st) return st;
  if (f != INT8_SYM) return WQ_ERR_UNSUPPORTED;
  if (rank < 0 || rank > (1 << 16)) return WQ_ERR_INVALID_ARG;
  if (!pw || !ps || (rank > 0 && (!mat1 || !mat2))) return WQ_ERR_INVALID_ARG;
  if (!aligned(pw, 16) || !aligned(ps, 16) || (mat1 && !aligned(mat1, 2)) ||
      (mat2 && !aligned(mat2, 2)))
    return WQ_ERR_ALIGNMENT;
  size_t wb = 0, sb = 0, ab = 0;
  wq_packed_sizes(f, N, K, G, &wb, &sb, &ab);
  if (overlap(pw, wb, ps, sb) || overlap(pw, wb, mat1, N * rank * 2) ||
      overlap(pw, wb, mat2, rank * K * 2))
    return WQ_ERR_INVALID_ARG;
  cudaError_t e = launch_addmm_requant_int8(N, K, G, pw, ps, mat1, mat2, rank, alpha, beta,
                                            use_seed, seed, (cudaStream_t)stream);
  if (e == cudaSuccess) e = end_weight_write((cudaStream_t)stream);
  return cuda_status(e);
}

// Lloyd-Max quantizer of N(0,1): thresholds at the midpoints of adjacent
// levels, each level the mean of N(0,1) over its cell, iterated from a
// uniform start on [-3, 3] until no level moves by 1e-14.
int wq_lloyd_max_centroids(int bits, float* out) {
  if (bits < 1 || bits > 8 || !out) return WQ_ERR_INVALID_ARG;
  const int L = 1 << bits;
  double lev[256], edge[257];
  const double inv_sqrt2 = 0.70710678118654752440084436210485;
  const double inv_sqrt2pi = 0.39894228040143267793994605993438;
  auto pdf = [&](double t) { return isinf(t) ? 0.0 : inv_sqrt2pi * exp(-0.5 * t * t); };
  // probability of (a, b] under N(0,1), using the complementary error
  // function on the side away from the mean to keep tail cells accurate
  auto mass = [&](double a, double b) {
    if (a >= 0.0) return 0.5 * (erfc(a * inv_sqrt2) - erfc(b * inv_sqrt2));
    if (b <= 0.0) return 0.5 * (erfc(-b * inv_sqrt2) - erfc(-a * inv_sqrt2));
    return 0.5 * (erf(b * inv_sqrt2) - erf(a * inv_sqrt2));
  };
  for (int i = 0; i < L; ++i) lev[i] = -3.0 + 6.0 * i / (L - 1);
  for (int it = 0; it < 1000000; ++it) {
    edge[0] = -INFINITY;
    edge[L] = INFINITY;
    for (int i = 1; i < L; ++i) edge[i] = 0.5 * (lev[i - 1] + lev[i]);
    double moved = 0.0;
    for (int i = 0; i < L; ++i) {
      double nl = (pdf(edge[i]) - pdf(edge[i + 1])) / mass(edge[i], edge[i + 1]);
      moved = fmax(moved, fabs(nl - lev[i]));
      lev[i] = nl;
    }
    if (moved < 1e-14) break;
  }
  for (int i = 0; i < L; ++i) out[i] = (float)lev[i];
  return WQ_OK;
}

int wq_device_error(unsigned* value, int clear) {
  if (!value) return WQ_ERR_INVALID_ARG;
  unsigned dec = 0;
  if (read_device_error(value, clear != 0) != cudaSuccess) return WQ_ERR_CUDA;
  if (read_decode_error(&dec, clear != 0) != cudaSuccess) return WQ_ERR_CUDA;
  *value |= dec;
  return *value ? WQ_ERR_DEVICE_CHECK : WQ_OK;
}

int wq_device_sm_count(int* n) {
  if (!n) return WQ_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return WQ_ERR_CUDA;
  *n = device_sm_count();
  return WQ_OK;
}

}  // extern "C"

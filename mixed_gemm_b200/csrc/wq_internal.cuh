// Internal declarations shared by the library's translation units.
//
// Packed layout (written by wq_pack, read by every kernel)
// --------------------------------------------------------
// Rows are grouped in tiles of 16 (n = 16*tile + r, r = g + 8*hr, g = 0..7,
// hr = 0/1).  Along K a tile is cut into blocks of 512 bytes: 64 K elements
// for 4-bit codes, 32 for byte codes (INT8, FP8).  Inside a block, lane L = 4*g + tq of a warp
// owns 16 contiguous bytes: the codes of rows g and g+8 for K offsets
// {32c + 8tq + 4s + e : c, s in {0,1} (4-bit) or c = 0 (bytes), e = 0..3}.
// One 16-byte load per lane therefore yields exactly the A-operand fragments
// of an m16n8k16 tensor-core step (W rows as the 16-row operand), with the K
// order inside each 16-step permuted consistently for A and B, so that the
// matching 8 activations of each lane are also contiguous (one 16-byte load).
//
//   4-bit word j = 2c + s holds the 8 nibbles of rows {g, g+8} x K offsets
//   {e = 0..3}.  Two nibble orders:
//     "magic" (INT4_SYM, INT4_ASYM, NVFP4, MXFP4):  p = 4*(e&1) + 2*(e>>1) + hr, so
//        that (word >> 4i) & 0x000F000F yields fragment register i as two
//        nibbles at bit 0 and bit 16;
//     "table" (CB4):                  p = 4*(e>>1) + 2*hr + (e&1), so that the
//        low/high 16 bits hold registers {0,1} / {2,3} as four nibbles each,
//        ready for byte-permute table lookups.
//   INT2_SYM: blocks of 256 bytes (64 K); lane L owns 8 bytes, word c (the
//   32-K chunk c) holds the 16 two-bit fields of rows {g, g+8} x K offsets
//   {32c + 8tq + 4s + e}, field p = 8*(e&1) + 4*s + 2*(e>>1) + hr at bit 2p,
//   so that (word >> 2(4s + i)) & 0x00030003 yields fragment register i of
//   step s as two fields at bit 0 and bit 16; stored offset-binary (v + 2).
//   INT3_SYM: blocks of 384 bytes (64 K) in two planes.  The low plane (the
//   first 256 bytes) holds bits 0..1 of each offset-binary code (v + 4)
//   exactly as INT2 holds its fields; the high plane (the last 128 bytes)
//   gives lane L the word at 256 + 4 L, holding bit 2 of field p of chunk c
//   at bit 16 (p >> 3) + 8 c + (p & 7), so that
//   (hi >> (8 c + 4 s + i)) & 0x00010001 yields the high bits of fragment
//   register i of step s of chunk c at bit 0 and bit 16.
//   INT4_SYM nibbles are stored offset-binary (v + 8); INT8 bytes likewise
//   (v + 128), word j = 2s + hr, byte e; FP8 (E4M3, E5M2) bytes as they
//   are, at the INT8 positions.
//
// Scales (INT formats):  bf16 [N/16][K/G][16], entry 2g + hr (so lane g
//   reads rows g and g+8 as one 32-bit word).
// Scales (FP8):          f32 [N/16][K/G][16], entry 2g + hr (one 64-bit word).
// Zero-points (ASYM):    u8 [N/16][K/G][8], byte g = z(row g) | z(row g+8) << 4.
// NVFP4 block scales:    u8 [N/16][K/16][16], entry 2g + hr.
// MXFP4 block scales:    u8 [N/16][K/32][16], entry 2g + hr.
// CB4 norms, CB4 centroids and the NVFP4 tensor scale keep their canonical
// layout.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/wq.h"

namespace wq {

enum Fmt { INT4_SYM = 0, INT4_ASYM = 1, INT8_SYM = 2, CB4 = 3, NVFP4 = 4, MXFP4 = 5,
           FP8_E4M3 = 6, FP8_E5M2 = 7, INT2_SYM = 8, INT3_SYM = 9 };

__host__ __device__ inline bool is_int_fmt(int f) {
  return f == INT4_SYM || f == INT4_ASYM || f == INT8_SYM || f == INT2_SYM || f == INT3_SYM;
}
// formats with one scale per group of G along K, folded into fp32 sums
__host__ __device__ inline bool is_fp8(int f) { return f == FP8_E4M3 || f == FP8_E5M2; }
__host__ __device__ inline bool is_grouped_fmt(int f) { return is_int_fmt(f) || is_fp8(f); }
// bits per packed code
__host__ __device__ inline int code_bits(int f) {
  return f == INT2_SYM ? 2 : f == INT3_SYM ? 3 : (f == INT8_SYM || is_fp8(f)) ? 8 : 4;
}
__host__ __device__ inline bool is_4bit(int f) { return code_bits(f) == 4; }
// bytes of one packed block (16 rows x block_k(f) K elements)
__host__ __device__ inline int block_bytes(int f) {
  return code_bits(f) == 2 ? 256 : code_bits(f) == 3 ? 384 : 512;
}
// elements of K per 512-byte block
__host__ __device__ inline int block_k(int f) { return code_bits(f) == 8 ? 32 : 64; }

// Byte offset and bit shift of element (n, k) inside the packed weight.
__host__ __device__ inline void packed_loc(int f, int64_t n, int64_t k, int64_t K,
                                           int64_t* byte_off, int* shift) {
  int64_t tile = n >> 4;
  int r = (int)(n & 15), g = r & 7, hr = r >> 3;
  if (code_bits(f) == 2) {
    int64_t b = k >> 6;
    int kk = (int)(k & 63), c = kk >> 5, kc = kk & 31, tq = kc >> 3, e8 = kc & 7, s = e8 >> 2,
        e = e8 & 3;
    int lane = 4 * g + tq;
    int p = 8 * (e & 1) + 4 * s + 2 * (e >> 1) + hr;
    *byte_off = ((tile * (K >> 6) + b) * 32 + lane) * 8 + c * 4 + (p >> 2);
    *shift = (p & 3) * 2;
  } else if (is_4bit(f)) {
    int64_t b = k >> 6;
    int kk = (int)(k & 63), c = kk >> 5, kc = kk & 31, tq = kc >> 3, e8 = kc & 7, s = e8 >> 2,
        e = e8 & 3;
    int lane = 4 * g + tq, j = 2 * c + s;
    int p = (f == CB4) ? (4 * (e >> 1) + 2 * hr + (e & 1))
                       : (4 * (e & 1) + 2 * (e >> 1) + hr);
    *byte_off = ((tile * (K >> 6) + b) * 32 + lane) * 16 + j * 4 + (p >> 1);
    *shift = (p & 1) * 4;
  } else {
    int64_t b = k >> 5;
    int kk = (int)(k & 31), tq = kk >> 3, e8 = kk & 7, s = e8 >> 2, e = e8 & 3;
    int lane = 4 * g + tq, j = 2 * s + hr;
    *byte_off = ((tile * (K >> 5) + b) * 32 + lane) * 16 + j * 4 + e;
    *shift = 0;
  }
}

// INT3: byte and shift of the low-plane field (bits 0..1) and of the
// high-plane bit (bit 2) of element (n, k).
__host__ __device__ inline void packed_loc3(int64_t n, int64_t k, int64_t K, int64_t* lo_off,
                                            int* lo_shift, int64_t* hi_off, int* hi_shift) {
  const int64_t tile = n >> 4;
  const int r = (int)(n & 15), g = r & 7, hr = r >> 3;
  const int64_t b = k >> 6;
  const int kk = (int)(k & 63), c = kk >> 5, kc = kk & 31, tq = kc >> 3, e8 = kc & 7,
            s = e8 >> 2, e = e8 & 3;
  const int lane = 4 * g + tq;
  const int p = 8 * (e & 1) + 4 * s + 2 * (e >> 1) + hr;
  const int64_t base = (tile * (K >> 6) + b) * 384;
  *lo_off = base + lane * 8 + c * 4 + (p >> 2);
  *lo_shift = (p & 3) * 2;
  const int bit = 16 * (p >> 3) + 8 * c + (p & 7);
  *hi_off = base + 256 + lane * 4 + (bit >> 3);
  *hi_shift = bit & 7;
}

// Index (in elements) of the packed group scale / NVFP4 block scale of (n, group).
__host__ __device__ inline int64_t packed_scale_idx(int64_t n, int64_t grp, int64_t groups) {
  int r = (int)(n & 15);
  return ((n >> 4) * groups + grp) * 16 + 2 * (r & 7) + (r >> 3);
}
// Byte and shift of the packed ASYM zero-point of (n, group).
__host__ __device__ inline int64_t packed_zero_byte(int64_t n, int64_t grp, int64_t groups,
                                                    int* shift) {
  int r = (int)(n & 15);
  *shift = (r >> 3) * 4;
  return ((n >> 4) * groups + grp) * 8 + (r & 7);
}

// ------------------------------------------------------------ device math
__device__ __forceinline__ float bf16_bits_to_f32(uint16_t h) {
  return __uint_as_float(((uint32_t)h) << 16);
}

// E4M3 (fn) code -> fp32, exact for all 256 codes (0x7F/0xFF -> NaN).
__device__ __forceinline__ float e4m3_to_f32(uint32_t c) {
  uint32_t s = (c >> 7) & 1u, e = (c >> 3) & 15u, m = c & 7u;
  float v;
  if (e == 15u && m == 7u) v = __uint_as_float(0x7FC00000u);
  else if (e == 0u) v = (float)m * 0.001953125f;  // m * 2^-9
  else v = __uint_as_float(((e + 120u) << 23) | (m << 20));
  return s ? -v : v;
}

// E5M2 code -> fp32, exact for all 256 codes (exponent 31: +-inf, NaN).
__device__ __forceinline__ float e5m2_to_f32(uint32_t c) {
  uint32_t s = (c >> 7) & 1u, e = (c >> 2) & 31u, m = c & 3u;
  float v;
  if (e == 31u) v = m ? __uint_as_float(0x7FC00000u) : __uint_as_float(0x7F800000u);
  else if (e == 0u) v = (float)m * 1.52587890625e-05f;  // m * 2^-16
  else v = __uint_as_float(((e + 112u) << 23) | (m << 21));
  return s ? -v : v;
}

// E8M0 (a power of two, 2^(c - 127)) -> fp32, exact; 255 -> NaN, 0 -> the
// fp32 subnormal 2^-127.
__device__ __forceinline__ float e8m0_to_f32(uint32_t c) {
  if (c == 255u) return __uint_as_float(0x7FC00000u);
  if (c == 0u) return __uint_as_float(0x00400000u);
  return __uint_as_float(c << 23);
}

// ------------------------------------------------------------- launchers
struct LinearArgs {
  const void* x;
  const void* w;
  const void* scales;
  const void* aux;
  const void* bias;
  void* out;
  int64_t M, N, K;
  int fmt, G;
  cudaStream_t stream;
  // x holds rows [up | gate] of 2K values; the activation is up * silu(gate)
  // (decode path only: the prefill path reads a materialized activation)
  bool swiglu = false;
  // grouped launch (prefill kernel only): device row offsets [E + 1], M = T
  // rows of x; w, scales, aux and bias are the first expert's, the others
  // follow at the packed sizes (scale_stride / aux_stride bytes, N for bias)
  const int64_t* offsets = nullptr;
  int E = 1;
  int64_t scale_stride = 0, aux_stride = 0;
};

// cudaErrorNotSupported (nothing launched) when the shape does not fit the
// decode kernel's shared memory (very long K); the prefill kernel takes any M
cudaError_t launch_decode(const LinearArgs& a);
// a[m, k] = bf16(up * silu(gate)) for x2 rows [up | gate], bf16 [M, 2K] -> [M, K]
cudaError_t launch_swiglu(const void* x2, int64_t M, int64_t K, void* a, cudaStream_t st);
// address and size of the library's static device scratch for the SwiGLU
// activation (a file-scope __device__ array; nothing is allocated)
cudaError_t static_swiglu_scratch(void** ptr, size_t* bytes);
constexpr size_t kSwigluStaticScratchBytes = 16u << 20;
cudaError_t launch_prefill(const LinearArgs& a);
// The same tcgen05 kernel on INT8 operands (kind::i8, s32 group sums): a.x is
// the INT8 activation codes [M, K], a.aux the per-token fp32 scales [M];
// INT8_SYM or INT4_SYM weights (the INT4 codes sign-extended to INT8 in the
// operand tile), K % 128 == 0 (else cudaErrorNotSupported, nothing launched)
cudaError_t launch_prefill_a8(const LinearArgs& a);
// One launch over every expert of a grouped linear (a.offsets on the device);
// cudaErrorNotSupported when the schedule's tile bound exceeds the grid limit
cudaError_t launch_prefill_grouped(const LinearArgs& a);
// Per-token INT8 quantization of bf16 x [M, K] (K % 8 == 0): codes xq [M, K],
// scales sx [M]
cudaError_t launch_quant_act_int8(const void* x, int64_t M, int64_t K, void* xq, float* sx,
                                  cudaStream_t st);
int device_sm_count();
// A 4-byte memset of a library word on `st`: a stream operation that is not a
// kernel, appended to every call that writes packed weights (wq_pack,
// wq_quantize, wq_addmm_requant).  The decode kernel is launched with
// programmatic dependent launch and reads the packed weights before it waits
// for the previous kernel; with this operation in between, the previous
// kernel of a following wq_linear is never the one that wrote its weights.
cudaError_t end_weight_write(cudaStream_t st);
// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per (device, kernel),
// thread-safe; a failure is returned and retried on the next call.
cudaError_t ensure_max_dynamic_smem(const void* fn, int bytes);
// The decode kernel's own error word (bit 128: its activation-slice wait ran
// out); synchronous read, optional clear.
cudaError_t read_decode_error(unsigned* value, bool clear);
// The kernels' own error word (bit per failed bounded wait); synchronous read.
cudaError_t read_device_error(unsigned* value, bool clear);

cudaError_t launch_pack(int f, int64_t N, int64_t K, int G, const void* codes, const void* scales,
                        const void* aux, void* pw, void* ps, void* pa, cudaStream_t st);
cudaError_t launch_unpack(int f, int64_t N, int64_t K, int G, const void* pw, const void* ps,
                          const void* pa, void* codes, void* scales, void* aux, cudaStream_t st);
cudaError_t launch_dequant(int f, int64_t N, int64_t K, int G, const void* pw, const void* ps,
                           const void* pa, float* out, cudaStream_t st);
cudaError_t launch_quantize(int f, int64_t N, int64_t K, int G, const float* w, void* codes,
                            void* scales, void* aux, cudaStream_t st);

}  // namespace wq

// Register-level conversion of packed codes to bf16 tensor-core fragments,
// shared by the decode kernel (fragments go straight into mma.sync) and the
// prefill kernel (fragments are scaled and stored to shared memory for
// tcgen05).  Fragment i of an m16n8k16 A operand holds two consecutive K
// elements of one row: i = 0 row g / K 0,1;  1 row g+8 / K 0,1;
// 2 row g / K 2,3;  3 row g+8 / K 2,3  (see the packed layout in
// wq_internal.cuh).
#pragma once

#include <stdint.h>

namespace wq {

static __device__ __forceinline__ uint32_t word(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

static __device__ __forceinline__ uint32_t bsub2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
static __device__ __forceinline__ uint32_t bmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
static __device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}
static __device__ __forceinline__ uint32_t f32_to_bf16_bits(float v) {
  return pack_bf16x2(v, 0.f) & 0xFFFFu;
}

// INT4, "magic" nibble order: fragment i = nibbles (i, i+4) as bf16 (128 + n),
// minus the per-row offset (136 for offset-binary signed codes, 128 + z).
static __device__ __forceinline__ void frag_int4(uint32_t wd, uint32_t off_g, uint32_t off_g8,
                                          uint32_t (&a)[4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t t = ((wd >> (4 * i)) & 0x000F000Fu) | 0x43004300u;
    a[i] = bsub2(t, (i & 1) ? off_g8 : off_g);
  }
}

// INT2, fields (4s + i, 8 + 4s + i) of the word: fragment i of tensor-core
// step s as bf16 (128 + c), minus the offset (130 for offset-binary codes).
static __device__ __forceinline__ void frag_int2(uint32_t wd, int s, uint32_t off,
                                                 uint32_t (&a)[4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t t = ((wd >> (2 * (4 * s + i))) & 0x00030003u) | 0x43004300u;
    a[i] = bsub2(t, off);
  }
}

// INT3, two planes: low bits as the INT2 fields of word `lo` (chunk c), the
// high bit from the lane's high-plane word `hi` at 8 c + 4 s + i (and 16
// above); fragment i of step s as bf16 (128 + c), minus the offset (132 for
// offset-binary codes).
static __device__ __forceinline__ void frag_int3(uint32_t lo, uint32_t hi, int c, int s,
                                                 uint32_t off, uint32_t (&a)[4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    // (the high bits move right first: the upper one may sit at bit 31)
    const uint32_t t = ((lo >> (2 * (4 * s + i))) & 0x00030003u) |
                       (((hi >> (8 * c + 4 * s + i)) << 2) & 0x00040004u) | 0x43004300u;
    a[i] = bsub2(t, off);
  }
}

// INT8 offset-binary bytes u = q + 128 -> exact bf16 pairs of q, all in
// bf16x2 integer arithmetic (no float conversion).  The byte pair (selected
// by `sel` into the low bytes of the two halves) gives x = u per half; under
// the exponent of 128 its low 7 bits read 128 + (u & 127), and adding -256
// (u < 128) or -128 (u >= 128) leaves u - 128 = q, an integer in
// [-128, 127] that bf16 holds exactly, so the addition rounds nothing.
static __device__ __forceinline__ uint32_t badd2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
static __device__ __forceinline__ uint32_t i8pair(uint32_t w, uint32_t sel) {
  const uint32_t x = __byte_perm(w, 0u, sel);
  return badd2((x & 0x007F007Fu) | 0x43004300u, (x & 0x00800080u) ^ 0xC380C380u);
}
static __device__ __forceinline__ void frag_int8(uint32_t wg, uint32_t wg8, uint32_t (&a)[4]) {
  a[0] = i8pair(wg, 0x4140u);   // bytes 0, 1
  a[1] = i8pair(wg8, 0x4140u);
  a[2] = i8pair(wg, 0x4342u);   // bytes 2, 3
  a[3] = i8pair(wg8, 0x4342u);
}

// FP8 E4M3 bytes -> exact bf16 fragments.  A byte placed at bits 8..15 of a
// 16-bit half (sign at bit 15) and its 7 magnitude bits moved to bits 4..10
// reads as the bf16 number e4m3 * 2^-120 (for the E4M3 subnormals too, whose
// spacing 2^-9 becomes the bf16 subnormal spacing); the exact product with
// 2^120 restores the value.  Fragment registers as in frag_int8.  The NaN
// codes 0x7F / 0xFF come out as +-480.
static __device__ __forceinline__ uint32_t e4m3x2_scaled_bits(uint32_t t8) {
  return ((t8 >> 4) & 0x07F007F0u) | (t8 & 0x80008000u);
}
static __device__ __forceinline__ void frag_e4m3(uint32_t wg, uint32_t wg8, uint32_t (&a)[4]) {
  const uint32_t k120 = 0x7B807B80u;  // bf16x2 (2^120, 2^120)
  a[0] = bmul2(e4m3x2_scaled_bits(__byte_perm(wg, 0u, 0x1404u)), k120);
  a[1] = bmul2(e4m3x2_scaled_bits(__byte_perm(wg8, 0u, 0x1404u)), k120);
  a[2] = bmul2(e4m3x2_scaled_bits(__byte_perm(wg, 0u, 0x3424u)), k120);
  a[3] = bmul2(e4m3x2_scaled_bits(__byte_perm(wg8, 0u, 0x3424u)), k120);
}

// FP8 E5M2 bytes -> exact bf16 fragments, as frag_e4m3: the 7 magnitude bits
// at bits 5..11 read as e5m2 * 2^-112 (subnormals included), restored by an
// exact multiply by 2^112.  The infinity / NaN codes (exponent 31) come out
// as finite values of magnitude 2^16 (1 + m/4).
static __device__ __forceinline__ uint32_t e5m2x2_scaled_bits(uint32_t t8) {
  return ((t8 >> 3) & 0x0FE00FE0u) | (t8 & 0x80008000u);
}
static __device__ __forceinline__ void frag_e5m2(uint32_t wg, uint32_t wg8, uint32_t (&a)[4]) {
  const uint32_t k112 = 0x77807780u;  // bf16x2 (2^112, 2^112)
  a[0] = bmul2(e5m2x2_scaled_bits(__byte_perm(wg, 0u, 0x1404u)), k112);
  a[1] = bmul2(e5m2x2_scaled_bits(__byte_perm(wg8, 0u, 0x1404u)), k112);
  a[2] = bmul2(e5m2x2_scaled_bits(__byte_perm(wg, 0u, 0x3424u)), k112);
  a[3] = bmul2(e5m2x2_scaled_bits(__byte_perm(wg8, 0u, 0x3424u)), k112);
}

// 16-entry bf16 lookup ("table" nibble order): byte tables H (high bytes) and
// L (low bytes), four entries per register.  `kSymLow` means the low-byte
// table does not depend on the top index bit (true for E2M1).
template <bool kSymLow>
static __device__ __forceinline__ void frag_table(uint32_t wd, const uint32_t (&H)[4],
                                           const uint32_t (&L)[4], uint32_t (&a)[4]) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t x = h ? (wd >> 16) : wd;
    uint32_t sel = x & 0x7777u;
    uint32_t mask = __byte_perm(0u, 0xFFFFFFFFu, (x >> 1) & 0x4444u);
    uint32_t hb = (__byte_perm(H[0], H[1], sel) & ~mask) | (__byte_perm(H[2], H[3], sel) & mask);
    uint32_t lb;
    if (kSymLow) lb = __byte_perm(L[0], L[1], sel);
    else lb = (__byte_perm(L[0], L[1], sel) & ~mask) | (__byte_perm(L[2], L[3], sel) & mask);
    a[2 * h] = __byte_perm(lb, hb, 0x5140u);
    a[2 * h + 1] = __byte_perm(lb, hb, 0x7362u);
  }
}


// NVFP4, "magic" nibble order: fragment i = E2M1 nibbles (i, i+4) times the
// block scale.  With t = the two nibbles at bits 0..3 and 16..19, the product
// t * 0x1040 is (t << 6) | (t << 12) (the fields do not overlap), and the mask
// 0x81C081C0 keeps the magnitude bits at 6..8 and the sign bit at 15 of each
// half: the bf16 bit pattern of +-e2m1 * 2^-126 (a subnormal for 0.5, zero for
// 0).  Multiplying by bf16(e4m3 * 2^119) gives e2m1 * e4m3 * 2^-7 exactly (at
// most 6 significant bits, between 2^-17 and 21); the caller multiplies the
// result by 2^7 in fp32.  Integer multiply and bf16 multiply issue on the FMA
// pipe, leaving the ALU pipe two logic operations per register.
static __device__ __forceinline__ void frag_nvfp4(uint32_t wd, uint32_t sc_g, uint32_t sc_g8,
                                                  uint32_t (&a)[4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t t = (wd >> (4 * i)) & 0x000F000Fu;
    a[i] = bmul2((t * 0x1040u) & 0x81C081C0u, (i & 1) ? sc_g8 : sc_g);
  }
}

// E4M3 (low byte of `b`) -> fp32, exact and branch-free: the 7 magnitude bits
// placed at fp32 bit 20 read as 2^(e-127)(1 + m/8) (or, for e = 0, the fp32
// subnormal m * 2^-129), and the power-of-two factor 2^120 moves both to the
// E4M3 values 2^(e-7)(1 + m/8) and m * 2^-9; the sign bit is copied and the
// NaN codes (magnitude 0x7F) give NaN.
static __device__ __forceinline__ float e4m3_bits_to_f32(uint32_t b) {
  const uint32_t m7 = b & 0x7Fu;
  const float mag = m7 == 0x7Fu ? __uint_as_float(0x7FC00000u)
                                : __uint_as_float(m7 << 20) * 0x1p120f;
  return __uint_as_float(__float_as_uint(mag) | ((b & 0x80u) << 24));
}

// bf16x2 (v, v) with v = e4m3(b) * 2^119 (exact), the factor frag_nvfp4 expects
static __device__ __forceinline__ uint32_t nvfp4_scale_pair(uint32_t b) {
  const float v = e4m3_bits_to_f32(b) * 0x1p119f;
  return pack_bf16x2(v, v);
}

// MXFP4: E8M0 code e -> bf16x2 (s, s), s = 2^(min(e, 128) - 1) (NaN for the
// NaN code 255).  With frag_nvfp4 (e2m1 * 2^-126 bit patterns) this gives
// e2m1 * 2^(min(e, 128) - 127) exactly; blocks with e > 128 take one more
// exact multiply by mx_hi_pair(e) = 2^(e - 128), so that no factor leaves the
// bf16 range.
static __device__ __forceinline__ uint32_t mx_lo_pair(uint32_t e) {
  if (e == 255u) return 0x7FC07FC0u;
  const uint32_t m = (e < 128u ? e : 128u) + 126u;  // exponent field of 2^(min(e,128) - 1)
  return (m << 7) * 0x00010001u;
}
static __device__ __forceinline__ uint32_t mx_hi_pair(uint32_t e) {
  return ((e - 128u + 127u) << 7) * 0x00010001u;  // 2^(e - 128), e in 129..254
}

// SwiGLU input: bf16 pairs up * silu(gate), silu(g) = g / (1 + e^-g), in
// fp32 (fast exponential; the result is rounded to bf16, nearest even)
static __device__ __forceinline__ uint32_t swiglu_pair(uint32_t u, uint32_t g) {
  const float u0 = __uint_as_float(u << 16), u1 = __uint_as_float(u & 0xFFFF0000u);
  const float g0 = __uint_as_float(g << 16), g1 = __uint_as_float(g & 0xFFFF0000u);
  const float a0 = u0 * (g0 / (1.f + __expf(-g0)));
  const float a1 = u1 * (g1 / (1.f + __expf(-g1)));
  return pack_bf16x2(a0, a1);
}

}  // namespace wq

// Offline reorder (pack / unpack) and the exact-dequant test export.
//
// Pack and unpack are pure permutations plus the offset-binary recoding of
// INT4_SYM / INT8_SYM codes, so unpack(pack(c)) == c bit for bit.  The
// packed layout is described in wq_internal.cuh.  Source: Petit README,
// "Techniques and performance" (weights shuffled offline to make GPU
// dequantization efficient); auto-round-lib README section 1
// (repack_quantized_weight / unpack_weight).
#include "wq_internal.cuh"

namespace wq {

namespace {

constexpr int kThreads = 256;

inline unsigned grid_for(int64_t n) {
  int64_t b = (n + kThreads - 1) / kThreads;
  if (b > (1LL << 30)) b = 1LL << 30;
  return (unsigned)(b < 1 ? 1 : b);
}

// canonical nibble/byte of element (n, k)
__device__ __forceinline__ uint32_t canon_code(int f, const uint8_t* codes, int64_t n, int64_t k,
                                               int64_t K) {
  if (code_bits(f) == 2) return (codes[n * (K >> 2) + (k >> 2)] >> (2 * (k & 3))) & 3u;
  if (code_bits(f) == 3) {  // bits 3k..3k+2 of the row's little-endian bit stream
    const uint8_t* row = codes + n * (3 * K / 8);
    const int64_t bit = 3 * k;
    uint32_t v = row[bit >> 3];
    if ((bit & 7) > 5) v |= (uint32_t)row[(bit >> 3) + 1] << 8;
    return (v >> (bit & 7)) & 7u;
  }
  if (is_4bit(f)) {
    uint8_t b = codes[n * (K >> 1) + (k >> 1)];
    return (k & 1) ? (b >> 4) : (b & 15u);
  }
  return codes[n * K + k];
}

// canonical -> packed encoding of one code
__device__ __forceinline__ uint32_t encode(int f, uint32_t c) {
  if (f == INT4_SYM) return c ^ 0x8u;
  if (f == INT2_SYM) return c ^ 0x2u;
  if (f == INT3_SYM) return c ^ 0x4u;
  if (f == INT8_SYM) return c ^ 0x80u;
  return c;
}

// One thread per packed weight byte: gather the canonical code(s) it holds.
__global__ void pack_w_kernel(int f, int64_t N, int64_t K, const uint8_t* __restrict__ codes,
                              uint8_t* __restrict__ pw) {
  const int64_t total = N * K * code_bits(f) / 8;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    if (code_bits(f) == 3) {  // 384-byte blocks of 64 K: low plane, then high plane
      const int64_t blk_global = i / 384, nblk = K >> 6;
      const int rem = (int)(i % 384);
      const int64_t tile = blk_global / nblk, b = blk_global % nblk;
      uint32_t out = 0;
      for (int h = 0; h < 8; ++h) {
        int lane, c, p, sh;
        if (rem < 256) {            // fields 4q .. 4q + 3 of word c, two bits each
          if (h >= 4) break;
          lane = rem >> 3;
          c = (rem >> 2) & 1;
          p = 4 * (rem & 3) + h;
          sh = 2 * h;
        } else {                    // bit 16 (p >> 3) + 8 c + (p & 7) of the lane's word
          const int rr = rem - 256, bit = 8 * (rr & 3) + h;
          lane = rr >> 2;
          c = (bit & 15) >> 3;
          p = 8 * (bit >> 4) + (bit & 7);
          sh = h;
        }
        const int g = lane >> 2, tq = lane & 3;
        const int hr = p & 1, e = ((p >> 1) & 1) * 2 + (p >> 3), s = (p >> 2) & 1;
        const int64_t n = tile * 16 + g + 8 * hr;
        const int64_t k = b * 64 + c * 32 + tq * 8 + s * 4 + e;
        const uint32_t v = encode(f, canon_code(f, codes, n, k, K));
        out |= (rem < 256 ? (v & 3u) : (v >> 2)) << sh;
      }
      pw[i] = (uint8_t)out;
      continue;
    }
    if (code_bits(f) == 2) {  // 8-byte lane chunks, 256-byte blocks of 64 K
      const int q = (int)(i & 3), c = (int)((i >> 2) & 1), lane = (int)((i >> 3) & 31);
      const int64_t blk_global = i >> 8, nblk = K >> 6;
      const int64_t tile = blk_global / nblk, b = blk_global % nblk;
      const int g = lane >> 2, tq = lane & 3;
      uint32_t out = 0;
      for (int h = 0; h < 4; ++h) {
        const int p = 4 * q + h;
        const int hr = p & 1, e = ((p >> 1) & 1) * 2 + (p >> 3), s = (p >> 2) & 1;
        const int64_t n = tile * 16 + g + 8 * hr;
        const int64_t k = b * 64 + c * 32 + tq * 8 + s * 4 + e;
        out |= encode(f, canon_code(f, codes, n, k, K)) << (2 * h);
      }
      pw[i] = (uint8_t)out;
      continue;
    }
    // decompose the packed byte offset
    int64_t word = i >> 2;
    int q = (int)(i & 3);
    int j = (int)(word & 3);
    int64_t chunk = word >> 2;  // 16-byte lane chunk
    int lane = (int)(chunk & 31);
    int64_t blk_global = chunk >> 5;
    int64_t nblk = K / block_k(f);
    int64_t tile = blk_global / nblk, b = blk_global % nblk;
    int g = lane >> 2, tq = lane & 3;
    uint32_t out = 0;
    if (is_4bit(f)) {
      int c = j >> 1, s = j & 1;
      for (int h = 0; h < 2; ++h) {
        int p = 2 * q + h;
        int hr, e;
        if (f == CB4) { hr = (p >> 1) & 1; e = (p >> 2) * 2 + (p & 1); }
        else { hr = p & 1; e = ((p >> 1) & 1) * 2 + (p >> 2); }
        int64_t n = tile * 16 + g + 8 * hr;
        int64_t k = b * 64 + c * 32 + tq * 8 + s * 4 + e;
        out |= encode(f, canon_code(f, codes, n, k, K)) << (4 * h);
      }
    } else {
      int s = j >> 1, hr = j & 1, e = q;
      int64_t n = tile * 16 + g + 8 * hr;
      int64_t k = b * 32 + tq * 8 + s * 4 + e;
      out = encode(f, canon_code(f, codes, n, k, K));
    }
    pw[i] = (uint8_t)out;
  }
}

// INT3: one thread per 8 elements (three canonical bytes).
__global__ void unpack_w3_kernel(int64_t N, int64_t K, const uint8_t* __restrict__ pw,
                                 uint8_t* __restrict__ codes) {
  const int64_t total = N * K / 8;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = i / (K >> 3), k0 = (i % (K >> 3)) * 8;
    uint32_t bits = 0;
    for (int h = 0; h < 8; ++h) {
      int64_t lo, hi;
      int ls, hs;
      packed_loc3(n, k0 + h, K, &lo, &ls, &hi, &hs);
      const uint32_t v = ((pw[lo] >> ls) & 3u) | (((pw[hi] >> hs) & 1u) << 2);
      bits |= encode(INT3_SYM, v) << (3 * h);
    }
    uint8_t* dst = codes + n * (3 * K / 8) + 3 * (k0 >> 3);
    dst[0] = (uint8_t)bits;
    dst[1] = (uint8_t)(bits >> 8);
    dst[2] = (uint8_t)(bits >> 16);
  }
}

// One thread per canonical byte: scatter back from the packed weight.
__global__ void unpack_w_kernel(int f, int64_t N, int64_t K, const uint8_t* __restrict__ pw,
                                uint8_t* __restrict__ codes) {
  const int64_t total = N * K * code_bits(f) / 8;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    uint32_t out = 0;
    if (code_bits(f) == 2) {
      int64_t n = i / (K >> 2), k0 = (i % (K >> 2)) * 4;
      for (int h = 0; h < 4; ++h) {
        int64_t off;
        int sh;
        packed_loc(f, n, k0 + h, K, &off, &sh);
        out |= encode(f, (pw[off] >> sh) & 3u) << (2 * h);
      }
    } else if (is_4bit(f)) {
      int64_t n = i / (K >> 1), k0 = (i % (K >> 1)) * 2;
      for (int h = 0; h < 2; ++h) {
        int64_t off;
        int sh;
        packed_loc(f, n, k0 + h, K, &off, &sh);
        uint32_t v = (pw[off] >> sh) & 15u;
        out |= encode(f, v) << (4 * h);  // the recoding is its own inverse
      }
    } else {
      int64_t n = i / K, k = i % K;
      int64_t off;
      int sh;
      packed_loc(f, n, k, K, &off, &sh);
      out = encode(f, pw[off]);
    }
    codes[i] = (uint8_t)out;
  }
}

// Group scales / NVFP4 block scales: canonical [N][groups] <-> packed.
template <typename T>
__global__ void permute_scales_kernel(int64_t N, int64_t groups, const T* __restrict__ src,
                                      T* __restrict__ dst, bool to_packed) {
  const int64_t total = N * groups;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    int64_t n = i / groups, grp = i % groups;
    int64_t p = packed_scale_idx(n, grp, groups);
    if (to_packed) dst[p] = src[i];
    else dst[i] = src[p];
  }
}

// ASYM zero-points: canonical u8 [N][groups] <-> packed nibbles.
__global__ void pack_zeros_kernel(int64_t N, int64_t groups, const uint8_t* __restrict__ z,
                                  uint8_t* __restrict__ pz) {
  const int64_t total = N * groups / 2;  // packed bytes
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    int64_t tile_grp = i >> 3;
    int g = (int)(i & 7);
    int64_t tile = tile_grp / groups, grp = tile_grp % groups;
    int64_t n0 = tile * 16 + g, n1 = n0 + 8;
    pz[i] = (uint8_t)((z[n0 * groups + grp] & 15u) | ((z[n1 * groups + grp] & 15u) << 4));
  }
}

__global__ void unpack_zeros_kernel(int64_t N, int64_t groups, const uint8_t* __restrict__ pz,
                                    uint8_t* __restrict__ z) {
  const int64_t total = N * groups;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    int64_t n = i / groups, grp = i % groups;
    int sh;
    int64_t b = packed_zero_byte(n, grp, groups, &sh);
    z[i] = (uint8_t)((pz[b] >> sh) & 15u);
  }
}

__global__ void copy_bytes_kernel(const uint8_t* __restrict__ s, uint8_t* __restrict__ d,
                                  int64_t n) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    d[i] = s[i];
}

// Exact dequantized value of (n, k) read from the packed buffers.
__global__ void dequant_kernel(int f, int64_t N, int64_t K, int G, const uint8_t* __restrict__ pw,
                               const void* __restrict__ ps, const void* __restrict__ pa,
                               float* __restrict__ out) {
  const int64_t total = N * K;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    int64_t n = i / K, k = i % K;
    int64_t off;
    int sh;
    uint32_t raw;
    if (f == INT3_SYM) {
      int64_t hi;
      int hs;
      packed_loc3(n, k, K, &off, &sh, &hi, &hs);
      raw = ((pw[off] >> sh) & 3u) | (((pw[hi] >> hs) & 1u) << 2);
    } else {
      packed_loc(f, n, k, K, &off, &sh);
      raw = (pw[off] >> sh) & ((1u << code_bits(f)) - 1u);
    }
    float v;
    if (f == INT4_SYM || f == INT8_SYM || f == INT2_SYM || f == INT3_SYM) {
      int q = (int)raw - (f == INT4_SYM ? 8 : f == INT2_SYM ? 2 : f == INT3_SYM ? 4 : 128);
      float s = bf16_bits_to_f32(((const uint16_t*)ps)[packed_scale_idx(n, k / G, K / G)]);
      v = (float)q * s;
    } else if (f == INT4_ASYM) {
      int zs;
      int64_t zb = packed_zero_byte(n, k / G, K / G, &zs);
      int z = (((const uint8_t*)pa)[zb] >> zs) & 15;
      float s = bf16_bits_to_f32(((const uint16_t*)ps)[packed_scale_idx(n, k / G, K / G)]);
      v = (float)((int)raw - z) * s;
    } else if (is_fp8(f)) {  // one rounding of the exact fp8 * s
      float s = ((const float*)ps)[packed_scale_idx(n, k / G, K / G)];
      v = __fmul_rn(f == FP8_E4M3 ? e4m3_to_f32(raw) : e5m2_to_f32(raw), s);
    } else if (f == CB4) {
      float c = ((const float*)pa)[raw];
      float nr = bf16_bits_to_f32(((const uint16_t*)ps)[n]);
      v = __fmul_rn(c, nr);
    } else if (f == NVFP4) {  // e2m1 * e4m3 is exact in fp32; one rounding when * ts
      const float mag[8] = {0.f, 0.5f, 1.f, 1.5f, 2.f, 3.f, 4.f, 6.f};
      float e = (raw & 8u) ? -mag[raw & 7u] : mag[raw & 7u];
      float sb = e4m3_to_f32(((const uint8_t*)ps)[packed_scale_idx(n, k >> 4, K >> 4)]);
      float ts = ((const float*)pa)[0];
      v = __fmul_rn(__fmul_rn(e, sb), ts);
    } else {  // MXFP4: e2m1 * 2^(e - 127), exact (or the fp32 overflow)
      const float mag[8] = {0.f, 0.5f, 1.f, 1.5f, 2.f, 3.f, 4.f, 6.f};
      float e = (raw & 8u) ? -mag[raw & 7u] : mag[raw & 7u];
      v = __fmul_rn(e, e8m0_to_f32(((const uint8_t*)ps)[packed_scale_idx(n, k >> 5, K >> 5)]));
    }
    out[i] = v;
  }
}

}  // namespace

cudaError_t launch_pack(int f, int64_t N, int64_t K, int G, const void* codes, const void* scales,
                        const void* aux, void* pw, void* ps, void* pa, cudaStream_t st) {
  const int64_t wbytes = N * K * code_bits(f) / 8;
  pack_w_kernel<<<grid_for(wbytes), kThreads, 0, st>>>(f, N, K, (const uint8_t*)codes,
                                                        (uint8_t*)pw);
  if (is_fp8(f)) {
    int64_t groups = K / G;
    permute_scales_kernel<uint32_t><<<grid_for(N * groups), kThreads, 0, st>>>(
        N, groups, (const uint32_t*)scales, (uint32_t*)ps, true);
  } else if (is_int_fmt(f)) {
    int64_t groups = K / G;
    permute_scales_kernel<uint16_t><<<grid_for(N * groups), kThreads, 0, st>>>(
        N, groups, (const uint16_t*)scales, (uint16_t*)ps, true);
    if (f == INT4_ASYM)
      pack_zeros_kernel<<<grid_for(N * groups / 2), kThreads, 0, st>>>(
          N, groups, (const uint8_t*)aux, (uint8_t*)pa);
  } else if (f == NVFP4 || f == MXFP4) {
    const int64_t blk = f == NVFP4 ? 16 : 32;  // K per block scale
    permute_scales_kernel<uint8_t><<<grid_for(N * (K / blk)), kThreads, 0, st>>>(
        N, K / blk, (const uint8_t*)scales, (uint8_t*)ps, true);
    if (f == NVFP4) copy_bytes_kernel<<<1, 32, 0, st>>>((const uint8_t*)aux, (uint8_t*)pa, 4);
  } else {  // CB4: norms and centroids keep their layout
    copy_bytes_kernel<<<grid_for(N * 2), kThreads, 0, st>>>((const uint8_t*)scales,
                                                            (uint8_t*)ps, N * 2);
    copy_bytes_kernel<<<1, 64, 0, st>>>((const uint8_t*)aux, (uint8_t*)pa, 64);
  }
  return cudaGetLastError();
}

cudaError_t launch_unpack(int f, int64_t N, int64_t K, int G, const void* pw, const void* ps,
                          const void* pa, void* codes, void* scales, void* aux, cudaStream_t st) {
  const int64_t wbytes = N * K * code_bits(f) / 8;
  if (f == INT3_SYM)
    unpack_w3_kernel<<<grid_for(N * K / 8), kThreads, 0, st>>>(N, K, (const uint8_t*)pw,
                                                               (uint8_t*)codes);
  else
    unpack_w_kernel<<<grid_for(wbytes), kThreads, 0, st>>>(f, N, K, (const uint8_t*)pw,
                                                            (uint8_t*)codes);
  if (is_fp8(f)) {
    int64_t groups = K / G;
    permute_scales_kernel<uint32_t><<<grid_for(N * groups), kThreads, 0, st>>>(
        N, groups, (const uint32_t*)ps, (uint32_t*)scales, false);
  } else if (is_int_fmt(f)) {
    int64_t groups = K / G;
    permute_scales_kernel<uint16_t><<<grid_for(N * groups), kThreads, 0, st>>>(
        N, groups, (const uint16_t*)ps, (uint16_t*)scales, false);
    if (f == INT4_ASYM)
      unpack_zeros_kernel<<<grid_for(N * groups), kThreads, 0, st>>>(
          N, groups, (const uint8_t*)pa, (uint8_t*)aux);
  } else if (f == NVFP4 || f == MXFP4) {
    const int64_t blk = f == NVFP4 ? 16 : 32;
    permute_scales_kernel<uint8_t><<<grid_for(N * (K / blk)), kThreads, 0, st>>>(
        N, K / blk, (const uint8_t*)ps, (uint8_t*)scales, false);
    if (f == NVFP4) copy_bytes_kernel<<<1, 32, 0, st>>>((const uint8_t*)pa, (uint8_t*)aux, 4);
  } else {
    copy_bytes_kernel<<<grid_for(N * 2), kThreads, 0, st>>>((const uint8_t*)ps,
                                                            (uint8_t*)scales, N * 2);
    copy_bytes_kernel<<<1, 64, 0, st>>>((const uint8_t*)pa, (uint8_t*)aux, 64);
  }
  return cudaGetLastError();
}

cudaError_t launch_dequant(int f, int64_t N, int64_t K, int G, const void* pw, const void* ps,
                           const void* pa, float* out, cudaStream_t st) {
  dequant_kernel<<<grid_for(N * K), kThreads, 0, st>>>(f, N, K, G, (const uint8_t*)pw, ps, pa,
                                                        out);
  return cudaGetLastError();
}

}  // namespace wq

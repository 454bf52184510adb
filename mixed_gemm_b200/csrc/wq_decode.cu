// Decode path (M <= 16): stream the packed weight once from HBM.
//
// Work split.  A CTA owns RT row tiles (16 output features each) and a slice
// of K; a cluster of CS CTAs covers all of K for those rows; the KW warps of a
// CTA split the CTA's K slice again.  Every lane issues one 16-byte
// no-L1-allocate load per row tile and 512-byte block, which holds exactly its
// tensor-core A fragments for that block (layout in wq_internal.cuh), and one
// 16-byte load of the 8 matching activations per token row.  Codes become
// bf16 in registers (magic-number nibble conversion for INT4, fp32 magic for
// INT8, byte-permute table lookups for CB4 and NVFP4) and feed
// mma.sync.m16n8k16 with the W rows as the 16-row operand and the (<= 16)
// tokens as the 8-column operand.  INT group scales are applied per 32-K
// chunk to the fp32 chunk accumulator (so the bf16 fragments are the exact
// integer codes); NVFP4 block scales are multiplied into the fragments (the
// product e2m1*e4m3 is exact in bf16); the CB4 row norm and the NVFP4 tensor
// scale are applied in the epilogue.  Partial sums are reduced across warps
// through shared memory and across the cluster through distributed shared
// memory (no global workspace), then rank 0 applies fold + bias, rounds to
// bf16 and stores.
//
// Sources: OrbitQuant card "Benchmark" (skinny batches are decode-bound; the
// Metal path dispatches a skinny GEMV for up to four rows with decoded weight
// segments reused across the batch); Petit README "Techniques and
// performance" (batches below 16 are the small-batch regime, weights shuffled
// offline for cheap dequantization).
#include <cooperative_groups.h>

#include "wq_frag.cuh"
#include "wq_internal.cuh"

namespace cg = cooperative_groups;

namespace wq {

namespace {

struct DecodeParams {
  const uint16_t* x;
  const uint4* w;
  const void* scales;
  const void* aux;
  const uint16_t* bias;
  uint16_t* out;
  int M, N, K, G, cs;
  int xs_stride;  // bytes per token row of the staged X slice
  int xs_bytes;   // bytes of the staged X slice (M rows)
  int side_rows;  // per row tile: scale groups (INT) or 16-K blocks (NVFP4) staged
  int side_bytes; // bytes of staged scales / zero-points / block scales
};

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 ld_nc(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async8(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t lds16(uint32_t addr) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t lds8(uint32_t addr) {
  unsigned short v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

template <int FMT, int NT, int RT, int KW, int UB>
__global__ void __launch_bounds__(KW * 32) decode_kernel(const DecodeParams p) {
  constexpr int KB = FMT == INT8_SYM ? 32 : 64;   // K per 512-byte block
  constexpr int CPB = FMT == INT8_SYM ? 1 : 2;    // 32-K chunks per block
  constexpr int NV = RT * NT * 4;                  // accumulators per lane
  constexpr bool kIntFmt = FMT == INT4_SYM || FMT == INT4_ASYM || FMT == INT8_SYM;

  extern __shared__ __align__(16) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, tq = lane & 3;
  const int cs = p.cs;
  const int rank = (int)(blockIdx.x % cs);
  const int64_t tile0 = (int64_t)(blockIdx.x / cs) * RT;
  const int64_t K = p.K;
  const int64_t nblk = K / KB;
  const int64_t groups = kIntFmt ? K / p.G : 0;

  // this CTA's K blocks [cb, ce), this warp's [wb, we)
  const int64_t cb = rank * nblk / cs, ce = (rank + 1) * nblk / cs;
  const int64_t wb = cb + warp * (ce - cb) / KW, we = cb + (warp + 1) * (ce - cb) / KW;

  // Stage in shared memory, with cp.async, everything the K loop reads besides
  // the weight stream: the CTA's slice of X (tokens < M, K in
  // [cb*KB, ce*KB)), and the group scales + zero-points (INT) or E4M3 block
  // scales (NVFP4) of its row tiles over that K range.
  const uint32_t xs = (uint32_t)__cvta_generic_to_shared(smem);
  const uint32_t side = xs + (uint32_t)p.xs_bytes;
  float* red = (float*)(smem + p.xs_bytes + p.side_bytes);
  const int64_t kbeg = cb * KB;
  const int64_t g_begin = kIntFmt ? kbeg / p.G : 0;   // first scale group staged
  const int64_t b16_begin = kbeg >> 4;                // first NVFP4 16-block staged
  {
    const int cpr = (int)((ce - cb) * KB / 8);  // 16-byte chunks per token row
    for (int i = threadIdx.x; i < p.M * cpr; i += KW * 32) {
      const int tok = i / cpr, c = i - tok * cpr;
      cp_async16(xs + tok * p.xs_stride + c * 16, p.x + tok * K + kbeg + c * 8);
    }
    if constexpr (kIntFmt) {
      const int64_t g_end = (ce * KB - 1) / p.G + 1;
      const int ng = (int)(g_end - g_begin);
      // scales: 32 bytes per (tile, group) -> two 16-byte chunks
      for (int i = threadIdx.x; i < RT * ng * 2; i += KW * 32) {
        const int r = i / (ng * 2), rem = i - r * ng * 2, gi = rem >> 1, h = rem & 1;
        cp_async16(side + (r * p.side_rows + gi) * 32 + h * 16,
                   (const uint8_t*)p.scales + ((tile0 + r) * groups + g_begin + gi) * 32 + h * 16);
      }
      if constexpr (FMT == INT4_ASYM) {
        const uint32_t zs = side + RT * p.side_rows * 32;
        for (int i = threadIdx.x; i < RT * ng; i += KW * 32) {
          const int r = i / ng, gi = i - r * ng;
          cp_async8(zs + (r * p.side_rows + gi) * 8,
                    (const uint8_t*)p.aux + ((tile0 + r) * groups + g_begin + gi) * 8);
        }
      }
    }
    if constexpr (FMT == NVFP4) {
      const int nb = (int)((ce - cb) * KB / 16);
      for (int i = threadIdx.x; i < RT * nb; i += KW * 32) {
        const int r = i / nb, bi = i - r * nb;
        cp_async16(side + (r * p.side_rows + bi) * 16,
                   (const uint8_t*)p.scales + ((tile0 + r) * (K >> 4) + b16_begin + bi) * 16);
      }
    }
  }

  // lookup tables (CB4: centroids rounded to bf16; NVFP4: E2M1 values)
  uint32_t H[4] = {0, 0, 0, 0}, L[4] = {0, 0, 0, 0};
  if constexpr (FMT == NVFP4) {
    H[0] = 0x3F3F3F00u; H[1] = 0x40404040u; H[2] = 0xBFBFBF80u; H[3] = 0xC0C0C0C0u;
    L[0] = 0xC0800000u; L[1] = 0xC0804000u; L[2] = L[0]; L[3] = L[1];
  }
  if constexpr (FMT == CB4) {
    const float* cen = (const float*)p.aux;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      uint32_t b = f32_to_bf16_bits(__ldg(cen + j));
      H[j >> 2] |= (b >> 8) << (8 * (j & 3));
      L[j >> 2] |= (b & 0xFFu) << (8 * (j & 3));
    }
  }

  float acc[RT][NT][4];
#pragma unroll
  for (int r = 0; r < RT; ++r)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[r][nt][i] = 0.f;

  const uint4 zero4 = make_uint4(0, 0, 0, 0);
  auto load_batch = [&](uint4 (&wv)[UB][RT], int64_t b0) {
#pragma unroll
    for (int u = 0; u < UB; ++u)
#pragma unroll
      for (int r = 0; r < RT; ++r)
        wv[u][r] = (b0 + u < we) ? ld_stream(p.w + ((tile0 + r) * nblk + b0 + u) * 32 + lane)
                                 : zero4;
  };

  auto compute_batch = [&](const uint4 (&wv)[UB][RT], int64_t b0) {
#pragma unroll
    for (int u = 0; u < UB; ++u) {
      if (b0 + u >= we) break;
      const int64_t kblk = (b0 + u) * KB;
      uint4 xv[CPB][NT];
#pragma unroll
      for (int c = 0; c < CPB; ++c)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int tok = g + 8 * nt;
          xv[c][nt] = tok < p.M ? lds128(xs + tok * p.xs_stride +
                                         (uint32_t)((kblk - kbeg) + 32 * c + 8 * tq) * 2u)
                                : zero4;
        }
#pragma unroll
      for (int c = 0; c < CPB; ++c) {
        const int64_t k0 = kblk + 32 * c;
#pragma unroll
        for (int r = 0; r < RT; ++r) {
          const int64_t tile = tile0 + r;
          if constexpr (kIntFmt) {
            const int gi = (int)(k0 / p.G - g_begin);
            const uint32_t sw = lds32(side + (r * p.side_rows + gi) * 32 + g * 4);
            uint32_t off_g = 0x43084308u, off_g8 = 0x43084308u;  // 136 = 128 + 8
            if constexpr (FMT == INT4_ASYM) {
              const uint32_t zb =
                  lds8(side + RT * p.side_rows * 32 + (r * p.side_rows + gi) * 8 + g);
              off_g = (0x4300u + (zb & 15u)) * 0x00010001u;
              off_g8 = (0x4300u + (zb >> 4)) * 0x00010001u;
            }
            float cacc[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
              for (int i = 0; i < 4; ++i) cacc[nt][i] = 0.f;
#pragma unroll
            for (int s = 0; s < 2; ++s) {
              uint32_t a[4];
              if constexpr (FMT == INT8_SYM)
                frag_int8(word(wv[u][r], 2 * s), word(wv[u][r], 2 * s + 1), a);
              else
                frag_int4(word(wv[u][r], 2 * c + s), off_g, off_g8, a);
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
                mma16816(cacc[nt], a, word(xv[c][nt], 2 * s), word(xv[c][nt], 2 * s + 1));
            }
            const float s_g = __uint_as_float(sw << 16), s_g8 = __uint_as_float(sw & 0xFFFF0000u);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              acc[r][nt][0] = fmaf(s_g, cacc[nt][0], acc[r][nt][0]);
              acc[r][nt][1] = fmaf(s_g, cacc[nt][1], acc[r][nt][1]);
              acc[r][nt][2] = fmaf(s_g8, cacc[nt][2], acc[r][nt][2]);
              acc[r][nt][3] = fmaf(s_g8, cacc[nt][3], acc[r][nt][3]);
            }
          } else {
            uint32_t sc_g = 0, sc_g8 = 0;
            if constexpr (FMT == NVFP4) {
              const int bi = (int)(((k0 + 8 * tq) >> 4) - b16_begin);
              const uint32_t sb = lds16(side + (r * p.side_rows + bi) * 16 + g * 2);
              sc_g = f32_to_bf16_bits(e4m3_to_f32(sb & 0xFFu)) * 0x00010001u;
              sc_g8 = f32_to_bf16_bits(e4m3_to_f32(sb >> 8)) * 0x00010001u;
            }
#pragma unroll
            for (int s = 0; s < 2; ++s) {
              uint32_t a[4];
              frag_table<FMT == NVFP4>(word(wv[u][r], 2 * c + s), H, L, a);
              if constexpr (FMT == NVFP4) {
                a[0] = bmul2(a[0], sc_g);
                a[1] = bmul2(a[1], sc_g8);
                a[2] = bmul2(a[2], sc_g);
                a[3] = bmul2(a[3], sc_g8);
              }
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
                mma16816(acc[r][nt], a, word(xv[c][nt], 2 * s), word(xv[c][nt], 2 * s + 1));
            }
          }
        }
      }
    }
  };

  // two register batches in flight: while one batch is converted and
  // multiplied, the loads of the next one are outstanding
  uint4 wa[UB][RT], wz[UB][RT];
  load_batch(wa, wb);
  cp_async_wait_all();
  __syncthreads();
  for (int64_t b0 = wb; b0 < we; b0 += 2 * UB) {
    load_batch(wz, b0 + UB);
    compute_batch(wa, b0);
    load_batch(wa, b0 + 2 * UB);
    compute_batch(wz, b0 + UB);
  }

  // ---- reduction: warps -> CTA partial (shared) -> cluster rank 0 (DSMEM)
#pragma unroll
  for (int r = 0; r < RT; ++r)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) red[(warp * NV + (r * NT + nt) * 4 + i) * 32 + lane] = acc[r][nt][i];
  __syncthreads();
  float* part = red + KW * NV * 32;
  for (int idx = threadIdx.x; idx < NV * 32; idx += KW * 32) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < KW; ++w) s += red[w * NV * 32 + idx];
    part[idx] = s;
  }
  if (cs > 1) cg::this_cluster().sync();
  else __syncthreads();
  if (rank == 0) {
    float tsc = 1.f;
    if constexpr (FMT == NVFP4) tsc = __ldg((const float*)p.aux);
    for (int idx = threadIdx.x; idx < NV * 32; idx += KW * 32) {
      float tot = part[idx];
      for (int q = 1; q < cs; ++q) tot += cg::this_cluster().map_shared_rank(part, q)[idx];
      const int v = idx >> 5, ln = idx & 31;
      const int r = v / (NT * 4), nt = (v / 4) % NT, i = v & 3;
      const int gg = ln >> 2, tt = ln & 3;
      const int64_t n = (tile0 + r) * 16 + gg + 8 * (i >> 1);
      const int m = nt * 8 + 2 * tt + (i & 1);
      if (m < p.M) {
        float fold = tsc;
        if constexpr (FMT == CB4) fold = bf16_bits_to_f32(__ldg((const uint16_t*)p.scales + n));
        float y = tot * fold;
        if (p.bias) y += bf16_bits_to_f32(__ldg(p.bias + n));
        p.out[(int64_t)m * p.N + n] = (uint16_t)f32_to_bf16_bits(y);
      }
    }
  }
  if (cs > 1) cg::this_cluster().sync();
}

template <int FMT, int NT, int RT>
cudaError_t launch_t(const DecodeParams& p, int grid, cudaStream_t st) {
  constexpr int KW = 4, UB = 4;
  auto kern = decode_kernel<FMT, NT, RT, KW, UB>;
  const size_t smem = (size_t)p.xs_bytes + (size_t)p.side_bytes +
                      (size_t)(KW + 1) * RT * NT * 4 * 32 * sizeof(float);
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         227 * 1024);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(KW * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.cs > 1 ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

template <int FMT>
cudaError_t launch_fmt(const DecodeParams& p, int nt, int rt, int grid, cudaStream_t st) {
  if (nt == 1) return rt == 2 ? launch_t<FMT, 1, 2>(p, grid, st) : launch_t<FMT, 1, 1>(p, grid, st);
  return rt == 2 ? launch_t<FMT, 2, 2>(p, grid, st) : launch_t<FMT, 2, 1>(p, grid, st);
}

}  // namespace

cudaError_t launch_decode(const LinearArgs& a) {
  DecodeParams p;
  p.x = (const uint16_t*)a.x;
  p.w = (const uint4*)a.w;
  p.scales = a.scales;
  p.aux = a.aux;
  p.bias = (const uint16_t*)a.bias;
  p.out = (uint16_t*)a.out;
  p.M = (int)a.M;
  p.N = (int)a.N;
  p.K = (int)a.K;
  p.G = a.G;
  const int nt = a.M <= 8 ? 1 : 2;
  const int64_t tiles = a.N / 16;
  const int rt = (tiles % 2 == 0) ? 2 : 1;
  const int64_t rowgroups = tiles / rt;
  const int kb = block_k(a.fmt);
  const int64_t nblk = a.K / kb;
  // split K over a cluster: enough CTAs to cover the SMs twice, and a staged
  // X slice of at most 96 KB
  const int64_t target = 2LL * device_sm_count();
  int64_t cs = (target + rowgroups - 1) / rowgroups;
  const int64_t x_bytes_all = a.M * a.K * 2;
  const int64_t cs_x = (x_bytes_all + 98303) / 98304;
  if (cs < cs_x) cs = cs_x;
  if (cs > 8) cs = 8;
  if (cs > nblk / 4) cs = nblk / 4;  // keep every warp busy
  if (cs < 1) cs = 1;
  const int64_t max_blocks = (nblk + cs - 1) / cs;
  const int64_t stride = ((max_blocks * kb * 2 + 127) / 128) * 128 + 64;
  if (stride * a.M > 200 * 1024) return cudaErrorInvalidValue;  // K too large for M <= 16
  p.cs = (int)cs;
  p.xs_stride = (int)stride;
  p.xs_bytes = (int)(stride * a.M);
  // staged side data per row tile: a K range of max_blocks*kb may touch one
  // more group than it spans
  if (is_int_fmt(a.fmt)) {
    p.side_rows = (int)((max_blocks * kb + a.G - 1) / a.G + 1);
    p.side_bytes = rt * p.side_rows * (a.fmt == INT4_ASYM ? 40 : 32);
  } else if (a.fmt == NVFP4) {
    p.side_rows = (int)(max_blocks * kb / 16);
    p.side_bytes = rt * p.side_rows * 16;
  } else {
    p.side_rows = 0;
    p.side_bytes = 0;
  }
  p.side_bytes = (p.side_bytes + 15) & ~15;
  const int grid = (int)(rowgroups * cs);
  switch (a.fmt) {
    case INT4_SYM: return launch_fmt<INT4_SYM>(p, nt, rt, grid, a.stream);
    case INT4_ASYM: return launch_fmt<INT4_ASYM>(p, nt, rt, grid, a.stream);
    case INT8_SYM: return launch_fmt<INT8_SYM>(p, nt, rt, grid, a.stream);
    case CB4: return launch_fmt<CB4>(p, nt, rt, grid, a.stream);
    case NVFP4: return launch_fmt<NVFP4>(p, nt, rt, grid, a.stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace wq

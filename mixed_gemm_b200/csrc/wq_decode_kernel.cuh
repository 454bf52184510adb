// The decode kernel (M <= 16) as a template, shared by the translation units
// that instantiate it (wq_decode_k*.cu, a few formats each, so that they
// compile in parallel); the launch heuristic lives in wq_decode.cu.  The
// design notes are at the top of wq_decode.cu.
#pragma once

#include <cooperative_groups.h>
#include <stdlib.h>

#include "wq_frag.cuh"
#include "wq_internal.cuh"

namespace wq {

struct DecodeParams {
  unsigned* err;  // the decode error word (bit 128: activation-slice wait ran out)
  const uint16_t* x;
  const uint4* w;
  const void* scales;
  const void* aux;
  const uint16_t* bias;
  uint16_t* out;
  int M, N, K, G, cs;
  int xs_stride;  // bytes per token row of the staged X slice
  int xs_bytes;   // bytes of the staged X slice (M rows)
  int gshift;     // log2(group size) for INT formats
  int side_rows;  // per row tile: scale groups (INT) or 16-K blocks (NVFP4) staged
  int side_bytes; // bytes of staged scales / zero-points / block scales
  int red_off;    // offset of the cluster partial slots (after the larger of
                  // the staged data and the per-warp partials)
  int bar_off;    // offset of the mbarrier the X-slice bulk copies complete on
  int swiglu;     // x rows are [up | gate] (2K values); the gate slice is
                  // staged at xs_bytes past the up slice
  // grouped (mixture-of-experts) launch: device row offsets [E + 1] (rows of
  // x sorted by expert, T rows); the y index of a CTA is a tile of the
  // device-side schedule (experts in order, ceil(count / (8 NT)) token
  // chunks each); expert e's packed weight, scales and aux lie e * *_stride
  // bytes after expert 0's, its bias e * N values.  NULL: one linear.
  const int64_t* offsets;
  int E, T, ytiles;
  int64_t w_stride, scale_stride, aux_stride;
#ifdef WQ_FAULT_TEST
  int fault_skip_x;  // test build only (see the activation-slice stage)
#endif
};

// Launch the decode kernel of format `fmt` (one of the formats its
// translation unit instantiates; cudaErrorInvalidValue otherwise).
cudaError_t launch_decode_k0(int fmt, const DecodeParams& p, int nt, int rt, int kw, int d,
                             int grid, cudaStream_t st);
cudaError_t launch_decode_k1(int fmt, const DecodeParams& p, int nt, int rt, int kw, int d,
                             int grid, cudaStream_t st);
cudaError_t launch_decode_k2(int fmt, const DecodeParams& p, int nt, int rt, int kw, int d,
                             int grid, cudaStream_t st);
cudaError_t launch_decode_k3(int fmt, const DecodeParams& p, int nt, int rt, int kw, int d,
                             int grid, cudaStream_t st);

namespace cg = cooperative_groups;

namespace {

__device__ __forceinline__ uint2 ld_stream8(const uint2* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}
__device__ __forceinline__ uint32_t ld_stream4(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
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
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
// Bounded wait for phase 0 of the X-slice barrier.  The limit is far beyond
// any copy time; a wait that runs out sets bit 128 of the decode error word
// and leaves the block's output unwritten.
__device__ __forceinline__ bool mbar_wait0(uint32_t bar, unsigned* err) {
#ifdef WQ_FAULT_TEST
  const uint32_t limit = 1u << 16;  // test build only: short wait
#else
  const uint32_t limit = 1u << 22;
#endif
  for (uint32_t i = 0; i < limit; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar)
        : "memory");
    if (ok) return true;
  }
  atomicOr(err, 128u);
  return false;
}
// The same bounded wait, at cluster scope (acquire of the other ranks'
// distributed-shared-memory writes), for phase 0 of the reduction barrier.
__device__ __forceinline__ bool mbar_wait0_cluster(uint32_t bar, unsigned* err) {
#ifdef WQ_FAULT_TEST
  const uint32_t limit = 1u << 16;
#else
  const uint32_t limit = 1u << 22;
#endif
  for (uint32_t i = 0; i < limit; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], 0;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar)
        : "memory");
    if (ok) return true;
  }
  atomicOr(err, 128u);
  return false;
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
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t addr, const uint4& v) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ uint4 swiglu_x8(const uint4& u, const uint4& g) {
  return make_uint4(swiglu_pair(u.x, g.x), swiglu_pair(u.y, g.y), swiglu_pair(u.z, g.z),
                    swiglu_pair(u.w, g.w));
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
}

// KW warps per CTA; each keeps a ring of D blocks (per row tile) of weight
// loads in flight: after block j is consumed, the load of block j + D is
// issued into the freed registers.
template <int FMT, int NT, int RT, int KW, int D>
__global__ void __launch_bounds__(KW * 32) decode_kernel(const DecodeParams p) {
  constexpr bool kFp8 = FMT == FP8_E4M3 || FMT == FP8_E5M2;
  constexpr bool kByte = FMT == INT8_SYM || kFp8;  // one byte per code
  constexpr int KB = kByte ? 32 : 64;             // K per 512-byte block
  constexpr int CPB = kByte ? 1 : 2;              // 32-K chunks per block
  constexpr int NV = RT * NT * 4;                  // accumulators per lane
  // one scale per group of K folded into fp32 sums (INT formats, FP8)
  constexpr bool kIntFmt =
      FMT == INT4_SYM || FMT == INT4_ASYM || FMT == INT8_SYM || FMT == INT2_SYM ||
      FMT == INT3_SYM || kFp8;
  constexpr int SB = kFp8 ? 64 : 32;   // bytes per (row tile, group) of scales

  extern __shared__ __align__(16) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, tq = lane & 3;
  const int cs = p.cs;
  // this call's (or, grouped, this schedule tile's) rows and buffers
  int M = p.M;
  const uint16_t* xg = p.x;
  uint16_t* outg = p.out;
  const uint4* wg = p.w;
  const uint8_t* scales_g = (const uint8_t*)p.scales;
  const uint8_t* aux_g = (const uint8_t*)p.aux;
  const uint16_t* bias_g = p.bias;
  if (p.offsets) {
    // The routing offsets may be the previous kernel's output: wait first
    // (no weight prefetch ahead of the dependency in this mode).  Warp 0
    // finds this CTA's (expert, token chunk) with a warp prefix sum over
    // the experts' chunk counts; invalid offsets make an expert empty.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    int* sched = (int*)(smem + p.bar_off + 16);
    if (warp == 0) {
      const int target = (int)blockIdx.y;
      int base = 0, found = 0;
      for (int c0 = 0; c0 < p.E && !found; c0 += 32) {
        const int ee = c0 + lane;
        int cnt = 0, a = 0;
        if (ee < p.E) {
          const int64_t a64 = p.offsets[ee], b64 = p.offsets[ee + 1];
          if (a64 >= 0 && a64 <= b64 && b64 <= p.T) {
            a = (int)a64;
            cnt = (int)(b64 - a64);
          } else if (blockIdx.x == 0 && blockIdx.y == 0) {
            atomicOr(p.err, 256u);
          }
        }
        const int nt = (cnt + 8 * NT - 1) / (8 * NT);
        int incl = nt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        const bool mine = nt > 0 && target >= base + incl - nt && target < base + incl;
        const unsigned bal = __ballot_sync(0xffffffffu, mine);
        if (mine) {
          sched[0] = ee;
          sched[1] = a + (target - (base + incl - nt)) * 8 * NT;
          const int left = cnt - (target - (base + incl - nt)) * 8 * NT;
          sched[2] = left < 8 * NT ? left : 8 * NT;
        }
        found = bal != 0;
        base += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (!found && lane == 0) sched[0] = -1;
    }
    __syncthreads();
    if (sched[0] < 0) return;  // the whole cluster shares blockIdx.y: all return
    const int e = sched[0];
    M = sched[2];
    const int64_t xrow_el = p.swiglu ? 2 * (int64_t)p.K : (int64_t)p.K;
    xg = p.x + (int64_t)sched[1] * xrow_el;
    outg = p.out + (int64_t)sched[1] * p.N;
    wg = p.w + (int64_t)e * (p.w_stride / 16);
    scales_g += (int64_t)e * p.scale_stride;
    if (aux_g) aux_g += (int64_t)e * p.aux_stride;
    if (bias_g) bias_g += (int64_t)e * p.N;
    __syncthreads();  // sched read by every thread before the barrier memory is reused
  }
  // cluster (cs, 1, 1) over a grid of rowgroups * cs blocks: the cluster
  // index is the row group, the rank in the cluster the K slice
  int rank = 0, rgroup = (int)blockIdx.x;
  if (cs > 1) {
    asm("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
    asm("mov.u32 %0, %%clusterid.x;" : "=r"(rgroup));
  }
  const int tile0 = rgroup * RT;
  const uint32_t xbar = (uint32_t)__cvta_generic_to_shared(smem) + (uint32_t)p.bar_off;
  // rank 0's reduction barrier: one arrival per other rank of the cluster
  const uint32_t rbar = xbar + 8u;
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(xbar) : "memory");
    if (cs > 1 && rank == 0)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(rbar), "r"(cs - 1) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  const int K = p.K;
  const int nblk = K / KB;
  const int groups = kIntFmt ? K >> p.gshift : 0;

  if (cs > 1) cluster_arrive_relaxed();  // matched by the wait before DSMEM writes

  // this CTA's K blocks [cb, ce), this warp's [wb, we)
  const int cb = (int)((unsigned)(rank * nblk) / (unsigned)cs);
  const int ce = (int)((unsigned)((rank + 1) * nblk) / (unsigned)cs);
  const int wb = cb + warp * (ce - cb) / KW, we = cb + (warp + 1) * (ce - cb) / KW;
  const int nb = we - wb;

  // Stage in shared memory, with cp.async, everything the K loop reads besides
  // the weight stream: the CTA's slice of X (tokens < M, K in
  // [cb*KB, ce*KB)), and the group scales + zero-points (INT) or E4M3 block
  // scales (NVFP4) of its row tiles over that K range.
  const uint32_t xs = (uint32_t)__cvta_generic_to_shared(smem);
  const uint32_t side = xs + (uint32_t)p.xs_bytes * (p.swiglu ? 2u : 1u);
  const int kbeg = cb * KB;
  const int g_begin = kIntFmt ? kbeg >> p.gshift : 0;  // first scale group staged
  const int b16_begin = kbeg >> 4;                      // first NVFP4 16-block staged
  {
    if constexpr (kIntFmt) {
      const int ng = ((ce * KB - 1) >> p.gshift) + 1 - g_begin;
      // scales: SB bytes per (tile, group) -> SB / 16 chunks of 16 bytes
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        const uint8_t* src = scales_g + ((int64_t)(tile0 + r) * groups + g_begin) * SB;
        for (int i = threadIdx.x; i < ng * (SB / 16); i += KW * 32)
          cp_async16(side + (r * p.side_rows) * SB + i * 16, src + i * 16);
      }
      if constexpr (FMT == INT4_ASYM) {
        const uint32_t zs = side + RT * p.side_rows * 32;
#pragma unroll
        for (int r = 0; r < RT; ++r) {
          const uint8_t* src = aux_g + ((int64_t)(tile0 + r) * groups + g_begin) * 8;
          for (int i = threadIdx.x; i < ng; i += KW * 32)
            cp_async8(zs + (r * p.side_rows + i) * 8, src + i * 8);
        }
      }
    }
    if constexpr (FMT == NVFP4 || FMT == MXFP4) {
      // block scales: one 16-byte entry per (row tile, block of 16 / 32 K)
      constexpr int LB = FMT == NVFP4 ? 4 : 5;  // log2 of the block
      const int nbk = ((ce - cb) * KB) >> LB;
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        const uint8_t* src = scales_g +
                             ((int64_t)(tile0 + r) * (K >> LB) + (kbeg >> LB)) * 16;
        for (int i = threadIdx.x; i < nbk; i += KW * 32)
          cp_async16(side + (r * p.side_rows + i) * 16, src + i * 16);
      }
    }
  }

  // weight ring: D blocks per row tile in flight
  const uint4* wrow[RT];
#pragma unroll
  for (int r = 0; r < RT; ++r) wrow[r] = wg + (int64_t)(tile0 + r) * nblk * 32 + lane;
  // INT2: 256-byte blocks, 8 bytes per lane (the words 0..1 of its uint4)
  // INT3: 384-byte blocks, 8 low-plane bytes and 4 high-plane bytes per lane
  auto ld_block = [&](int r, int blk) -> uint4 {
    if constexpr (FMT == INT3_SYM) {
      const uint8_t* bp = (const uint8_t*)wg + ((int64_t)(tile0 + r) * nblk + blk) * 384;
      const uint2 lo = ld_stream8((const uint2*)(bp + lane * 8));
      const uint32_t hi = ld_stream4((const uint32_t*)(bp + 256 + lane * 4));
      return make_uint4(lo.x, lo.y, hi, 0u);
    } else if constexpr (FMT == INT2_SYM) {
      const uint2 v = ld_stream8((const uint2*)wg + ((int64_t)(tile0 + r) * nblk + blk) * 32 + lane);
      return make_uint4(v.x, v.y, 0u, 0u);
    } else {
      return ld_stream(wrow[r] + blk * 32);
    }
  };
  uint4 wv[D][RT];
#pragma unroll
  for (int j = 0; j < D; ++j)
#pragma unroll
    for (int r = 0; r < RT; ++r)
      if (j < nb) wv[j][r] = ld_block(r, wb + j);

  // Programmatic dependent launch: the packed weight and its scales never
  // depend on the previous kernel in the stream, so they are requested above
  // before waiting for it; X (typically the previous kernel's output) is read
  // and Y written only after the wait.  The next kernel may be scheduled as
  // soon as every block of this one got here (signalling at kernel entry
  // instead measured slower: the next kernel's blocks then compete with this
  // one's compute).  One bulk copy per token row stages the X slice.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int64_t xrow = p.swiglu ? 2 * (int64_t)K : (int64_t)K;  // elements per x row
#ifdef WQ_FAULT_TEST
  // test build only: block 0 neither arrives on nor copies into its
  // activation-slice barrier, so its bounded wait runs out
  if (warp == 0 && !(p.fault_skip_x && blockIdx.x == 0)) {
#else
  if (warp == 0) {
#endif
    // lane 0 announces the bytes, then lane t copies token row t (rows
    // issued in parallel rather than one after another)
    const uint32_t xbytes = (uint32_t)((ce - cb) * KB * 2);
    if (lane == 0)
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(xbar),
                   "r"(xbytes * (uint32_t)M * (p.swiglu ? 2u : 1u))
                   : "memory");
    __syncwarp();
    for (int tok = lane; tok < M; tok += 32) {
      bulk_g2s(xs + tok * p.xs_stride, xg + tok * xrow + kbeg, xbytes, xbar);
      if (p.swiglu)
        bulk_g2s(xs + p.xs_bytes + tok * p.xs_stride, xg + tok * xrow + K + kbeg, xbytes,
                 xbar);
    }
  }

  // NVFP4: a 256-entry table E4M3 code -> bf16x2 (e4m3 * 2^119) pair, the
  // factor frag_nvfp4 expects, built once per CTA (covered by the barrier
  // after the staging wait)
  const uint32_t scale_tab = side + (uint32_t)(RT * p.side_rows * 16);
  if constexpr (FMT == NVFP4 || FMT == MXFP4) {
    for (int c = threadIdx.x; c < 256; c += KW * 32)
      asm volatile("st.shared.u32 [%0], %1;" ::"r"(scale_tab + c * 4),
                   "r"(FMT == NVFP4 ? nvfp4_scale_pair(c) : mx_lo_pair(c))
                   : "memory");
  }

  // lookup tables (CB4): each fp32 centroid as a bf16 high part plus the
  // bf16 rounding of the remainder (c - hi is exact in fp32), so the two
  // tensor-core products carry the centroid to within 2^-18 of its value
  uint32_t H[4] = {0, 0, 0, 0}, L[4] = {0, 0, 0, 0};
  uint32_t H2[4] = {0, 0, 0, 0}, L2[4] = {0, 0, 0, 0};
  if constexpr (FMT == CB4) {
    const float* cen = (const float*)aux_g;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float c = __ldg(cen + j);
      const uint32_t b = f32_to_bf16_bits(c);
      const uint32_t b2 = f32_to_bf16_bits(c - bf16_bits_to_f32((uint16_t)b));
      H[j >> 2] |= (b >> 8) << (8 * (j & 3));
      L[j >> 2] |= (b & 0xFFu) << (8 * (j & 3));
      H2[j >> 2] |= (b2 >> 8) << (8 * (j & 3));
      L2[j >> 2] |= (b2 & 0xFFu) << (8 * (j & 3));
    }
  }

  // NVFP4 / CB4 with one token tile: the two 16-K steps of a chunk
  // accumulate into separate chains (NS = 2), so consecutive tensor-core
  // steps overlap (INT formats already alternate per group; measured faster
  // with one chain).
  constexpr int NS = (NT == 1 && !kIntFmt) ? 2 : 1;
  float acc[NS][RT][NT][4];
#pragma unroll
  for (int q = 0; q < NS; ++q)
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[q][r][nt][i] = 0.f;
  // INT group state: chunk accumulators, packed scales, zero-point offsets
  // (bf16 pairs of 128 + z; 136 = 128 + 8 for offset-binary signed codes)
  float cacc[NS][kIntFmt ? RT : 1][NT][4];
  uint32_t gsw[RT], gsw2[RT], goff[RT][2];
  const int gmask = kIntFmt ? (1 << p.gshift) - 1 : 0;
#pragma unroll
  for (int r = 0; r < RT; ++r) {
    gsw[r] = gsw2[r] = 0;
    goff[r][0] = goff[r][1] = 0x43084308u;
  }

  cp_async_wait_all();
  __syncthreads();  // staged scales, the NVFP4 table and the barrier init are visible
  const bool xok = mbar_wait0(xbar, p.err);  // false never in practice: then nothing is stored
  if (p.swiglu) {
    // SwiGLU input: a = bf16(up * silu(gate)), written over the staged up slice
    const int chunks = (ce - cb) * KB / 8;  // 16-byte chunks per token row
    for (int i = threadIdx.x; i < M * chunks; i += KW * 32) {
      const int tok = i / chunks, c = i - tok * chunks;
      const uint32_t ua = xs + (uint32_t)(tok * p.xs_stride + c * 16);
      const uint4 u = lds128(ua), gt = lds128(ua + (uint32_t)p.xs_bytes);
      sts128(ua, swiglu_x8(u, gt));
    }
    __syncthreads();
  }

  const uint4 zero4 = make_uint4(0, 0, 0, 0);
  auto compute_block = [&](const uint4 (&wb_)[RT], int b) {
    const int kblk = b * KB;
    uint4 xv[CPB][NT];
#pragma unroll
    for (int c = 0; c < CPB; ++c)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int tok = g + 8 * nt;
        xv[c][nt] = tok < M ? lds128(xs + tok * p.xs_stride +
                                       (uint32_t)((kblk - kbeg) + 32 * c + 8 * tq) * 2u)
                              : zero4;
      }
#pragma unroll
    for (int c = 0; c < CPB; ++c) {
      const int k0 = kblk + 32 * c;
      // INT formats: one accumulator per group of K (per row tile), scaled
      // once when the group ends; the group's scale and zero-point are read
      // once when it starts (a warp's range may begin or end inside a group)
      const bool gstart = ((k0 & gmask) == 0) || (k0 == wb * KB);
      const bool gend = (((k0 + 32) & gmask) == 0) || (k0 + 32 == we * KB);
      if constexpr (kIntFmt) {
        if (gstart) {
          const int gi = (k0 >> p.gshift) - g_begin;
#pragma unroll
          for (int r = 0; r < RT; ++r) {
            if constexpr (kFp8) {  // fp32 scales of rows g, g + 8
              const uint2 sv = lds64(side + (r * p.side_rows + gi) * 64 + g * 8);
              gsw[r] = sv.x;
              gsw2[r] = sv.y;
            } else {
              gsw[r] = lds32(side + (r * p.side_rows + gi) * 32 + g * 4);
            }
            if constexpr (FMT == INT4_ASYM) {
              const uint32_t zb =
                  lds8(side + RT * p.side_rows * 32 + (r * p.side_rows + gi) * 8 + g);
              goff[r][0] = (0x4300u + (zb & 15u)) * 0x00010001u;
              goff[r][1] = (0x4300u + (zb >> 4)) * 0x00010001u;
            }
#pragma unroll
            for (int q = 0; q < NS; ++q)
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) cacc[q][r][nt][i] = 0.f;
          }
        }
      }
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        if constexpr (kIntFmt) {
#pragma unroll
          for (int s = 0; s < 2; ++s) {
            uint32_t a[4];
            if constexpr (FMT == INT8_SYM)
              frag_int8(word(wb_[r], 2 * s), word(wb_[r], 2 * s + 1), a);
            else if constexpr (FMT == FP8_E4M3)
              frag_e4m3(word(wb_[r], 2 * s), word(wb_[r], 2 * s + 1), a);
            else if constexpr (FMT == FP8_E5M2)
              frag_e5m2(word(wb_[r], 2 * s), word(wb_[r], 2 * s + 1), a);
            else
              if constexpr (FMT == INT3_SYM)
                frag_int3(word(wb_[r], c), wb_[r].z, c, s, 0x43044304u, a);
              else if constexpr (FMT == INT2_SYM)
                frag_int2(word(wb_[r], c), s, 0x43024302u, a);
              else
                frag_int4(word(wb_[r], 2 * c + s), goff[r][0], goff[r][1], a);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
              mma16816(cacc[s % NS][r][nt], a, word(xv[c][nt], 2 * s),
                       word(xv[c][nt], 2 * s + 1));
          }
          if (gend) {
            const float s_g =
                kFp8 ? __uint_as_float(gsw[r]) : __uint_as_float(gsw[r] << 16);
            const float s_g8 = kFp8 ? __uint_as_float(gsw2[r])
                                               : __uint_as_float(gsw[r] & 0xFFFF0000u);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              float c4[4];
#pragma unroll
              for (int i = 0; i < 4; ++i)
                c4[i] = NS == 2 ? cacc[0][r][nt][i] + cacc[NS - 1][r][nt][i] : cacc[0][r][nt][i];
              acc[0][r][nt][0] = fmaf(s_g, c4[0], acc[0][r][nt][0]);
              acc[0][r][nt][1] = fmaf(s_g, c4[1], acc[0][r][nt][1]);
              acc[0][r][nt][2] = fmaf(s_g8, c4[2], acc[0][r][nt][2]);
              acc[0][r][nt][3] = fmaf(s_g8, c4[3], acc[0][r][nt][3]);
            }
          }
        } else {
          uint32_t sc_g = 0, sc_g8 = 0, eg = 0, eg8 = 0;
          if constexpr (FMT == NVFP4) {
            const int bi = ((k0 + 8 * tq) >> 4) - b16_begin;
            const uint32_t sb = lds16(side + (r * p.side_rows + bi) * 16 + g * 2);
            sc_g = lds32(scale_tab + (sb & 0xFFu) * 4);
            sc_g8 = lds32(scale_tab + (sb >> 8) * 4);
          }
          if constexpr (FMT == MXFP4) {  // a 32-K chunk is one MXFP4 block
            const int bi = (k0 >> 5) - (kbeg >> 5);
            const uint32_t sb = lds16(side + (r * p.side_rows + bi) * 16 + g * 2);
            eg = sb & 0xFFu;
            eg8 = sb >> 8;
            sc_g = lds32(scale_tab + eg * 4);
            sc_g8 = lds32(scale_tab + eg8 * 4);
          }
#pragma unroll
          for (int s = 0; s < 2; ++s) {
            uint32_t a[4];
            if constexpr (FMT == NVFP4 || FMT == MXFP4)
              frag_nvfp4(word(wb_[r], 2 * c + s), sc_g, sc_g8, a);
            else
              frag_table<false>(word(wb_[r], 2 * c + s), H, L, a);
            if constexpr (FMT == MXFP4) {
              if (eg > 128u && eg != 255u) {
                a[0] = bmul2(a[0], mx_hi_pair(eg));
                a[2] = bmul2(a[2], mx_hi_pair(eg));
              }
              if (eg8 > 128u && eg8 != 255u) {
                a[1] = bmul2(a[1], mx_hi_pair(eg8));
                a[3] = bmul2(a[3], mx_hi_pair(eg8));
              }
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
              mma16816(acc[s % NS][r][nt], a, word(xv[c][nt], 2 * s),
                       word(xv[c][nt], 2 * s + 1));
            if constexpr (FMT == CB4) {  // the centroids' remainders
              frag_table<false>(word(wb_[r], 2 * c + s), H2, L2, a);
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
                mma16816(acc[s % NS][r][nt], a, word(xv[c][nt], 2 * s),
                         word(xv[c][nt], 2 * s + 1));
            }
          }
        }
      }
    }
  };

  for (int i = 0; i < nb; i += D) {
#pragma unroll
    for (int j = 0; j < D; ++j) {
      if (i + j < nb) {
        compute_block(wv[j], wb + i + j);
        if (i + j + D < nb) {
#pragma unroll
          for (int r = 0; r < RT; ++r) wv[j][r] = ld_block(r, wb + i + j + D);
        }
      }
    }
  }

  // ---- reduction: warps -> CTA partial in this CTA's shared memory (the X
  // slice region is free now); the CTA partial goes into slot `rank` of
  // cluster rank 0's shared memory.  The other ranks then arrive once each
  // on rank 0's reduction barrier (release at cluster scope) and finish;
  // rank 0 waits for their arrivals, sums the slots in rank order and stores.
  __syncthreads();  // every warp is done reading the staged slice
  float* loc = (float*)smem;
  float* slots = (float*)(smem + p.red_off);
#pragma unroll
  for (int r = 0; r < RT; ++r)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i)
        loc[(warp * NV + (r * NT + nt) * 4 + i) * 32 + lane] =
            NS == 2 ? acc[0][r][nt][i] + acc[NS - 1][r][nt][i] : acc[0][r][nt][i];
  __syncthreads();
  float* slots0 = slots;
  if (cs > 1) {
    cluster_wait();  // every CTA of the cluster has started
    slots0 = cg::this_cluster().map_shared_rank(slots, 0);
  }
  for (int idx = threadIdx.x; idx < NV * 32; idx += KW * 32) {
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < KW; ++w) sum += loc[w * NV * 32 + idx];
    slots0[rank * NV * 32 + idx] = sum;
  }
  bool rok = true;
  if (cs > 1 && rank != 0) {
    asm volatile("fence.acq_rel.cluster;" ::: "memory");  // this thread's slot writes
    __syncthreads();
    if (threadIdx.x == 0) {
      uint32_t rb0;
      asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(rb0) : "r"(rbar));
      asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(rb0)
                   : "memory");
    }
    return;
  }
  __syncthreads();  // rank 0's own slot
  if (cs > 1) rok = mbar_wait0_cluster(rbar, p.err);

  float tsc = 1.f;
  if constexpr (FMT == NVFP4) tsc = __ldg((const float*)aux_g) * 128.f;  // 2^7 of frag_nvfp4
  for (int idx = threadIdx.x; idx < NV * 32; idx += KW * 32) {
    float tot = 0.f;
    for (int q = 0; q < cs; ++q) tot += slots[q * NV * 32 + idx];
    const int v = idx >> 5, ln = idx & 31;
    const int r = v / (NT * 4), nt = (v / 4) % NT, i = v & 3;
    const int gg = ln >> 2, tt = ln & 3;
    const int n = (tile0 + r) * 16 + gg + 8 * (i >> 1);
    const int m = nt * 8 + 2 * tt + (i & 1);
    if (m < M && xok && rok) {
      float fold = tsc;
      if constexpr (FMT == CB4) fold = bf16_bits_to_f32(__ldg((const uint16_t*)scales_g + n));
      float y = tot * fold;
      if (bias_g) y += bf16_bits_to_f32(__ldg(bias_g + n));
      outg[(int64_t)m * p.N + n] = (uint16_t)f32_to_bf16_bits(y);
    }
  }
}

template <int FMT, int NT, int RT, int KW, int D>
cudaError_t launch_t(const DecodeParams& p, int grid, cudaStream_t st) {
  auto kern = decode_kernel<FMT, NT, RT, KW, D>;
  const size_t smem = (size_t)p.bar_off + 32;
  cudaError_t e = ensure_max_dynamic_smem((const void*)kern, 227 * 1024);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, p.ytiles);
  cfg.blockDim = dim3(KW * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = p.cs;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.cs > 1 ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

// d = 8 (a deeper weight ring) is instantiated for one or two row tiles only
template <int FMT, int KW>
cudaError_t launch_kw(const DecodeParams& p, int nt, int rt, int d, int grid, cudaStream_t st) {
  if (d == 8 && rt <= 2) {
    if (nt == 1)
      return rt == 2 ? launch_t<FMT, 1, 2, KW, 8>(p, grid, st) : launch_t<FMT, 1, 1, KW, 8>(p, grid, st);
    return rt == 2 ? launch_t<FMT, 2, 2, KW, 8>(p, grid, st) : launch_t<FMT, 2, 1, KW, 8>(p, grid, st);
  }
  if (nt == 1) {
    if (rt == 4) return launch_t<FMT, 1, 4, KW, 4>(p, grid, st);
    if (rt == 2) return launch_t<FMT, 1, 2, KW, 4>(p, grid, st);
    return launch_t<FMT, 1, 1, KW, 4>(p, grid, st);
  }
  if (rt == 4) return launch_t<FMT, 2, 4, KW, 4>(p, grid, st);
  if (rt == 2) return launch_t<FMT, 2, 2, KW, 4>(p, grid, st);
  return launch_t<FMT, 2, 1, KW, 4>(p, grid, st);
}

template <int FMT>
cudaError_t launch_fmt(const DecodeParams& p, int nt, int rt, int kw, int d, int grid,
                       cudaStream_t st) {
  return kw == 8 ? launch_kw<FMT, 8>(p, nt, rt, d, grid, st)
                 : launch_kw<FMT, 4>(p, nt, rt, d, grid, st);
}

}  // namespace

}  // namespace wq

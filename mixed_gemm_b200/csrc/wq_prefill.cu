// Prefill path (M > 16): tcgen05 tensor cores, weights dequantized in shared
// memory, accumulators in tensor memory.
//
// The product is computed transposed, D[w_row, token] = W[w_row, :] . X[token, :],
// so that the dequantized weight tile is the 128-row A operand and the tokens
// are the N side of the MMA (N = 32..256, chosen from M).  Four warpgroups:
//   warp 0              one lane TMA-loads, per 64-wide K step, the X tile
//                       (bf16, 128-byte swizzle, zero fill past M) and the
//                       packed tile of 8 row tiles into a stage of the TMA
//                       ring; the other lanes copy the stage's NVFP4 block
//                       scales or zero-points beside it (cp.async completing
//                       on the same barrier), so the dequant warps never wait
//                       on global memory;
//   warps 4..7          convert packed codes to bf16 in registers (the decode
//                       path's fragment decoders) and store them, in the
//                       canonical 128-byte-swizzled K-major layout, into the
//                       A tile that belongs to the same ring slot;
//   warp 1 (one lane)   issues four tcgen05.mma.kind::f16 (K = 16 each) per
//                       K step and returns the slot with one commit;
//   warps 8..15         fold and epilogue.
// A slot (X tile, packed tile, A tile) is refilled once its MMAs complete:
// their completion implies the dequant warps read the packed tile before, so
// one commit per K step frees everything the slot holds.  The MMA issuer is
// the busiest serial chain of the kernel (each tcgen05 instruction costs it
// tens of cycles), so it carries as few barrier operations as possible.
// INT formats keep the tile values exact: the tile holds the integer code (or
// code minus zero-point), each group of K is accumulated into its own
// tensor-memory buffer (two buffers alternate; a group boundary may fall
// inside a stage for groups of 32), and the fold warps add
// group_scale[row] * partial into fp32 registers -- the same arithmetic as
// the decode path, so no bf16 rounding of q*s ever enters the sum.  NVFP4
// tiles hold e2m1 * e4m3 (exact in bf16); CB4 uses two tiles, the bf16 high
// part of each centroid and the bf16 remainder (two MMAs per K step).  The
// epilogue applies the CB4 row norm / NVFP4 tensor scale and the bias, rounds
// to bf16 and stores Y.  When the tiles would fill at most half of the SMs,
// the K range is split over a thread-block cluster (1, 1, S) and the fp32
// partial tiles are summed through distributed shared memory before the
// epilogue; otherwise the CTAs are persistent (at most one per SM, each
// looping over tiles with its pipelines running on from one tile to the
// next).  Registers are rebalanced per warpgroup with
// setmaxnreg (56 / 104 / 168 / 168 of the 128 per thread launched).  Every
// mbarrier wait has an iteration limit; a wait that runs out records an error
// word and the CTA winds down.
//
// Sources: Petit README "Techniques and performance" (compute-bound at larger
// batch; offline-shuffled weights make GPU dequantization cheap); OrbitQuant
// card "Benchmark" (larger batches are GEMM-bound, the packed path decodes
// weights on the fly instead of materializing a dense copy); auto-round-lib
// README section 1 (per-group scales along K).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>
#include <stdlib.h>

#include "wq_frag.cuh"
#include "wq_internal.cuh"

namespace wq {

__device__ unsigned int g_wq_device_error;

namespace {

constexpr int kThreads = 512;  // 4 warpgroups: TMA+MMA, dequant, 2x fold/epilogue
#ifdef WQ_FAULT_TEST
// test build only: short waits, and one skipped arrival (see fault_stage)
constexpr uint32_t kWaitLimit = 1u << 16;
#else
constexpr uint32_t kWaitLimit = 1u << 22;
#endif

struct PrefillParams {
  const void* scales;
  const void* aux;
  const uint16_t* bias;
  uint16_t* out;
  int M, N, K, G;
  int BN, stages;
  int splits;  // K split over a cluster of this many CTAs (1: no cluster)
  uint32_t tmem_cols;
#ifdef WQ_FAULT_TEST
  // test build only: the first dequant warp does not arrive on the A-tile
  // barrier of this K step (-1: never), so the MMA issuer's bounded wait
  // runs out; no copy is skipped or altered
  int fault_stage;
#endif
  // grouped (mixture-of-experts) launch: device row offsets [E + 1] of the
  // experts (rows of x sorted by expert), T rows in x; the experts' packed
  // weights are stacked (expert e's row tiles follow expert e - 1's) and
  // their scales / aux / bias lie `*_stride` bytes apart.  NULL: one linear.
  const int64_t* offsets;
  int E, T;
  int64_t scale_stride, aux_stride;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: false when the CTA is aborting or the limit ran out (which
// raises the abort flag and the device error word).  Waits for this CTA's
// own copies or MMAs in flight (teardown, drain) pass honor_abort = false:
// they always complete, and the CTA must not release its shared or tensor
// memory before they do.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                          unsigned code, bool honor_abort = true) {
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    if (mbar_try(bar, parity)) return true;
    if (honor_abort && (i & 255u) == 255u && *abort) return false;
  }
  *abort = 1;
  atomicOr(&g_wq_device_error, code);
  return false;
}

// 8- and 16-byte cp.async into shared memory; completion is reported to an
// mbarrier by cp_async_arrive (one expected arrival per calling thread).
__device__ __forceinline__ void cp_async8(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_arrive(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(map), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

// Cluster-wide barrier (every thread of every CTA in the cluster), and the
// distributed-shared-memory address of `addr` in cluster CTA `rank`.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
__device__ __forceinline__ uint32_t dsmem_addr(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b),
               "f"(c), "f"(d)
               : "memory");
}

// UMMA shared-memory descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (stride byte offset), descriptor version 1.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;              // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024u >> 4) << 32;    // stride byte offset
  d |= (uint64_t)1u << 46;              // version
  d |= (uint64_t)2u << 61;              // SWIZZLE_128B
  return d;
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
// the four K = 16 steps of one 64-K stage (descriptor start addresses +32
// bytes per step); the first accumulates into D unless `accumulate` is 0
__device__ __forceinline__ void umma_f16_x4(uint32_t tmem_d, uint64_t a, uint64_t b,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %9, 0;\n\t"
      "setp.eq.b32 q, %9, %9;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %8, p;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %4, %8, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %5, %6, %8, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %7, %10, %8, q;\n\t}" ::"r"(tmem_d),
      "l"(a), "l"(b), "l"(a + 2), "l"(b + 2), "l"(a + 4), "l"(b + 4), "l"(a + 6), "r"(idesc),
      "r"(accumulate), "l"(b + 6)
      : "memory");
}
__device__ __forceinline__ void umma_i8(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
// an accumulator word read from tensor memory: fp32, or (i8 MMAs) s32,
// exact in fp32 for the group sums (|sum| <= 256 * 127 * 127 < 2^24)
template <bool kS32>
__device__ __forceinline__ float tmem_val(uint32_t v) {
  if constexpr (kS32) return (float)(int)v;
  return __uint_as_float(v);
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 32 consecutive columns: two x16 loads, one wait
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];"
      : "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]),
        "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]),
        "=r"(v[30]), "=r"(v[31])
      : "r"(taddr + 16u));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// byte offset of 16-byte chunk j (K elements 8j..8j+7) of row R in a
// 128-row x 64-K bf16 tile, 128-byte swizzle, 8-row groups of 1024 bytes
__device__ __forceinline__ uint32_t swz(int R, int j) {
  return (uint32_t)((R >> 3) * 1024 + (R & 7) * 128 + ((j ^ (R & 7)) << 4));
}

__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t lds_u8(uint32_t addr) {
  unsigned short v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}

// Four offset-binary INT4 codes (v + 8) in nibbles 0, 2, 4, 6 of w (the
// K order e = 0, 2, 1, 3 of the magic nibble order) -> the four int8 values
// v in K order: the byte permute restores the order, the XOR makes each
// nibble the 4-bit two's complement of v, and the multiply copies its sign
// bit into the high nibble (0x08 * 0x1E = 0xF0 stays inside its byte).
__device__ __forceinline__ uint32_t s8_of_nibbles(uint32_t w) {
  const uint32_t t = __byte_perm(w & 0x0F0F0F0Fu, 0u, 0x3120) ^ 0x08080808u;
  return t | ((t & 0x08080808u) * 0x1Eu);
}
__device__ __forceinline__ void st_shared_v2(uint32_t addr, uint32_t a, uint32_t b) {
  asm volatile("st.shared.v2.b32 [%0], {%1,%2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

template <int FMT, int BN, bool A8>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                   const PrefillParams p) {
  // one scale per group of K, folded into fp32 sums (INT formats, FP8)
  constexpr bool kInt = FMT == INT4_SYM || FMT == INT4_ASYM || FMT == INT8_SYM ||
                        FMT == INT2_SYM || FMT == INT3_SYM || FMT == FP8_E4M3 ||
                        FMT == FP8_E5M2;
  constexpr bool kFp8 = FMT == FP8_E4M3 || FMT == FP8_E5M2;
  constexpr bool kByte = FMT == INT8_SYM || kFp8;  // one byte per code
  // A8: INT8 activations x INT8 weight codes (kind::i8, s32 accumulators);
  // a stage covers 128 K (128 bytes of each operand row), else 64 K of bf16
  constexpr int KS = A8 ? 128 : 64;
  static_assert(!A8 || FMT == INT8_SYM || FMT == INT4_SYM,
                "the i8 path takes INT8 or INT4 weight codes");
  // packed bytes per stage (8 row tiles x KS)
  constexpr uint32_t kWpk =
      (kByte ? 8192u : FMT == INT2_SYM ? 2048u : FMT == INT3_SYM ? 3072u : 4096u) *
      (A8 ? 2u : 1u);
  // elements of the packed tensor map's inner dimension per row tile and stage
  constexpr int kWbox = (int)(kWpk / 8u / (kWpk / 8u > 1024u ? 8u : 4u));
  // A stage: one 128 x 64 bf16 tile; CB4 adds a second tile holding the
  // bf16 remainders of its centroids (two MMAs per K step)
  constexpr uint32_t kAsub = FMT == CB4 ? 2u : 1u;
  constexpr uint32_t kAtile = 16384u * kAsub;
  constexpr uint32_t kXbytes = (uint32_t)BN * 128u;
  constexpr uint32_t kTstage = kXbytes + kWpk;  // one TMA stage: X tile + packed tile
  // per-stage side data (same ring index): NVFP4 block scales of the 8 row
  // tiles (8 x 64 bytes), ASYM zero-points (8 x up to two 8-byte groups)
  constexpr uint32_t kSide = FMT == NVFP4 ? 512u : FMT == MXFP4 ? 256u : FMT == INT4_ASYM ? 128u : 0u;
  constexpr bool kHasSide = kSide != 0;
  constexpr int kHalf = BN / 2;  // accumulator columns per fold thread

  // One ring of ST slots, each a TMA stage (X tile, packed tile), an A tile
  // and the side data.  A slot is released by the commit of its MMAs: the
  // dequant warps have read its packed tile before they signalled its A tile.
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  // ring of ST slots: TMA stage (X tile + packed tile), A tile, side data
  const int ST = p.stages;
  uint8_t* aring = smem + ST * kTstage;
  uint8_t* sring = aring + ST * kAtile;  // side data, kSide bytes per slot
  uint64_t* bars = (uint64_t*)(sring + ST * kSide);
  uint32_t* tmem_slot = (uint32_t*)(bars + 3 * ST + 5);
  volatile int* abort = (volatile int*)(tmem_slot + 1);
  auto tfull_bar = [&](int s) { return smem_u32(bars + s); };       // TMA data landed
  auto empty_bar = [&](int s) { return smem_u32(bars + ST + s); };  // slot's MMAs done
  auto afull_bar = [&](int s) { return smem_u32(bars + 2 * ST + s); };  // A tile written
  auto gfull_bar = [&](int b) { return smem_u32(bars + 3 * ST + b); };
  auto gempty_bar = [&](int b) { return smem_u32(bars + 3 * ST + 2 + b); };
  const uint32_t drain_bar = smem_u32(bars + 3 * ST + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Tile order.  One linear: the token tile varies fastest, so the CTAs
  // resident at once share a few column blocks of the weight (each read by up
  // to M / BN CTAs close in time) and the activation tiles stay in L2.
  // Grouped: the column block varies fastest within a schedule tile.
  const int mtiles = (p.M + BN - 1) / BN;
  const int ncolb = (p.N + 127) / 128;  // column blocks of 128 rows (8 row tiles)
  // K split: the S CTAs of a cluster (1, 1, S) share a tile and take
  // consecutive ranges of KT K steps each (whole scale groups); their fp32
  // partial tiles are summed through distributed shared memory at the end
  const int S = p.splits;
  const int split = S > 1 ? (int)blockIdx.z : 0;
  const int KT = p.K / KS / S;
  const int kt0 = split * KT;  // first K step of this CTA
  const int ntiles = p.N / 16;
  // group-scale fold: exact integer tiles, one accumulator per group of K;
  // groups are counted in MMA steps of KS / 4 (16 for bf16, 32 for i8)
  const int KPG = kInt ? p.G / (KS / 4) : 4 * KT;  // MMA steps per accumulation group
  const int NG = 4 * KT / KPG;

  // Device-side tile schedule of a grouped launch: experts in order, each
  // with ceil(count / BN) token tiles.  Offsets outside [0, T] or decreasing
  // make an expert empty and set bit 256 of the error word.  `lookup` finds
  // schedule tile y (a warp-collective scan over the experts; false past the
  // end); with y < 0 it returns the number of schedule tiles in `mm0_`.
  int* sched = (int*)(bars + 3 * ST + 6);  // 16 bytes before the scale table
  auto lookup = [&](int y, int& e_, int& r0_, int& mm0_, int& rws_) -> bool {
    int base = 0, found = 0;
    for (int c0 = 0; c0 < p.E && !found; c0 += 32) {
      const int ee = c0 + lane;
      int cnt = 0, a = 0;
      if (ee < p.E) {
        const int64_t a64 = __ldg(p.offsets + ee), b64 = __ldg(p.offsets + ee + 1);
        if (a64 >= 0 && a64 <= b64 && b64 <= p.T) {
          a = (int)a64;
          cnt = (int)(b64 - a64);
        } else if (blockIdx.x == 0 && blockIdx.y == 0) {
          atomicOr(&g_wq_device_error, 256u);
        }
      }
      const int nt = (cnt + BN - 1) / BN;
      int incl = nt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (y >= 0) {
        const bool mine = nt > 0 && y >= base + incl - nt && y < base + incl;
        const unsigned bal = __ballot_sync(0xffffffffu, mine);
        if (bal) {
          const int src = __ffs(bal) - 1;
          e_ = __shfl_sync(0xffffffffu, ee, src);
          r0_ = __shfl_sync(0xffffffffu, a, src);
          mm0_ = (y - (base + __shfl_sync(0xffffffffu, incl - nt, src))) * BN;
          rws_ = __shfl_sync(0xffffffffu, cnt, src);
          found = 1;
        }
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (y < 0) mm0_ = base;
    return found != 0;
  };
  // Persistent CTAs (no K split; grouped launches except CB4, whose dequant
  // tables are per expert): the grid holds at most one CTA per SM and CTA b
  // takes tiles b, b + gridDim.x, ... (one linear: token tile fastest within
  // a column block; grouped: column block fastest within a schedule tile).
  // The ring, the K-step count and the group count run on across a CTA's
  // tiles, so the next tile's loads start while the MMAs of the current one
  // drain, and its fold and stores overlap the next tile's main loop.
  // Otherwise one tile per CTA, from the grid coordinates.
  const bool persist = S == 1 && !(p.offsets && FMT == CB4);
  int ytot = mtiles;  // token tiles per column block
  int tile0 = 0, m0 = 0, row0 = 0, rows = p.M, expert = 0;
  if (p.offsets) {
    if (warp == 0) {
      int e_ = 0, r0_ = 0, mm0_ = 0, rws_ = 0;
      const bool f = lookup(persist ? -1 : (int)blockIdx.y, e_, r0_, mm0_, rws_);
      if (lane == 0) {
        sched[0] = persist ? mm0_ : (f ? e_ : -1);
        sched[1] = r0_;
        sched[2] = mm0_;
        sched[3] = rws_;
      }
    }
    __syncthreads();
    if (persist) {
      ytot = sched[0];
    } else {
      if (sched[0] < 0) return;  // past the end of the schedule: nothing to do
      tile0 = (int)blockIdx.x * 8;
      expert = sched[0];
      row0 = sched[1];
      m0 = sched[2];
      rows = sched[3];
    }
  } else if (!persist) {
    tile0 = ((int)blockIdx.x / mtiles) * 8;
    m0 = ((int)blockIdx.x % mtiles) * BN;
  }
  const int tiles_total = ncolb * ytot;
  const int my_tiles =
      persist ? ((int)blockIdx.x < tiles_total
                     ? (tiles_total - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x
                     : 0)
              : 1;
  if (my_tiles == 0) return;  // (grouped) more CTAs than tiles: nothing to do
  // Tile i of this CTA: first row tile, token offset, expert, x / out row base
  // and expert rows.  Warp-collective for a persistent grouped launch.
  struct Tile {
    int t0, mm0, e, r0, rws;
  };
  auto tile_at = [&](int i) -> Tile {
    Tile u{tile0, m0, expert, row0, rows};
    if (persist) {
      const int t = (int)blockIdx.x + i * (int)gridDim.x;
      if (p.offsets) {
        u.t0 = (t % ncolb) * 8;
        lookup(t / ncolb, u.e, u.r0, u.mm0, u.rws);
      } else {
        u.t0 = (t / mtiles) * 8;
        u.mm0 = (t % mtiles) * BN;
      }
    }
    return u;
  };
  // the first tile's expert (the dequant warps' CB4 centroids: CB4 grouped
  // launches keep one tile per CTA)
  const uint8_t* aux_p = (const uint8_t*)p.aux + (int64_t)expert * p.aux_stride;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(tfull_bar(s), kHasSide ? 1 + 32 : 1);  // + one cp.async arrival per lane
      mbar_init(empty_bar(s), 1);                       // the MMA issuer's commit
      mbar_init(afull_bar(s), 4);                       // the four dequant warps
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(gfull_bar(b), 1);
      mbar_init(gempty_bar(b), 8);
    }
    mbar_init(drain_bar, 1);
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(p.tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 56;\n" ::: "memory");
    if (warp == 0) {
      // ---------------------------------------------------------- producer
      const int64_t groups = kInt ? p.K / p.G : 0;
      int issued = 0;
      bool run = true;
      for (int i = 0; i < my_tiles && run; ++i) {
        const Tile u = tile_at(i);
        // this tile's expert: its block scales (NVFP4 / MXFP4) or zero-points
        const uint8_t* scales_t = (const uint8_t*)p.scales + (int64_t)u.e * p.scale_stride;
        const uint8_t* aux_t = (const uint8_t*)p.aux + (int64_t)u.e * p.aux_stride;
        for (int kt = 0; kt < KT; ++kt) {
          const int s = issued % ST;
          const uint32_t ph = (uint32_t)(issued / ST) & 1u;
          if (issued >= ST && !mbar_wait(empty_bar(s), ph ^ 1u, abort, 1u)) {
            run = false;
            break;
          }
          if (lane == 0) {
            uint8_t* st = smem + s * kTstage;
            mbar_expect_tx(tfull_bar(s), kXbytes + kWpk);
            tma_load_2d(smem_u32(st), &tmX, (kt0 + kt) * KS, u.r0 + u.mm0, tfull_bar(s));
            tma_load_2d(smem_u32(st + kXbytes), &tmW, (kt0 + kt) * kWbox, u.e * ntiles + u.t0,
                        tfull_bar(s));
          }
          if constexpr (kHasSide) {
            const uint32_t sd = smem_u32(sring + s * kSide);
            const int rt = lane >> 2, c = lane & 3;  // row tile, 16-byte quarter
            const int64_t tile = u.t0 + rt;
            if (tile < ntiles) {
              if constexpr (FMT == NVFP4) {
                // 4 blocks of 16 K x 16 rows = 64 bytes per row tile
                cp_async16(sd + rt * 64 + c * 16,
                           scales_t + (tile * (p.K >> 4) + (kt0 + kt) * 4 + c) * 16);
              } else if constexpr (FMT == MXFP4) {
                // 2 blocks of 32 K x 16 rows = 32 bytes per row tile
                if (c < 2)
                  cp_async16(sd + rt * 32 + c * 16,
                             scales_t + (tile * (p.K >> 5) + (kt0 + kt) * 2 + c) * 16);
              } else {
                // the (one or two) groups of this K step: 8 bytes each
                const int64_t g0 = ((int64_t)(kt0 + kt) * 64) / p.G;
                const int ng = p.G == 32 ? 2 : 1;
                if (c < ng)
                  cp_async8(sd + rt * 16 + c * 8, aux_t + (tile * groups + g0 + c) * 8);
              }
            }
            cp_async_arrive(tfull_bar(s));
          }
          ++issued;
        }
      }
      // before teardown, make sure no copy into this CTA's memory is in flight
      for (int kt = issued - ST < 0 ? 0 : issued - ST; kt < issued; ++kt)
        mbar_wait(tfull_bar(kt % ST), (uint32_t)(kt / ST) & 1u, abort, 2u, false);
    } else if (warp == 1 && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      // instruction descriptor: D f32 (A8: s32), A and B bf16 (A8: signed
      // 8-bit), both K-major, N = BN, M = 128
      const uint32_t idesc = ((A8 ? 2u : 1u) << 4) | (1u << 7) | (1u << 10) |
                             ((uint32_t)(BN >> 3) << 17) | ((128u >> 4) << 24);
      // descriptors of slot 0 (X tile, A tile); a slot / K step is a plain
      // add to the start-address field (smem addresses stay below 2^18)
      const uint64_t xdesc0 = umma_desc_sw128(smem_u32(smem));
      const uint64_t adesc0 = umma_desc_sw128(smem_u32(aring));
      bool ok = true;
      int s = 0, g = 0, in_g = 0, gb = 0;
      uint32_t ph = 0, d = tmem;
      for (int kt = 0; kt < my_tiles * KT && ok; ++kt) {
        // the dequant warps arrive on afull only after they have seen this
        // slot's tfull, so afull alone orders the X tile too
        ok = mbar_wait(afull_bar(s), ph, abort, 8u);
        if (!ok) break;
        tc_fence_after();
        const uint64_t xd = xdesc0 + (uint64_t)((uint32_t)s * (kTstage >> 4));
        const uint64_t ad = adesc0 + (uint64_t)((uint32_t)s * (kAtile >> 4));
        if constexpr (!A8 && FMT != CB4) {
          if (KPG % 4 == 0) {
            // a stage lies inside one accumulation group: its four MMAs in one
            // instruction sequence (each tcgen05.mma issue costs ~200 cycles
            // in this loop; issuing them back to back measured 2-3% faster)
            if (in_g == 0) {
              gb = g & 1;
              d = tmem + (uint32_t)(gb * BN);
              // the fold of group g-2 must have drained this buffer
              if (g >= 2 && !mbar_wait(gempty_bar(gb), (uint32_t)((g >> 1) - 1) & 1u, abort, 4u)) {
                ok = false;
                break;
              }
              tc_fence_after();
            }
            umma_f16_x4(d, ad, xd, idesc, (uint32_t)in_g);
            in_g += 4;
            if (in_g == KPG) {
              umma_commit(gfull_bar(gb));
              in_g = 0;
              ++g;
            }
            umma_commit(empty_bar(s));
            if (++s == ST) { s = 0; ph ^= 1u; }
            continue;
          }
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          if (in_g == 0) {
            gb = g & 1;
            d = tmem + (uint32_t)(gb * BN);
            // the fold of group g-2 must have drained this buffer
            if (g >= 2 && !mbar_wait(gempty_bar(gb), (uint32_t)((g >> 1) - 1) & 1u, abort, 4u)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
          if constexpr (A8)  // +32 bytes (32 K) per step
            umma_i8(d, ad + 2 * kk, xd + 2 * kk, idesc, in_g != 0);
          else  // +32 bytes (16 K) per step
            umma_f16(d, ad + 2 * kk, xd + 2 * kk, idesc, in_g != 0);
          if constexpr (FMT == CB4)  // the centroids' remainders, same X columns
            umma_f16(d, ad + (16384u >> 4) + 2 * kk, xd + 2 * kk, idesc, 1u);
          if (++in_g == KPG) {
            umma_commit(gfull_bar(gb));
            in_g = 0;
            ++g;
          }
        }
        umma_commit(empty_bar(s));
        if (++s == ST) { s = 0; ph ^= 1u; }
      }
      if (!ok) {  // wait for this thread's own MMAs before the memory goes away
        umma_commit(drain_bar);
        mbar_wait(drain_bar, 0u, abort, 16u, false);
      }
    }
  } else if (warp < 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 104;\n" ::: "memory");
    // ------------------------------------------------------------ dequant
    const int dw = warp - 4;  // 0..3
    const int g = lane >> 2, tq = lane & 3;
    // CB4: each fp32 centroid as a bf16 high part (tables H, L) plus the bf16
    // rounding of the exact remainder (H2, L2)
    uint32_t H[4] = {0, 0, 0, 0}, L[4] = {0, 0, 0, 0};
    uint32_t H2[4] = {0, 0, 0, 0}, L2[4] = {0, 0, 0, 0};
    if constexpr (FMT == CB4) {
      const float* cen = (const float*)aux_p;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float cv = __ldg(cen + j);
        const uint32_t b = f32_to_bf16_bits(cv);
        const uint32_t b2 = f32_to_bf16_bits(cv - bf16_bits_to_f32((uint16_t)b));
        H[j >> 2] |= (b >> 8) << (8 * (j & 3));
        L[j >> 2] |= (b & 0xFFu) << (8 * (j & 3));
        H2[j >> 2] |= (b2 >> 8) << (8 * (j & 3));
        L2[j >> 2] |= (b2 & 0xFFu) << (8 * (j & 3));
      }
    }
    // NVFP4: E4M3 code -> bf16x2 pair (e4m3 * 2^119), the factor frag_nvfp4
    // expects, as a 256-entry table shared by the four dequant warps
    const uint32_t sctab = smem_u32(bars + 3 * ST + 8);
    if constexpr (FMT == NVFP4 || FMT == MXFP4) {
      for (int c = threadIdx.x - 128; c < 256; c += 128)
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(sctab + c * 4),
                     "r"(FMT == NVFP4 ? nvfp4_scale_pair(c) : mx_lo_pair(c))
                     : "memory");
      asm volatile("bar.sync 1, 128;" ::: "memory");
    }
    for (int kt = 0; kt < my_tiles * KT; ++kt) {
      const int s = kt % ST;
      const uint32_t ph = (uint32_t)(kt / ST) & 1u;
      // The slot's previous MMAs are complete: the TMA warp waited for them
      // (empty) before the load that completes this phase of tfull.
      if (!mbar_wait(tfull_bar(s), ph, abort, 32u)) break;
      const uint32_t abase = smem_u32(aring + s * kAtile);
      const uint8_t* wpk = smem + s * kTstage + kXbytes;
      const uint32_t sd = smem_u32(sring + s * kSide);
      // Rows of tiles past N hold zero-filled codes (TMA fill) and stale side
      // data; their accumulator rows are never stored.
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const int rt = 2 * dw + rr;
        const int Rg = rt * 16 + g, Rg8 = Rg + 8;
        if constexpr (A8 && FMT == INT4_SYM) {
          // INT4 codes sign-extended into the i8 operand tile: two 512-byte
          // blocks of 64 K per row tile; word 2c + s of a lane holds rows g
          // (even nibbles) and g + 8 (odd nibbles) at K 64 blk + 32 c + 8 tq
          // + 4 s + e, nibble 4 (e & 1) + 2 (e >> 1) + hr
#pragma unroll
          for (int blk = 0; blk < 2; ++blk) {
            const uint4 ch = *(const uint4*)(wpk + rt * 1024 + blk * 512 + lane * 16);
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const uint32_t w0 = c ? ch.z : ch.x, w1 = c ? ch.w : ch.y;
              const int j = 4 * blk + 2 * c + (tq >> 1);
              const uint32_t half = (uint32_t)(tq & 1) * 8u;
              st_shared_v2(abase + swz(Rg, j) + half, s8_of_nibbles(w0), s8_of_nibbles(w1));
              st_shared_v2(abase + swz(Rg8, j) + half, s8_of_nibbles(w0 >> 4),
                           s8_of_nibbles(w1 >> 4));
            }
          }
        } else if constexpr (A8) {
          // INT8 codes into the i8 operand tile: four 512-byte blocks of 32 K
          // per row tile; a lane's 16 bytes hold rows g and g + 8 at K
          // 32 blk + 8 tq + (0..3 | 4..7); offset-binary -> two's complement
#pragma unroll
          for (int blk = 0; blk < 4; ++blk) {
            const uint4 ch = *(const uint4*)(wpk + rt * 2048 + blk * 512 + lane * 16);
            const int j = 2 * blk + (tq >> 1);
            const uint32_t half = (uint32_t)(tq & 1) * 8u;
            st_shared_v2(abase + swz(Rg, j) + half, ch.x ^ 0x80808080u, ch.z ^ 0x80808080u);
            st_shared_v2(abase + swz(Rg8, j) + half, ch.y ^ 0x80808080u, ch.w ^ 0x80808080u);
          }
        } else if constexpr (kByte) {
          // (lanes with odd g take the two 8-K chunks in the other order, so
          // that the eight lanes of each quarter warp store to eight different
          // 16-byte bank groups of the swizzled tile)
#pragma unroll
          for (int bb = 0; bb < 2; ++bb) {
            const int blk = bb ^ (g & 1);
            const uint4 ch = *(const uint4*)(wpk + rt * 1024 + blk * 512 + lane * 16);
            // exact codes; the group scale is applied by the fold warps
            uint32_t a[4], b[4];
            if constexpr (FMT == FP8_E4M3) {
              frag_e4m3(ch.x, ch.y, a);
              frag_e4m3(ch.z, ch.w, b);
            } else if constexpr (FMT == FP8_E5M2) {
              frag_e5m2(ch.x, ch.y, a);
              frag_e5m2(ch.z, ch.w, b);
            } else {
              frag_int8(ch.x, ch.y, a);
              frag_int8(ch.z, ch.w, b);
            }
            const int j = 4 * blk + tq;
            st_shared_v4(abase + swz(Rg, j), a[0], a[2], b[0], b[2]);
            st_shared_v4(abase + swz(Rg8, j), a[1], a[3], b[1], b[3]);
          }
        } else if constexpr (FMT == INT3_SYM) {
          // 384 bytes per row tile and K step: the INT2-ordered low plane
          // (8 bytes per lane) and the high plane (4 bytes per lane)
          const uint2 lo = *(const uint2*)(wpk + rt * 384 + lane * 8);
          const uint32_t hi = *(const uint32_t*)(wpk + rt * 384 + 256 + lane * 4);
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int c = cc ^ (g & 1);  // chunk order by lane, as above
            const uint32_t w = c ? lo.y : lo.x;
            uint32_t a[4], b[4];
            frag_int3(w, hi, c, 0, 0x43044304u, a);
            frag_int3(w, hi, c, 1, 0x43044304u, b);
            const int j = 4 * c + tq;
            st_shared_v4(abase + swz(Rg, j), a[0], a[2], b[0], b[2]);
            st_shared_v4(abase + swz(Rg8, j), a[1], a[3], b[1], b[3]);
          }
        } else if constexpr (FMT == INT2_SYM) {
          // 256 bytes per row tile and K step; word c = the 32-K chunk c,
          // both tensor-core steps of it; exact codes, scale in the fold
          const uint2 ch = *(const uint2*)(wpk + rt * 256 + lane * 8);
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int c = cc ^ (g & 1);  // chunk order by lane, as above
            const uint32_t w = c ? ch.y : ch.x;
            uint32_t a[4], b[4];
            frag_int2(w, 0, 0x43024302u, a);
            frag_int2(w, 1, 0x43024302u, b);
            const int j = 4 * c + tq;
            st_shared_v4(abase + swz(Rg, j), a[0], a[2], b[0], b[2]);
            st_shared_v4(abase + swz(Rg8, j), a[1], a[3], b[1], b[3]);
          }
        } else {
          const uint4 ch = *(const uint4*)(wpk + rt * 512 + lane * 16);
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int c = cc ^ (g & 1);  // chunk order by lane, as above
            const uint32_t w0 = c ? ch.z : ch.x, w1 = c ? ch.w : ch.y;
            uint32_t a[4], b[4];
            if constexpr (kInt) {
              // exact code (minus zero-point); the fold warps apply the scale
              uint32_t off_g = 0x43084308u, off_g8 = 0x43084308u;
              if constexpr (FMT == INT4_ASYM) {
                const int dg = p.G == 32 ? c : 0;  // group of this half within the step
                const uint32_t zb = lds_u8(sd + rt * 16 + dg * 8 + g);
                off_g = (0x4300u + (zb & 15u)) * 0x00010001u;
                off_g8 = (0x4300u + (zb >> 4)) * 0x00010001u;
              }
              frag_int4(w0, off_g, off_g8, a);
              frag_int4(w1, off_g, off_g8, b);
            } else if constexpr (FMT == NVFP4) {
              // block of 16 K for this lane: 2c + (tq >> 1); rows g, g + 8
              const uint32_t sb = lds_u16(sd + rt * 64 + (2 * c + (tq >> 1)) * 16 + 2 * g);
              const uint32_t sc_g = lds_u32(sctab + (sb & 0xFFu) * 4);
              const uint32_t sc_g8 = lds_u32(sctab + (sb >> 8) * 4);
              frag_nvfp4(w0, sc_g, sc_g8, a);
              frag_nvfp4(w1, sc_g, sc_g8, b);
            } else if constexpr (FMT == MXFP4) {
              // one E8M0 block of 32 K per half step; rows g, g + 8
              const uint32_t sb = lds_u16(sd + rt * 32 + c * 16 + 2 * g);
              const uint32_t eg = sb & 0xFFu, eg8 = sb >> 8;
              frag_nvfp4(w0, lds_u32(sctab + eg * 4), lds_u32(sctab + eg8 * 4), a);
              frag_nvfp4(w1, lds_u32(sctab + eg * 4), lds_u32(sctab + eg8 * 4), b);
              if (eg > 128u && eg != 255u) {
                const uint32_t h = mx_hi_pair(eg);
                a[0] = bmul2(a[0], h); a[2] = bmul2(a[2], h);
                b[0] = bmul2(b[0], h); b[2] = bmul2(b[2], h);
              }
              if (eg8 > 128u && eg8 != 255u) {
                const uint32_t h = mx_hi_pair(eg8);
                a[1] = bmul2(a[1], h); a[3] = bmul2(a[3], h);
                b[1] = bmul2(b[1], h); b[3] = bmul2(b[3], h);
              }
            } else {
              frag_table<false>(w0, H, L, a);
              frag_table<false>(w1, H, L, b);
              uint32_t a2[4], b2[4];  // remainder tile, 16 KB after the high tile
              frag_table<false>(w0, H2, L2, a2);
              frag_table<false>(w1, H2, L2, b2);
              const int j2 = 4 * c + tq;
              st_shared_v4(abase + 16384u + swz(Rg, j2), a2[0], a2[2], b2[0], b2[2]);
              st_shared_v4(abase + 16384u + swz(Rg8, j2), a2[1], a2[3], b2[1], b2[3]);
            }
            const int j = 4 * c + tq;
            st_shared_v4(abase + swz(Rg, j), a[0], a[2], b[0], b[2]);
            st_shared_v4(abase + swz(Rg8, j), a[1], a[3], b[1], b[3]);
          }
        }
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
#ifdef WQ_FAULT_TEST
        if (!(dw == 0 && kt == p.fault_stage))
#endif
          mbar_arrive(afull_bar(s));  // A tile written (the packed tile is read)
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 168;\n" ::: "memory");
    // ------------------------------------------------------------ fold + epilogue
    const int q = warp & 3;            // tensor-memory lane quarter this warp may read
    const int frow = q * 32 + lane;    // accumulator row
    const int hcol = ((warp - 8) >> 2) * kHalf;
    const int64_t groups = kInt ? p.K / p.G : 0;
    const int gfirst = kInt ? (kt0 * KS) / p.G : 0;  // first group of this CTA's K range
    // A8: the per-token activation scale multiplies each output column
    auto colscale = [&](int m) -> float {
      if constexpr (A8) return __ldg((const float*)p.aux + m);
      return 1.f;
    };
    bool ok = true;
    for (int i = 0; i < my_tiles && ok; ++i) {
      const Tile u = tile_at(i);
      const int mm0 = u.mm0, row0 = u.r0, rows = u.rws;
      const int64_t n = (int64_t)u.t0 * 16 + frow;
      // this tile's expert (or the only) scales, aux and bias
      const uint8_t* scales_p = (const uint8_t*)p.scales + (int64_t)u.e * p.scale_stride;
      const uint8_t* aux_t = (const uint8_t*)p.aux + (int64_t)u.e * p.aux_stride;
      const uint16_t* bias_p = p.bias ? p.bias + (int64_t)u.e * p.N : nullptr;
      // group scales: bf16 (INT formats) or fp32 (FP8), same packed indexing
      const uint16_t* srow = (const uint16_t*)scales_p;
      const uint32_t* srow32 = (const uint32_t*)scales_p;
      const bool nvalid = n < p.N;
      // per-row factors, requested before the first wait: the group scales of
      // the next two groups ride in registers ahead of the group being folded
      int64_t sidx = 0;
      if (kInt && nvalid) {
        const int r16 = (int)(n & 15);
        sidx = (n >> 4) * groups * 16 + 2 * (r16 & 7) + (r16 >> 3);
      }
      auto group_scale = [&](int gi) -> uint32_t {
        if (!(kInt && nvalid && gi < NG)) return 0u;
        if constexpr (kFp8) return __ldg(srow32 + sidx + (int64_t)(gfirst + gi) * 16);
        return (uint32_t)__ldg(srow + sidx + (int64_t)(gfirst + gi) * 16);
      };
      uint32_t sc0 = group_scale(0), sc1 = group_scale(1);
      float post = 1.f, bval = 0.f;
      if (nvalid) {
        if constexpr (FMT == CB4) post = bf16_bits_to_f32(__ldg((const uint16_t*)scales_p + n));
        if constexpr (FMT == NVFP4) post = __ldg((const float*)aux_t) * 128.f;  // 2^7 of frag_nvfp4
        if (bias_p) bval = bf16_bits_to_f32(__ldg(bias_p + n));
      }
      float acc[kHalf];
#pragma unroll
      for (int j = 0; j < kHalf; ++j) acc[j] = 0.f;
      for (int g = 0; g < NG; ++g) {
        const int gg = i * NG + g, gb = gg & 1;  // group count across this CTA's tiles
        const uint32_t sc2 = group_scale(g + 2);
        ok = mbar_wait(gfull_bar(gb), (uint32_t)(gg >> 1) & 1u, abort, 64u);
        if (!__all_sync(0xffffffffu, ok ? 1 : 0)) { ok = false; break; }
        tc_fence_after();
        const float sc = kFp8 ? __uint_as_float(sc0)
                         : kInt          ? bf16_bits_to_f32((uint16_t)sc0)
                                         : 1.f;
        sc0 = sc1;
        sc1 = sc2;
        const uint32_t base = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(gb * BN + hcol);
        if constexpr (kHalf >= 32) {
#pragma unroll
          for (int c = 0; c < kHalf; c += 32) {
            uint32_t v[32];
            tmem_ld32(base + (uint32_t)c, v);
#pragma unroll
            for (int j = 0; j < 32; ++j) acc[c + j] = fmaf(sc, tmem_val<A8>(v[j]), acc[c + j]);
          }
        } else {
          uint32_t v[16];
          tmem_ld16(base, v);
#pragma unroll
          for (int j = 0; j < 16; ++j) acc[j] = fmaf(sc, tmem_val<A8>(v[j]), acc[j]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(gempty_bar(gb));
      }
      if (S == 1) {
        if (ok && nvalid) {
#pragma unroll
          for (int j = 0; j < kHalf; ++j) {
            const int m = mm0 + hcol + j;
            if (m < rows)
              p.out[(int64_t)(row0 + m) * p.N + n] =
                  (uint16_t)f32_to_bf16_bits(acc[j] * post * colscale(m) + bval);
          }
        }
      } else {
        // Split-K reduction.  After the first cluster barrier the rings of
        // every CTA in the cluster are idle (all its roles are done); CTA r
        // owns columns [r*CW, (r+1)*CW) of the tile and receives every CTA's
        // fp32 partial of them in slot [source][row][col] of its ring memory;
        // after the second barrier it adds the slots in source order, folds
        // and stores.
        const int CW = BN / S;
        const uint32_t slots = smem_u32(smem);
        cluster_sync_all();
#pragma unroll
        for (int j = 0; j < kHalf; j += 4) {
          const int col = hcol + j;
          const int owner = col / CW;
          const uint32_t off = (uint32_t)(((split * 128 + frow) * CW + (col - owner * CW)) * 4);
          st_cluster_v4(dsmem_addr(slots + off, (uint32_t)owner), acc[j], acc[j + 1], acc[j + 2],
                        acc[j + 3]);
        }
        cluster_sync_all();
        if (ok && nvalid) {
          // this CTA's CW columns, split between the two fold warpgroups
          const int half = (warp - 8) >> 2;
          const float* sl = (const float*)smem;
          for (int c = half * (CW / 2); c < (half + 1) * (CW / 2); ++c) {
            float tot = 0.f;
            for (int src = 0; src < S; ++src) tot += sl[(src * 128 + frow) * CW + c];
            const int m = mm0 + split * CW + c;
            if (m < rows)
              p.out[(int64_t)(row0 + m) * p.N + n] =
                  (uint16_t)f32_to_bf16_bits(tot * post * colscale(m) + bval);
          }
        }
      }
    }
  }

  // the other roles take part in the two cluster barriers of the split-K
  // reduction once their own work is done
  if (S > 1 && warp < 8) {
    cluster_sync_all();
    cluster_sync_all();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(p.tmem_cols)
                 : "memory");
  }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled_v12000)f;
  });
  return fn;
}

template <int FMT, int BN, bool A8>
cudaError_t launch_bn(const LinearArgs& a) {
  constexpr int KS = A8 ? 128 : 64;  // K per stage
  constexpr uint32_t kWpk = ((FMT == INT8_SYM || FMT == FP8_E4M3 || FMT == FP8_E5M2) ? 8192u
                             : FMT == INT2_SYM                                      ? 2048u
                             : FMT == INT3_SYM                                      ? 3072u
                                                                                    : 4096u) *
                            (A8 ? 2u : 1u);
  // the packed tile of a row tile per stage as one box row of 4- or 8-byte
  // elements (at most 256 per box dimension)
  constexpr uint32_t kEsz = kWpk / 8u > 1024u ? 8u : 4u;
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  CUtensorMap tmX, tmW;
  {
    // X: bf16 [M, K], or (A8) the INT8 activation codes [M, K]; rows of
    // 128 bytes per stage in the 128-byte swizzle
    cuuint64_t dims[2] = {(cuuint64_t)a.K, (cuuint64_t)a.M};
    cuuint64_t strides[1] = {(cuuint64_t)a.K * (A8 ? 1 : 2)};
    cuuint32_t box[2] = {(cuuint32_t)KS, (cuuint32_t)BN};
    cuuint32_t es[2] = {1u, 1u};
    if (fn(&tmX, A8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
           const_cast<void*>(a.x), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const uint64_t row_bytes = (uint64_t)a.K * 2 * code_bits(FMT);  // bytes per row tile
    // all experts' row tiles, stacked, for a grouped launch
    cuuint64_t dims[2] = {(cuuint64_t)(row_bytes / kEsz),
                          (cuuint64_t)(a.N / 16) * (cuuint64_t)(a.offsets ? a.E : 1)};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {kWpk / 8u / kEsz, 8u};
    cuuint32_t es[2] = {1u, 1u};
    if (fn(&tmW, kEsz == 8u ? CU_TENSOR_MAP_DATA_TYPE_UINT64 : CU_TENSOR_MAP_DATA_TYPE_UINT32, 2,
           const_cast<void*>(a.w), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
           CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  // ring depth: as many slots (TMA stage + A tile + side data) as fit
  const uint32_t side = FMT == NVFP4 ? 512u : FMT == MXFP4 ? 256u : FMT == INT4_ASYM ? 128u : 0u;
  const uint32_t slot = (uint32_t)BN * 128u + kWpk + 16384u * (FMT == CB4 ? 2u : 1u) + side;
  const uint32_t fixed = 1024u /* alignment */ + 8u * (3 * 8 + 8) /* barriers, tensor-memory slot,
                         abort flag, grouped schedule */ + 1024u /* NVFP4 / MXFP4 scale table */;
  int ST = (int)((227u * 1024u - fixed) / slot);
  if (ST > 8) ST = 8;
  if (ST < 2) ST = 2;
  const size_t smem = (size_t)ST * slot + fixed;
  cudaError_t attr_err =
      ensure_max_dynamic_smem((const void*)prefill_kernel<FMT, BN, A8>, 227 * 1024);
  if (attr_err != cudaSuccess) return attr_err;
  PrefillParams p;
  p.scales = a.scales;
  p.aux = a.aux;
  p.bias = (const uint16_t*)a.bias;
  p.out = (uint16_t*)a.out;
  p.M = (int)a.M;
  p.N = (int)a.N;
  p.K = (int)a.K;
  p.G = a.G;
  p.BN = BN;
  p.stages = ST;
#ifdef WQ_FAULT_TEST
  p.fault_stage = getenv("WQ_FAULT_PREFILL_STAGE") ? atoi(getenv("WQ_FAULT_PREFILL_STAGE")) : -1;
#endif
  p.offsets = a.offsets;
  p.E = a.offsets ? a.E : 1;
  p.T = (int)a.M;
  p.scale_stride = a.offsets ? a.scale_stride : 0;
  p.aux_stride = a.offsets ? a.aux_stride : 0;
  // K split over a cluster of S CTAs only when the tiles fill at most half
  // of the SMs: the distributed-shared-memory reduction (every CTA sends
  // (S-1)/S of a 128 x BN fp32 tile) costs more than a partly empty last wave
  // (measured: the 24 tiles of a 3072-row layer at M = 256 run 1.4x faster
  // with S = 4; the 224 or 256 tiles of larger layers run slower with any S).
  // S is the largest power of two <= 8 with S x tiles <= SMs that splits K
  // into whole scale groups and leaves each CTA a multiple of 4 columns.
  {
    const int64_t tiles = (int64_t)((a.N + 127) / 128) * ((a.M + BN - 1) / BN);
    const int64_t KTall = a.K / KS;
    const int64_t unit = (is_grouped_fmt(FMT) && a.G > KS) ? a.G / KS : 1;
    const int64_t sms = device_sm_count();
    int best_s = 1;
    if (2 * tiles <= sms && !a.offsets) {  // no K split in a grouped launch
      for (int sp = 8; sp >= 2; sp /= 2) {
        if (tiles * sp <= sms && KTall % (sp * unit) == 0 && BN % (4 * sp) == 0 && KTall / sp >= 8) {
          best_s = sp;
          break;
        }
      }
    }
#ifdef WQ_TUNING
    if (const char* e = getenv("WQ_PREFILL_SPLITS")) {
      const int v = atoi(e);
      if (v == 1 || ((v == 2 || v == 4 || v == 8) && KTall % (v * unit) == 0 && BN % (4 * v) == 0))
        best_s = v;
    }
#endif
    p.splits = best_s;
  }
  const bool groups2 = is_grouped_fmt(FMT) && (a.K / a.G) > 1;  // two alternating accumulators
  p.tmem_cols = (uint32_t)(groups2 ? 2 * BN : (BN < 32 ? 32 : BN));
  // grouped: an upper bound on the schedule's token tiles (sum over experts
  // of ceil(count / BN) <= ceil(T / BN) + E); the CTAs past its end exit
  const int64_t ytiles = (a.M + BN - 1) / BN + (a.offsets ? a.E : 0);
  if (a.offsets && ytiles > 65535) return cudaErrorNotSupported;
  const int64_t ncol = (a.N + 127) / 128;
  if (!a.offsets && ncol * ytiles > 0x7FFFFFFFLL) return cudaErrorNotSupported;
  // no K split (and, grouped, not CB4): persistent CTAs, at most one per SM
  // (the shared-memory ring admits one CTA per SM), looping over the tiles
  // (grouped: over an upper bound of them; the kernel reads the schedule)
  const bool persist = p.splits == 1 && !(a.offsets && FMT == CB4);
  const int64_t tiles_total = ncol * ytiles;
  const int64_t sms_avail = device_sm_count();
  const int64_t ctas = (persist && tiles_total > sms_avail) ? sms_avail : tiles_total;
  dim3 grid = persist ? dim3((unsigned)ctas, 1u, 1u)
              : a.offsets ? dim3((unsigned)ncol, (unsigned)ytiles, (unsigned)p.splits)
                          : dim3((unsigned)ctas, 1u, (unsigned)p.splits);
  if (p.splits > 1) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = a.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = (unsigned)p.splits;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, prefill_kernel<FMT, BN, A8>, tmX, tmW, p);
    if (e != cudaSuccess) return e;
  } else {
    prefill_kernel<FMT, BN, A8><<<grid, kThreads, smem, a.stream>>>(tmX, tmW, p);
  }
  return cudaGetLastError();
}

template <int FMT>
cudaError_t launch_fmt(const LinearArgs& a, int BN) {
  switch (BN) {
    case 32: return launch_bn<FMT, 32, false>(a);
    case 64: return launch_bn<FMT, 64, false>(a);
    case 128: return launch_bn<FMT, 128, false>(a);
    default: return launch_bn<FMT, 256, false>(a);
  }
}

}  // namespace

cudaError_t launch_prefill(const LinearArgs& a) {
  int BN = a.M <= 32 ? 32 : a.M <= 64 ? 64 : a.M <= 128 ? 128 : 256;
#ifdef WQ_TUNING
  if (const char* e = getenv("WQ_PREFILL_BN")) {
    const int v = atoi(e);
    if (v == 32 || v == 64 || v == 128 || v == 256) BN = v;
  }
#endif
  switch (a.fmt) {
    case INT4_SYM: return launch_fmt<INT4_SYM>(a, BN);
    case INT4_ASYM: return launch_fmt<INT4_ASYM>(a, BN);
    case INT8_SYM: return launch_fmt<INT8_SYM>(a, BN);
    case CB4: return launch_fmt<CB4>(a, BN);
    case NVFP4: return launch_fmt<NVFP4>(a, BN);
    case MXFP4: return launch_fmt<MXFP4>(a, BN);
    case FP8_E4M3: return launch_fmt<FP8_E4M3>(a, BN);
    case FP8_E5M2: return launch_fmt<FP8_E5M2>(a, BN);
    case INT2_SYM: return launch_fmt<INT2_SYM>(a, BN);
    case INT3_SYM: return launch_fmt<INT3_SYM>(a, BN);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_prefill_grouped(const LinearArgs& a) {
  // token tile from the mean rows per expert (the counts are on the device)
  const int64_t avg = (a.M + a.E - 1) / (a.E > 0 ? a.E : 1);
  const int BN = avg <= 32 ? 32 : avg <= 64 ? 64 : avg <= 128 ? 128 : 256;
  switch (a.fmt) {
    case INT4_SYM: return launch_fmt<INT4_SYM>(a, BN);
    case INT4_ASYM: return launch_fmt<INT4_ASYM>(a, BN);
    case INT8_SYM: return launch_fmt<INT8_SYM>(a, BN);
    case CB4: return launch_fmt<CB4>(a, BN);
    case NVFP4: return launch_fmt<NVFP4>(a, BN);
    case MXFP4: return launch_fmt<MXFP4>(a, BN);
    case FP8_E4M3: return launch_fmt<FP8_E4M3>(a, BN);
    case FP8_E5M2: return launch_fmt<FP8_E5M2>(a, BN);
    case INT2_SYM: return launch_fmt<INT2_SYM>(a, BN);
    case INT3_SYM: return launch_fmt<INT3_SYM>(a, BN);
  }
  return cudaErrorInvalidValue;
}

template <int FMT>
cudaError_t launch_a8_fmt(const LinearArgs& a, int BN) {
  switch (BN) {
    case 32: return launch_bn<FMT, 32, true>(a);
    case 64: return launch_bn<FMT, 64, true>(a);
    case 128: return launch_bn<FMT, 128, true>(a);
    default: return launch_bn<FMT, 256, true>(a);
  }
}

cudaError_t launch_prefill_a8(const LinearArgs& a) {
  if ((a.fmt != INT8_SYM && a.fmt != INT4_SYM) || a.K % 128) return cudaErrorNotSupported;
  const int BN = a.M <= 32 ? 32 : a.M <= 64 ? 64 : a.M <= 128 ? 128 : 256;
  return a.fmt == INT8_SYM ? launch_a8_fmt<INT8_SYM>(a, BN) : launch_a8_fmt<INT4_SYM>(a, BN);
}

cudaError_t read_device_error(unsigned* value, bool clear) {
  cudaError_t e = cudaMemcpyFromSymbol(value, g_wq_device_error, sizeof(unsigned));
  if (e != cudaSuccess || !clear) return e;
  unsigned z = 0;
  return cudaMemcpyToSymbol(g_wq_device_error, &z, sizeof(unsigned));
}

}  // namespace wq

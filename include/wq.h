/*
 * wq.h - C ABI of the B200 weight-only quantized linear.
 *
 *     Y[M,N] = X[M,K] . dequant(Wq)[N,K]^T + bias          X, Y, bias: bf16
 *
 * The weights stay packed in device memory and are expanded tile by tile
 * inside the kernels, never as a full bf16 matrix.  This is the operation of
 * the OrbitQuant packed matmul card ("API": matmul_packed_weight consumes
 * packed indices, row norms and centroids "directly, avoiding a full BF16/FP16
 * dequantized weight cache"), of the auto-round-lib README (section 1
 * "Linear": woqgemm over a repacked weight blob, activation [M,K] ->
 * output [M,N], optional bias [1,N]), of the Petit README ("Features": dense
 * FP16/BF16 x NVFP4 / MXFP4 GEMM) and of the piper-kernels README ("ConvRot INT8":
 * group-wise INT8 weight used as a normal linear weight).
 *
 * Conventions shared by every entry point
 *  - Every pointer named "device" is CUDA device memory owned by the caller;
 *    the library never allocates, frees or keeps a pointer after returning.
 *  - Every call is asynchronous on `stream` (0 = legacy default stream) unless
 *    its comment says it synchronizes.  No entry point allocates memory.
 *  - Arguments are checked on the host first; a failed check returns a status
 *    other than WQ_OK and launches nothing.  A launch failure is reported as
 *    WQ_ERR_CUDA (from cudaGetLastError).  No C++ exception crosses the ABI.
 *  - bf16 values are IEEE bfloat16 bit patterns (uint16_t).
 *  - Shapes: N % 16 == 0 and K % 64 == 0 for every format (the packed tile is
 *    16 rows by 64 (2-, 3- and 4-bit) or 32 (INT8, FP8) K elements); INT formats take
 *    group_size in {32, 64, 128, 256} with K % group_size == 0; NVFP4 has a
 *    fixed block of 16 (group_size 16 or 0), MXFP4 one of 32 (group_size 32
 *    or 0); CB4 ignores group_size; the FP8 formats take the INT group sizes.
 *  - Every device pointer must be 16-byte aligned, except the NVFP4 tensor
 *    scale and the CB4 centroids (4-byte aligned).
 *
 * Canonical (unpacked) layouts -- what wq_quantize writes and wq_pack reads.
 * Rows are output features n (the weight is [out_features, in_features] as
 * in the ConvRot INT8 section), groups run along K:
 *   WQ_INT4_SYM : codes  u8 [N, K/2]  two's complement nibbles, element 2i in
 *                                      the low nibble (the nibble order of the
 *                                      Mamba-2 paired-nibble pack helper)
 *                 scales bf16 [N, K/G]
 *   WQ_INT4_ASYM: codes  u8 [N, K/2]  unsigned nibbles 0..15, same order
 *                 scales bf16 [N, K/G];  aux = zeros u8 [N, K/G] (0..15)
 *   WQ_INT8_SYM : codes  i8 [N, K];    scales bf16 [N, K/G]
 *   WQ_CB4      : codes  u8 [N, K/2]  codebook indices, same nibble order
 *                 scales = row norms bf16 [N]; aux = centroids f32 [16]
 *   WQ_NVFP4    : codes  u8 [N, K/2]  E2M1 nibbles, same nibble order
 *                 scales = block scales u8 [N, K/16] (E4M3)
 *                 aux = tensor scale f32 [1]
 *   WQ_MXFP4    : codes  u8 [N, K/2]  E2M1 nibbles, same nibble order
 *                 scales = block scales u8 [N, K/32] (E8M0: 2^(e-127),
 *                 e = 255 is NaN); aux = NULL
 *   WQ_FP8_E4M3 : codes  u8 [N, K]    E4M3 (fn) bytes; scales f32 [N, K/G];
 *                 aux = NULL
 *   WQ_FP8_E5M2 : codes  u8 [N, K]    E5M2 bytes; scales f32 [N, K/G]; aux = NULL
 *   WQ_INT2_SYM : codes  u8 [N, K/4]  two's complement 2-bit fields, element
 *                                      4i+j at bits 2j..2j+1 of byte i
 *                 scales bf16 [N, K/G]
 *   WQ_INT3_SYM : codes  u8 [N, 3K/8] two's complement 3-bit fields, a
 *                                      little-endian bit stream per row:
 *                                      element k at bits 3k..3k+2
 *                 scales bf16 [N, K/G]
 * Dequantized value of element (n, k) -- what wq_dequant returns:
 *   INT2/INT3/INT4/INT8_SYM: q * s      ASYM: (q - z) * s          (exact fp32)
 *   CB4: fp32(c[idx] * norm[n])         NVFP4: fp32(e2m1(q) * e4m3(sb) * ts)
 *   MXFP4: fp32(e2m1(q) * 2^(e-127))    (exact; +-inf where the product
 *                                          reaches 2^128, NaN for e = 255)
 *   FP8_E4M3: fp32(e4m3(q) * s)         (one rounding; NaN for the codes
 *                                          0x7F / 0xFF, which wq_linear does
 *                                          not accept as weights: its kernels
 *                                          read them as +-480)
 *   FP8_E5M2: fp32(e5m2(q) * s)         (one rounding; +-inf / NaN for the
 *                                          exponent-31 codes, which wq_linear
 *                                          does not accept either: its kernels
 *                                          read them as finite values)
 */
#ifndef WQ_H_
#define WQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Packed weight formats (auto-round-lib "Supported Data Types"; OrbitQuant
 * card "Inputs"; Petit "Features"). */
typedef enum {
  WQ_INT4_SYM = 0,  /* symmetric INT4, bf16 scale per group                    */
  WQ_INT4_ASYM = 1, /* asymmetric INT4, bf16 scale + uint4 zero-point per group */
  WQ_INT8_SYM = 2,  /* symmetric INT8, bf16 scale per group                    */
  WQ_CB4 = 3,       /* 4-bit codebook: 16 fp32 centroids, bf16 norm per row    */
  WQ_NVFP4 = 4,     /* E2M1 values, E4M3 scale per 16, fp32 tensor scale       */
  WQ_MXFP4 = 5,     /* E2M1 values, E8M0 power-of-two scale per 32 (OCP MX)    */
  WQ_FP8_E4M3 = 6,  /* E4M3 values, fp32 scale per group (FP8 weight-only)     */
  WQ_FP8_E5M2 = 7,  /* E5M2 values, fp32 scale per group (FP8 weight-only)     */
  WQ_INT2_SYM = 8,  /* symmetric INT2, bf16 scale per group                    */
  WQ_INT3_SYM = 9   /* symmetric INT3, bf16 scale per group                    */
} wq_format_t;

typedef enum {
  WQ_OK = 0,
  WQ_ERR_INVALID_ARG = 1,  /* null pointer, bad shape, bad format, bad group   */
  WQ_ERR_UNSUPPORTED = 2,  /* valid request this build has no kernel for        */
  WQ_ERR_ALIGNMENT = 3,    /* a pointer is not aligned as required              */
  WQ_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed              */
  WQ_ERR_DEVICE_CHECK = 5  /* a kernel's own check failed (bad input found)      */
} wq_status_t;

/* Human-readable name of a status; never NULL. */
const char* wq_status_string(int status);

/* Sizes in bytes of the three canonical buffers (codes, scales, aux) and of
 * the three packed buffers of one weight; pure host arithmetic, any pointer
 * may be NULL.  Packed and canonical buffers have the same sizes except the
 * ASYM zero-points (two per byte once packed).
 * Source: auto-round-lib README section 1 (repack_quantized_weight sizes the
 * ARK blob from n, k, blocksize and the weight/scale types). */
int wq_canonical_sizes(int format, int64_t N, int64_t K, int group_size, size_t* codes_bytes,
                       size_t* scales_bytes, size_t* aux_bytes);
int wq_packed_sizes(int format, int64_t N, int64_t K, int group_size, size_t* w_bytes,
                    size_t* scales_bytes, size_t* aux_bytes);

/* Offline reorder of canonical codes, scales and aux into the packed layout
 * the kernels stream (16-row tiles whose 512-byte blocks hand every lane of a
 * warp its tensor-core fragments in one 16-byte load; nibbles interleaved for
 * two-at-a-time conversion; scales and zero-points grouped per tile).
 * Source: Petit README "Techniques and performance" (weights shuffled offline,
 * as Marlin does, to make GPU dequantization efficient); auto-round-lib
 * README section 1 (repack_quantized_weight).
 * All six buffers are device memory; canonical and packed must not overlap.
 * A pure permutation: every byte pattern is accepted and round-trips through
 * wq_unpack.  The Petit README "Known limitations" (positive scales, no
 * negative-zero FP4 codes) needs no check here, because every E4M3 / E2M1
 * bit pattern decodes by its definition.  Asynchronous; never synchronizes.
 * Ends with a 4-byte memset of a library word on `stream` (a stream operation
 * that is not a kernel), so that a wq_linear enqueued after it on the same
 * stream cannot start reading the packed buffers before they are written
 * (see wq_linear on programmatic dependent launch). */
int wq_pack(int format, int64_t N, int64_t K, int group_size, const void* codes,
            const void* scales, const void* aux, void* packed_w, void* packed_scales,
            void* packed_aux, void* stream);

/* Inverse of wq_pack: packed (device) -> canonical (device). */
int wq_unpack(int format, int64_t N, int64_t K, int group_size, const void* packed_w,
              const void* packed_scales, const void* packed_aux, void* codes, void* scales,
              void* aux, void* stream);

/* Test export: out_f32[N, K] (device, row-major) = the exact dequantized
 * weight (definitions above) read from the packed buffers.
 * Source: auto-round-lib README section 1 (unpack_weight, "decompose back to
 * full precision for verification"). */
int wq_dequant(int format, int64_t N, int64_t K, int group_size, const void* packed_w,
               const void* packed_scales, const void* packed_aux, float* out_f32, void* stream);

/* The hot path.  Y[M,N] = X[M,K] . dequant(W)[N,K]^T (+ bias[N]).
 *   x        device bf16 [M, K] row-major
 *   packed_w device, from wq_pack
 *   scales   device: INT formats packed group scales; CB4 row norms;
 *            NVFP4 packed E4M3 block scales; MXFP4 packed E8M0 block scales;
 *            FP8 packed fp32 group scales
 *   aux      device: ASYM packed zero-points; CB4 centroids f32[16];
 *            NVFP4 tensor scale f32[1]; NULL for INT2_SYM / INT4_SYM /
 *            INT8_SYM / MXFP4 / FP8
 *   bias     device bf16 [N], or NULL
 *   out      device bf16 [M, N] row-major; must not overlap any input
 * M == 0 is a no-op returning WQ_OK.  Asynchronous; no workspace.
 * Launched with programmatic dependent launch: the kernel may start while
 * the previous kernel on `stream` is finishing, requests the packed weight,
 * scales and aux at once, and reads x / writes out only after the previous
 * kernel has completed.  The packed buffers must therefore already be final
 * when the previous kernel on `stream` starts.  wq_pack, wq_quantize and
 * wq_addmm_requant end with a stream operation that is not a kernel, which
 * satisfies this on their stream; a caller that writes packed buffers with
 * its own kernels must do the same (any memset or memcpy on the stream after
 * them) or synchronize before the first wq_linear that reads them.
 * M <= 16 runs the decode kernel (register dequant, warp-level tensor-core
 * fragments, split-K over warps) unless K is too long for its staged
 * activation slice; larger M (and those) run the prefill kernel (TMA into
 * shared memory, dequant to bf16 in shared memory, tcgen05 MMA into tensor
 * memory).  Both end in the fused fold/bias/bf16 epilogue.
 * Source: OrbitQuant card "API" (matmul_packed_weight(x, idx, row_norms,
 * centroids, bits, out_features, in_features, bias)) and "Benchmark"
 * (skinny batches decode-bound, larger batches GEMM-bound); auto-round-lib
 * README section 1 (woqgemm(activation, packw, bias, n, k, groupsize, ...));
 * Petit README "Techniques and performance" (batch below 16 vs larger). */
int wq_linear(const void* x, const void* packed_w, const void* scales, const void* aux,
              const void* bias, int64_t M, int64_t N, int64_t K, int format, int group_size,
              void* out, void* stream);

/* Grouped (mixture-of-experts) linear: E experts of one format, shape [N, K]
 * and group size.  The rows of x (bf16 [T, K]) are sorted by expert: expert e
 * owns rows [offsets[e], offsets[e+1]) and writes the same rows of out
 * (bf16 [T, N]).
 *   offsets   host int64 [E + 1], offsets[0] = 0, non-decreasing, T = offsets[E]
 *   packed_w, scales, aux, bias
 *             host arrays of E device pointers (expert e's buffers as for
 *             wq_linear); aux and bias may be NULL arrays (no aux / no bias)
 * Every expert's arguments are checked before anything is launched; each
 * non-empty expert then runs wq_linear on its rows (the decode kernel for
 * at most 16 rows, the prefill kernel otherwise), in expert order on `stream`.
 * Source: Petit README "Features" (fused MoE kernels for BF16 and MXFP4
 * workloads); auto-round-lib README (quantized experts); the per-expert
 * token counts of a routed layer. */
int wq_linear_grouped(const void* x, const void* const* packed_w, const void* const* scales,
                      const void* const* aux, const void* const* bias, const int64_t* offsets,
                      int64_t E, int64_t N, int64_t K, int format, int group_size, void* out,
                      void* stream);

/* Grouped (mixture-of-experts) linear in ONE launch, with the routing on the
 * device: E experts of one format, shape [N, K] and group size, whose packed
 * buffers are stacked (expert e's packed weight at packed_w + e * w_bytes,
 * its scales at scales + e * scale_bytes, its aux at aux + e * aux_bytes,
 * the sizes from wq_packed_sizes; bias [E, N] or NULL).  The T rows of x
 * (bf16 [T, K]) are sorted by expert: expert e owns rows
 * [offsets[e], offsets[e+1]) and writes the same rows of out (bf16 [T, N]).
 *   offsets   DEVICE int64 [E + 1], read by the kernel (no host sync), so the
 *             routing counts may come straight from a device-side router;
 *             an expert whose offsets leave [0, T] or decrease is skipped and
 *             sets bit 256 of wq_device_error; rows no expert owns are not
 *             written
 * The kernel builds its tile schedule on the device: experts in order,
 * ceil(count / C) token chunks each.  With at most 16 rows per expert on
 * average (decode-like routing) the decode kernel runs it (C = 8 or 16 rows,
 * weights streamed once per chunk); otherwise the tcgen05 kernel (C = its
 * token tile BN, from the mean rows per expert).  The grid holds
 * ceil(T / C) + E chunks per column of output tiles and the chunks past the
 * schedule's end exit at once.  A bound above the grid limit (65535)
 * returns WQ_ERR_UNSUPPORTED.  Asynchronous; the offsets are read after the
 * previous kernel on `stream` has completed.
 * Source: auto-round-lib README section 2 (moe_gemm(activations, weights,
 * num_tokens_per_expert, ...): quantized experts, per-expert token counts);
 * Petit README "Features" (fused MoE kernels). */
int wq_linear_grouped_dev(const void* x, const void* packed_w, const void* scales,
                          const void* aux, const void* bias, const int64_t* offsets, int64_t E,
                          int64_t T, int64_t N, int64_t K, int format, int group_size, void* out,
                          void* stream);

/* The same linear with a SwiGLU input: x2 is bf16 [M, 2K], each row holding
 * [up | gate] (K values each), and the activation is
 *     a = bf16(up * silu(gate)),   silu(g) = g / (1 + e^-g)  (fp32, then RNE)
 * so that Y = a . dequant(W)^T (+ bias).
 *   workspace  device scratch for the materialized activation a (bf16
 *              [M, K], 16-byte aligned, at least M*K*2 bytes, overlapping no
 *              other buffer) when M > 16; may be NULL when M <= 16, where
 *              the decode kernel applies the step to its staged activation
 *              slice (except for a K too long to stage, which then needs the
 *              workspace and returns WQ_ERR_UNSUPPORTED without one).  Its
 *              contents are not preserved.
 * Everything else as wq_linear (same checks, same kernels after the step).
 * Source: piper-kernels README (convrot_linear(up_gate, weight, bias,
 * input_activation="swiglu") computes up * silu(gate) before the linear;
 * the input is [..., 2 * in_features]; other than for measured
 * configurations the page materializes the SwiGLU activation and then runs
 * the ordinary linear). */
int wq_linear_swiglu(const void* x2, const void* packed_w, const void* scales, const void* aux,
                     const void* bias, int64_t M, int64_t N, int64_t K, int format,
                     int group_size, void* workspace, size_t workspace_bytes, void* out,
                     void* stream);

/* wq_linear_swiglu without a caller workspace: for M > 16 the activation is
 * materialized in the library's static device scratch (16 MiB, a
 * file-scope __device__ array reserved when the module loads), so the call
 * allocates nothing.  M * K * 2 > 16 MiB returns WQ_ERR_UNSUPPORTED (use
 * wq_linear_swiglu with a workspace).  The scratch is one buffer per
 * device: calls of this entry point must not overlap in time on different
 * streams (calls on one stream are ordered by the stream).  M <= 16 uses
 * the scratch only for a K too long for the decode kernel's staged slice. */
int wq_linear_swiglu_static(const void* x2, const void* packed_w, const void* scales,
                            const void* aux, const void* bias, int64_t M, int64_t N, int64_t K,
                            int format, int group_size, void* out, void* stream);

/* Activation-quantized linear (W8A8): the activations are quantized per
 * token to INT8 and multiplied with the INT8 weight codes on the integer
 * tensor cores; each group's integer sum is scaled once:
 *     s_x[m] = fp32(max_k |x[m,k]| / 127)  (quotient in fp64)
 *     x_q[m,k] = clamp(round_half_even(x[m,k] / s_x[m]), -127, 127)
 *     Y[m,n] = s_x[m] * sum_g s_w[n,g] * (sum_{k in g} x_q[m,k] * q[n,k]) + bias[n]
 * This is a different computation from wq_linear (the activations are
 * quantized), with its own reference; the group sums are exact integers and
 * the scaling is fp32.
 *   x, packed_w, scales, bias, out   as wq_linear (formats WQ_INT8_SYM, and
 *                                    WQ_INT4_SYM whose codes are used as INT8:
 *                                    W4A8)
 *   workspace   device scratch of at least wq_linear_a8_workspace_size(M, K)
 *               bytes, 16-byte aligned, overlapping no other buffer: the
 *               INT8 codes [M, K] at offset 0 and the fp32 scales [M] at the
 *               next multiple of 256 bytes; contents not preserved
 * Other formats, or K % 128 != 0, return WQ_ERR_UNSUPPORTED.  M == 0 is a
 * no-op.  Asynchronous: two kernels (the quantizer, then the tcgen05 kernel
 * with tcgen05.mma.kind::i8 and s32 accumulators in tensor memory).
 * Source: auto-round-lib README section 1 ("Key Features": INT8 compute with
 * dynamic per-token activation quantization, low-bit weights used as INT8;
 * the W8A8 / W4A8 backends). */
int wq_linear_a8_workspace_size(int64_t M, int64_t K, size_t* bytes);
int wq_linear_a8(const void* x, const void* packed_w, const void* scales, const void* bias,
                 int64_t M, int64_t N, int64_t K, int format, int group_size, void* workspace,
                 size_t workspace_bytes, void* out, void* stream);

/* The per-token INT8 activation quantizer of wq_linear_a8 on its own (device
 * buffers): xq int8 [M, K] (16-byte aligned), sx f32 [M]; K % 8 == 0.
 * Source: as wq_linear_a8. */
int wq_quantize_act_int8(const void* x, int64_t M, int64_t K, void* xq, void* sx, void* stream);

/* In-place LoRA merge into a packed INT8_SYM weight:
 *     weight = beta * weight + alpha * (mat1 @ mat2)
 * requantized with the weight's unchanged group scales.  With use_seed == 0
 * each code is the nearest (ties to even) of w'/s; otherwise one of the two
 * adjacent codes, the upper one with probability equal to the fractional
 * part of w'/s (draw for element (n, k): output n*K + k of SplitMix64 keyed
 * by `seed`, top 53 bits * 2^-53), so the same seed replays the same codes.
 * Codes are clamped to [-127, 127]; a zero scale keeps code 0.  All
 * arithmetic is fp64 with round-to-nearest steps in a fixed order.
 *   packed_w       device, in/out (from wq_pack)
 *   packed_scales  device, unchanged
 *   mat1, mat2     device bf16 [N, rank] and [rank, K] (rank 0: no update)
 * Other formats return WQ_ERR_UNSUPPORTED.  Offline; asynchronous.  Repeated
 * merges are lossy (each one requantizes).  Ends, like wq_pack, with a
 * 4-byte memset of a library word on `stream`, so that a following
 * wq_linear on the same stream reads the merged codes.
 * Source: piper-kernels README (weight.addmm_(lora_b, lora_a, alpha=...,
 * rounding_seed=seed): beta * weight + alpha * (mat1 @ mat2), requantized,
 * deterministic row scales kept, stochastic choice of one of the two adjacent
 * INT8 codes with probability proportional to distance). */
int wq_addmm_requant(int format, int64_t N, int64_t K, int group_size, void* packed_w,
                     const void* packed_scales, const void* mat1, const void* mat2, int64_t rank,
                     double alpha, double beta, int use_seed, uint64_t seed, void* stream);

/* Offline round-to-nearest quantizer on the GPU: w_f32[N, K] (device) ->
 * canonical codes / scales / aux (device), bit-identical to the CPU
 * definitions listed above.  CB4 reads its 16 centroids from `aux`
 * (device f32[16], left unchanged) and writes the row norms; NVFP4 writes the
 * tensor scale into `aux` (three stream-ordered passes: tensor maximum,
 * codes, tensor scale).  Asynchronous; ends, like wq_pack, with a 4-byte memset.
 * The FP8 formats write fp32 scales amax/448 (E4M3) or amax/57344 (E5M2).
 * Source: piper-kernels README "ConvRot INT8" (ConvRotInt8Tensor.from_hp
 * quantizes a dense weight, group_size=256); Mamba-2 pack helper (scale =
 * amax/qmax, round, clamp). */
int wq_quantize(int format, int64_t N, int64_t K, int group_size, const float* w_f32,
                void* codes, void* scales, void* aux, void* stream);

/* Host: the 2^bits-level Lloyd-Max quantizer of N(0,1) (bits 1..8), as fp32,
 * ascending, written to centroids_out[2^bits] (host memory).  Fixed-point
 * iteration in fp64 from a uniform start on [-3, 3] until no level moves by
 * 1e-14.  Source: OrbitQuant card "Inputs" (fp32 Lloyd-Max centroids with
 * shape [2**bits]). */
int wq_lloyd_max_centroids(int bits, float* centroids_out);

/* The kernels' own error word on the current device.  Every wait of the
 * prefill kernel on a shared-memory barrier has an iteration limit; a wait that
 * runs out sets a bit here (1 producer, 2 producer drain, 4/8 MMA waits, 16
 * MMA drain, 32 dequant, 64 epilogue; 128 the decode kernel's wait for its
 * staged activation slice) and the thread block winds down instead of
 * hanging, leaving the CUDA context usable.  Bit 256 reports routing offsets
 * of wq_linear_grouped_dev outside [0, T] or decreasing.  Synchronizes the device (a
 * symbol copy).  Writes the word to *value, clears it when `clear` is non-zero,
 * and returns WQ_ERR_DEVICE_CHECK when it was non-zero, WQ_OK otherwise. */
int wq_device_error(unsigned* value, int clear);

/* Device properties the dispatcher uses (SM count of the current device);
 * exported for the benchmark's launch accounting.  Returns WQ_ERR_CUDA when
 * no device is usable. */
int wq_device_sm_count(int* sm_count);

#ifdef __cplusplus
}
#endif

#endif /* WQ_H_ */

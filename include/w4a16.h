/*
 * w4a16.h - C ABI of the W4A16 weight-only 4-bit matmul library for NVIDIA
 * B200 (sm_100a).
 *
 * What it computes: y[M][N] = x[M][K] . W_deq[N][K]^T, with BF16 activations
 * x, BF16 outputs y, and weights stored in one of two 4-bit checkpoint
 * formats, dequantised on the fly:
 *
 *  - W4A16_FMT_INT4_G128: symmetric GPTQ-style int4, q in [-8, 7], one BF16
 *    scale per group of 128 K-elements per output column, no zero point, no
 *    act-order (the checkpoint contract in the NVIDIA developer-forum post
 *    "Qwen3.8-27B on single DGX Spark ...", section "Quality").
 *    W_deq[n][k] = RNE_bf16(q[n][k] * s[n][k/128]).
 *  - W4A16_FMT_NVFP4_G16: FP4-E2M1 values, one FP8-E4M3 scale per 16
 *    K-elements per output column, one FP32 per-tensor scale g (the
 *    compressed-tensors nvfp4-pack-quantized format of the model card
 *    "Qwen3.8 27B - NVFP4 for veloGB10", section "Specifications"; group 16
 *    per "SuperQwen3.8-27b-abliterated-NVFP4-2xDGX", "Release highlights").
 *    W_deq[n][k] = RNE_bf16(e2m1(c[n][k]) * e4m3(s8[n][k/16]) * g).
 *
 * Row counts are those of single-token decode and speculative verification
 * (M = 1 .. 64): the full model checks several drafted tokens in one batched
 * pass (blog post "One Config Line Made My 27B Model 2.7x Faster", section
 * "The fix: use the MTP head you already downloaded").  The kernel is picked
 * by row count (forum post above, section "How").
 *
 * Conventions shared by every entry point:
 *  - Every call returns a status (W4A16_OK or a negative W4A16_ERR_*), never
 *    throws and never aborts.  Arguments are validated before any launch.
 *  - Device calls are asynchronous and ordered on the given stream (a
 *    cudaStream_t passed as void*, NULL = legacy default stream).  The library
 *    keeps no pointer after a call returns; buffers must stay alive until the
 *    stream has executed the work.
 *  - The caller owns every buffer passed in.  The GEMM keeps a
 *    library-owned workspace per (device, stream): fp32 split-K partial sums
 *    and, on the tensor-core path for NVFP4 and FP8, an FP16 copy of x.  It is
 *    allocated (stream-ordered) on the first call that needs it on that
 *    stream and grown when a larger problem needs more; make a call of the
 *    largest shape before capturing the stream into a CUDA graph.
 *  - Accuracy: per element |y - y_ref| <= 2^-7 * sum_k |W_deq[n][k] x[m][k]|
 *    + 1e-3 against the fp64 dequantise-then-matmul, and w4a16_dequant is
 *    bit-exact.  The FP16 tensor-core operands (the GEMV in every format, the
 *    tcgen05 path for NVFP4 and FP8) take each activation row (slice) scaled
 *    by a power of two into FP16: elements more than 2^29 below their row
 *    slice's largest magnitude lose low bits (absolute error at most 2^-40 of
 *    that largest magnitude per element).
 */
#ifndef W4A16_H
#define W4A16_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Weight formats. */
#define W4A16_FMT_INT4_G128 0  /* int4 GPTQ, BF16 scale per 128-group */
#define W4A16_FMT_NVFP4_G16 1  /* e2m1, E4M3 scale per 16-group, fp32 per-tensor scale */
#define W4A16_FMT_FP8_E4M3 2   /* E4M3 weights (W8A16), fp32 per-tensor scale, no packed scales */
#define W4A16_FMT_NVFP4_BS 3   /* NVFP4 weights in the block-scaled tensor-core layout (W4A4 only) */

/* Status codes. */
#define W4A16_OK 0
#define W4A16_ERR_ARG (-1)     /* bad format, null pointer, out-of-range code, bad path id */
#define W4A16_ERR_SHAPE (-2)   /* M, N or K outside the supported range */
#define W4A16_ERR_ALIGN (-3)   /* a device pointer is not 16-byte aligned */
#define W4A16_ERR_DEVICE (-4)  /* the current device is not sm_100 */
#define W4A16_ERR_CUDA (-5)    /* a CUDA runtime call or launch failed */
#define W4A16_ERR_TIMEOUT (-6) /* a kernel gave up a bounded wait (see w4a16_device_status) */
#define W4A16_ERR_NOMEM (-7)   /* the workspace could not be allocated */
#define W4A16_ERR_SCRATCH (-8) /* w4a16_gemm_noalloc: the problem needs more than its fixed scratch */

/* Limits of this version. */
#define W4A16_MAX_M 8192       /* decode, speculative verify and prefill chunks */

/* Kernel paths (for w4a16_gemm_path / w4a16_gemm_ex). */
#define W4A16_PATH_AUTO 0      /* row-count dispatch */
#define W4A16_PATH_GEMV 1      /* weight-streaming split-K GEMV (mma.sync fragments), M <= 16 */
#define W4A16_PATH_TC 2        /* tcgen05 tensor-core path (A in tensor memory), M <= 8192 */
#define W4A16_PATH_BS 3        /* W4A4 block-scaled tensor-core path (w4a16_plan queries only) */
#define W4A16_GEMV_MAX_M 16

/*
 * Shape rules: 1 <= M <= 8192; N >= 1 (any value; packed buffers are padded
 * to a multiple of 16 rows); K >= 128 and K a multiple of 128 (every format).
 * The tensor-core path splits M > 128 into ceil(M / 128) chunks of equal row
 * counts inside one launch (beyond M = 128 the tensor cores, not HBM, set the
 * time).
 */

/* Bytes of the packed weight buffer: ceil(N/16)*16 * K / 2 (4-bit formats),
 * ceil(N/16)*16 * K (FP8).  0 on bad args. */
size_t w4a16_packed_weight_bytes(int fmt, int N, int K);

/* Bytes of the packed scale buffer: INT4 ceil(N/16)*16 * K/128 * 2;
 * NVFP4 ceil(N/16)*16 * K/16; FP8 0 (one per-tensor scale, passed to the
 * matmul as global_scale).  0 on bad args. */
size_t w4a16_packed_scale_bytes(int fmt, int N, int K);

/*
 * Host-side packer: logical checkpoint tensors -> the library's packed layout.
 *   codes:  INT4: int8 q[N][K] in [-8, 7];  NVFP4: uint8 e2m1 codes c[N][K] in 0..15;
 *           FP8: uint8 E4M3 bytes w8[N][K] (0x7F/0xFF NaN patterns rejected).
 *   scales: INT4: BF16 bit patterns (uint16) s[N][K/128];
 *           NVFP4: E4M3 bytes s8[N][K/16] (0x7F/0xFF NaN patterns rejected);
 *           FP8: unused (may be NULL), as is packed_scales.
 *   packed_w / packed_scales: host buffers of the sizes above.
 * All pointers are host pointers.  Returns W4A16_ERR_ARG on an out-of-range
 * code or scale (nothing useful is left in the outputs then).
 */
int w4a16_pack_host(int fmt, int N, int K, const void* codes, const void* scales,
                    void* packed_w, void* packed_scales);

/* Inverse of w4a16_pack_host (host pointers), for round-trip checks. */
int w4a16_unpack_host(int fmt, int N, int K, const void* packed_w, const void* packed_scales,
                      void* codes, void* scales);

/*
 * Device-side packer: same layouts as w4a16_pack_host, all four pointers are
 * device pointers, asynchronous on `stream`.  Codes outside the format's range
 * are not detected (4-bit formats store only the low 4 bits; FP8 NaN bytes
 * are stored as they are).  FP8: scales and packed_scales unused (may be NULL).
 */
int w4a16_pack(int fmt, int N, int K, const void* codes, const void* scales,
               void* packed_w, void* packed_scales, void* stream);

/*
 * Dequantise to BF16, bit-exact:
 *   w_bf16[n][k] = W_deq[n][k] for n < N, k < K (row-major [N][K], device).
 * global_scale: NVFP4 and FP8: device pointer to one fp32 g; INT4: must be NULL.
 * FP8: W_deq = RNE_bf16(e4m3 * g); packed_scales unused (may be NULL).
 */
int w4a16_dequant(int fmt, int N, int K, const void* packed_w, const void* packed_scales,
                  const float* global_scale, void* w_bf16, void* stream);

/*
 * The matmul: y[M][N] = x[M][K] . W_deq[N][K]^T.
 *   x_bf16:   device, [M][K] BF16 row-major, 16-byte aligned.
 *   packed_w, packed_scales: device, produced by a packer above, 16-byte aligned
 *             (FP8: packed_scales unused, may be NULL).
 *   global_scale: NVFP4 and FP8: device pointer to one fp32 g; INT4: must be NULL.
 *   y_bf16:   device, [M][N] BF16 row-major; must not overlap any input.
 * Picks the kernel by row count (W4A16_PATH_AUTO): the split-K GEMV for
 * M <= 8, and for 9 <= M <= 16 when N >= 16384; the tensor-core path
 * otherwise.  w4a16_gemm_path() reports the choice.
 */
int w4a16_gemm(int fmt, int M, int N, int K, const void* x_bf16, const void* packed_w,
               const void* packed_scales, const float* global_scale, void* y_bf16, void* stream);

/* Same as w4a16_gemm with an explicit path (W4A16_PATH_*); W4A16_ERR_SHAPE if
 * the path does not support M. */
int w4a16_gemm_ex(int path, int fmt, int M, int N, int K, const void* x_bf16,
                  const void* packed_w, const void* packed_scales, const float* global_scale,
                  void* y_bf16, void* stream);

/*
 * The fused gate/up layer of the MLP: h[M][I] = BF16(SiLU(gate) * up) with
 *   gate = x . W_deq[0:I]^T,  up = x . W_deq[I:2I]^T,  SiLU(z) = z / (1 + e^-z),
 * gate and up kept in fp32 until the product (one kernel, or two when K is
 * split across CTAs on the tensor-core path: the reduction applies SiLU).
 * Reading of the pages' MLP linears (model card "Qwen3.8 27B - NVFP4 for
 * veloGB10", section "Specifications"): the [2I][K] weight holds the gate
 * rows first and the up rows second.
 *   packed_w, packed_scales: that [2I][K] weight packed as for w4a16_gemm
 *     with N = 2I.  I >= 16 and a multiple of 16 (else W4A16_ERR_SHAPE).
 *   x_bf16, global_scale: as for w4a16_gemm.
 *   h_bf16: device, [M][I] BF16 row-major; must not overlap any input.
 * Same row limits and dispatch as w4a16_gemm with N = 2I.
 */
int w4a16_gemm_gate_up_silu(int fmt, int M, int I, int K, const void* x_bf16,
                            const void* packed_w, const void* packed_scales,
                            const float* global_scale, void* h_bf16, void* stream);

/* Same as w4a16_gemm_gate_up_silu with an explicit path (W4A16_PATH_*). */
int w4a16_gemm_gate_up_silu_ex(int path, int fmt, int M, int I, int K, const void* x_bf16,
                               const void* packed_w, const void* packed_scales,
                               const float* global_scale, void* h_bf16, void* stream);

/*
 * The split-K GEMV (M <= W4A16_GEMV_MAX_M) for callers that cannot allocate
 * device memory: applications that reserve all device memory up front for
 * their own pool or allocator and forbid any later cudaMalloc (including the
 * one w4a16_gemm makes the first time a stream needs split-K workspace), and
 * latency-critical code that must not allocate in its steady state, because
 * an allocation can synchronise the device.  No counterpart on the source
 * pages: it is a deployment variant of w4a16_gemm.
 *   Same arguments, layouts and results as w4a16_gemm on the GEMV path.
 *   Scratch: a fixed 8 MiB array in device global memory owned by the library
 *   (every GPU that loads the library holds it until the process exits).  A
 *   call that would need more (split-K partials of large N) returns
 *   W4A16_ERR_SCRATCH without launching; M > W4A16_GEMV_MAX_M returns
 *   W4A16_ERR_SHAPE.  Calls neither allocate nor free device memory.
 *   The first call on a device resolves the array's device address and sets
 *   the launch attributes of every kernel variant this entry point uses.
 *   All calls share the array: calls whose GPU work overlaps (different
 *   streams, or threads sharing a device) race and must be serialised by the
 *   caller.  Each call clears, in stream order, the part that must start at
 *   zero.  The GEMV has no bounded waits, so these calls cannot time out.
 */
int w4a16_gemm_noalloc(int fmt, int M, int N, int K, const void* x_bf16, const void* packed_w,
                       const void* packed_scales, const float* global_scale, void* y_bf16,
                       void* stream);

/*
 * W4A4 NVFP4: the activations quantised to NVFP4 as well (model card
 * "SuperQwen3.8-27b-abliterated-NVFP4-2xDGX", table "Release highlights":
 * W4A4 NVFP4, group size 16).  The pages name only the format; the reading
 * taken, every step in fp32 with round-to-nearest:
 *   g_x = amax|x| / (6 * 448)                 (1.0 for an all-zero x)
 *   s[m][j] = RNE_e4m3(amax_{k in 16-block j}|x[m][k]| / (6 * g_x)), saturating at 448
 *   q[m][k] = RNE_e2m1(x[m][k] / (e4m3(s[m][k/16]) * g_x)), ties to the even code,
 *             saturating at +-6 (0 when the scale is 0)
 *
 * Quantiser alone: x_bf16 [M][K] (device, 16-byte aligned, K a multiple of
 * 128, 1 <= M <= 8192) -> codes (device, [M][K] bytes, one E2M1 code in the
 * low 4 bits of each, 16-byte aligned), scales (device, [M][K/16] E4M3
 * bytes), g_x (device, one fp32).  Asynchronous on `stream`.
 */
int w4a16_quantize_act_nvfp4(int M, int K, const void* x_bf16, void* codes, void* scales,
                             float* g_x, void* stream);

/*
 * The W4A4 matmul: y[M][N] = BF16(sum_k x_hat[m][k] * W[n][k]) with
 * x_hat = e2m1(q) * e4m3(s) * g_x (the quantiser above, run inside the call)
 * and W the NVFP4 weights at their exact values e2m1 * e4m3 * g_w.
 *   x_bf16, y_bf16: as for w4a16_gemm.  packed_w, packed_scales: NVFP4
 *   weights packed as for w4a16_gemm (W4A16_FMT_NVFP4_G16).  global_scale_w:
 *   device pointer to the weights' fp32 g_w.
 * Accuracy: |y - y_ref| <= 2^-7 * sum_k |x_hat W| + 1e-3 against the exact
 * W4A4 product.  The library keeps a scratch per (device, stream) for the
 * quantised activations (M x K BF16), allocated like the matmul workspace.
 */
int w4a16_gemm_w4a4(int M, int N, int K, const void* x_bf16, const void* packed_w,
                    const void* packed_scales, const float* global_scale_w, void* y_bf16,
                    void* stream);

/* Same as w4a16_gemm_w4a4 with an explicit path (W4A16_PATH_*). */
int w4a16_gemm_w4a4_ex(int path, int M, int N, int K, const void* x_bf16, const void* packed_w,
                       const void* packed_scales, const float* global_scale_w, void* y_bf16,
                       void* stream);

/*
 * W4A4 NVFP4 on the block-scaled tensor cores (tcgen05.mma kind::mxf4nvf4
 * with one E4M3 scale per 16 k on both operands): the same result contract as
 * w4a16_gemm_w4a4 (the same quantiser, run inside the call, then the exact
 * W4A4 product within the same bound), with the weights packed in the tensor
 * cores' own layout, format W4A16_FMT_NVFP4_BS (w4a16_pack / w4a16_pack_host
 * with that format; sizes from w4a16_packed_weight_bytes / _scale_bytes):
 *   packed_w: [N][K/2] bytes, byte j of row n = code(k = 2j) | code(2j + 1) << 4;
 *   packed_sf: E4M3 scales in atoms of 128 rows x 64 k (512 bytes), atom
 *     (n / 128, kb) at ((n / 128) * (K / 64) + kb) * 512, row r = n % 128 and
 *     16-block j of kb at byte 16 * (r % 32) + 4 * (r / 32) + j; rows past N
 *     of the last atom row hold 0.
 * No tensor-core instruction or thread of this path converts a weight: the
 * tensor cores read the codes from shared memory and the scales from tensor
 * memory.  1 <= M <= 8192 (chunks of at most 128 activation rows), N >= 1,
 * K a multiple of 128; every pointer a 16-byte aligned device pointer.  The
 * library keeps a scratch per (device, stream) for the quantised activations
 * (M x K/2 codes and their scale atoms) and, when K is split, fp32 partials.
 */
int w4a16_gemm_w4a4_bs(int M, int N, int K, const void* x_bf16, const void* packed_w,
                       const void* packed_sf, const float* global_scale_w, void* y_bf16,
                       void* stream);

/* The path W4A16_PATH_AUTO would take for these arguments (>0), or a status. */
int w4a16_gemm_path(int fmt, int M, int N, int K);

/*
 * Synchronises `stream`, then reads and clears the device error word that
 * kernels set when a bounded wait gives up.  Returns W4A16_OK,
 * W4A16_ERR_TIMEOUT, or W4A16_ERR_CUDA if the synchronisation itself failed.
 */
int w4a16_device_status(void* stream);

/* Human-readable name of a status code (static string). */
/*
 * Diagnostics: the launch plan the library would use, computed on the host
 * (no device call; num_sms stands for the device's SM count).  path:
 * W4A16_PATH_AUTO, _GEMV or _TC; fuse: 1 for w4a16_gemm_gate_up_silu with
 * N = 2I.  out[0..8] (out_len >= 9):
 *   GEMV: K splits, K elements per split, CTAs per split, 8-row tiles, bands
 *         in flight per CTA, K pieces per band, ring depth, groups per piece,
 *         dynamic shared memory bytes;
 *   TC:   row chunks, rows per chunk, padded rows (MMA N), K splits, 64-blocks
 *         per split, work units, CTAs, dynamic shared memory bytes, 0;
 *   BS (path W4A16_PATH_BS, fmt W4A16_FMT_NVFP4_BS, the plan of
 *         w4a16_gemm_w4a4_bs): 128-row tiles, row chunks, rows per chunk,
 *         padded rows (MMA N), K splits, 256-k stages per split, work units,
 *         CTAs, dynamic shared memory bytes.
 * Returns the path (W4A16_PATH_GEMV, _TC or _BS) or a negative status.
 */
int w4a16_plan(int path, int fmt, int M, int N, int K, int fuse, int num_sms, int* out,
               int out_len);

/*
 * Diagnostics of the kernels' failure path, without a fault: launches a tiny
 * kernel whose two warps wait, through the library's own bounded mbarrier
 * waits, on a barrier that nothing arrives at.  After the bound (about two
 * seconds of SM clock) the first warp records W4A16_ERR_TIMEOUT in the device
 * error word and raises its CTA's abort flag, the second gives up on seeing
 * the flag, and the kernel exits normally.  Synchronises `stream`, then
 * checks and clears the error word.  Returns W4A16_OK when all of that
 * happened as designed, W4A16_ERR_TIMEOUT when it did not (or when an
 * earlier timeout was still unreported), W4A16_ERR_CUDA / W4A16_ERR_NOMEM /
 * W4A16_ERR_DEVICE on failures of the call itself.
 */
int w4a16_selftest_wait_timeout(void* stream);

const char* w4a16_status_string(int status);

/* Library version: major * 10000 + minor * 100 + patch. */
int w4a16_version(void);

#ifdef __cplusplus
}
#endif

#endif /* W4A16_H */

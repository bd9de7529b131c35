/*
 * fgfp8 — fine-grained FP8 W8A8 linear layers for NVIDIA B200 (sm_100a).
 *
 * C ABI.  Plain pointers and sizes only.  Every pointer argument is a DEVICE
 * pointer on the current CUDA device, except where a comment says otherwise.
 * `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 * stream).  The caller allocates and owns every buffer.  These calls never
 * allocate device memory.
 *
 * Every call validates its arguments on the host first.  A violation returns
 * an error code, launches nothing and leaves a message for
 * fgfp8_last_error_string().  A call that passes validation enqueues its kernels
 * on `stream` and returns FGFP8_OK without waiting for them.  There is no CPU
 * fallback: on a machine without a usable sm_100a GPU every compute call
 * returns FGFP8_ERR_CUDA.
 *
 * Method (page titles and sections of the source documentation):
 *   - "Fine-grained FP8" (Transformers docs), introduction: weights are
 *     quantized to 8 bits per 128x128 block; activations per token, in groups
 *     that match the weight's 128-wide input-channel block.
 *   - "Fine-grained FP8", "DeepGEMM fast path": the dynamic activation scheme
 *     (scales computed from each group at run time).
 *   - "Fine-grained FP8", "UE8M0 scale format": scales stored either as
 *     float32 or as packed float8_e8m0fnu (a power of two 2^(e-127) in one
 *     byte).
 *   - "FP8 W8A8" (vLLM docs), "Two FP8 representations": E4M3 has one sign,
 *     four exponent and three mantissa bits, reaches +-448, and has NaN.
 * The steps the pages leave open are fixed as follows.  Each step is one
 * IEEE fp32 operation with round-to-nearest-even:
 *   amax   = max |x| over the group/block; it is raised to 1e-4 if smaller,
 *            and a NaN element makes it NaN
 *   fp32   : scale = amax / 448
 *   UE8M0  : scale = the smallest power of two >= amax / 448
 *   code   = E4M3( x / scale ), rounded to nearest even and saturated to +-448
 *   GEMM   : Y[m,n] = bf16_rne( sum_kb sa[m,kb] * sw[n/128,kb] *
 *                               sum_{k in block kb} Xq[m,k] * Wq[n,k] ).
 * The GEMM accumulates in fp32.  Its result is accurate to within
 * |Y - Y_exact| <= 2^-7 |Y_exact| + 1e-4 sum_k |x_hat w_hat|.  The
 * quantizers are bit-exact.
 */
#ifndef FGFP8_H
#define FGFP8_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FGFP8_VERSION 1

/* Scale storage ("Fine-grained FP8", "UE8M0 scale format"). */
typedef enum {
  FGFP8_SCALE_F32 = 0,   /* float32, 4 bytes per scale */
  FGFP8_SCALE_UE8M0 = 1  /* float8_e8m0fnu: one byte e, value 2^(e-127); 0xFF = NaN */
} fgfp8_scale_fmt;

typedef enum {
  FGFP8_OK = 0,
  FGFP8_ERR_INVALID_ARG = 1, /* null pointer, bad enum, negative size */
  FGFP8_ERR_SHAPE = 2,       /* K or N not a multiple of 128, ld too small, size too large */
  FGFP8_ERR_ALIGN = 3,       /* a pointer or leading dimension breaks the 16-byte rule */
  FGFP8_ERR_UNSUPPORTED = 4, /* a valid request the library does not implement */
  FGFP8_ERR_CUDA = 5,        /* a CUDA runtime or driver call failed */
  FGFP8_ERR_TIMEOUT = 6,     /* a kernel gave up on a barrier wait (device status) */
  FGFP8_ERR_DEVICE = 7       /* a kernel rejected its device-side inputs (device status) */
} fgfp8_status;

/* FGFP8_VERSION of the loaded library. */
int fgfp8_version(void);

/* Message for the last error on the calling thread ("" if none).  The string
 * is owned by the library.  It stays valid until the next call from the same
 * thread. */
const char* fgfp8_last_error_string(void);

/*
 * 128x128 block weight quantization ("Fine-grained FP8", introduction).
 *   W   bf16 [N, K], row stride ldw elements (ldw >= K, ldw % 8 == 0,
 *       16-byte aligned).
 *   Wq  E4M3 codes [N, K], row stride K bytes, 16-byte aligned.
 *   Ws  [N/128, K/128] row-major: float (fmt F32, 4-byte aligned) or UE8M0
 *       bytes.  Ws[nb*(K/128) + kb] is the scale of rows nb*128.. and columns
 *       kb*128..
 * N % 128 == 0 and K % 128 == 0.  N == 0 is a no-op.  For a stack of E expert
 * matrices, pass N = E * N_expert: blocks never straddle experts.
 */
fgfp8_status fgfp8_quant_weight(const void* W, int64_t N, int64_t K, int64_t ldw, uint8_t* Wq, void* Ws,
                                int fmt, void* stream);

/*
 * Dynamic per-token activation quantization, groups of 128 along K
 * ("Fine-grained FP8", introduction and "DeepGEMM fast path").
 *   X   bf16 [M, K], row stride ldx elements (ldx >= K, ldx % 8 == 0,
 *       16-byte aligned).
 *   Xq  E4M3 codes [M, K], row stride K bytes, 16-byte aligned.
 *   Xs  scales stored MN-major: the scale of token m, group g is
 *       Xs[g*ld_s + m] (float for F32, byte for UE8M0).  ld_s >= M.  ld_s is
 *       a multiple of 4 (F32) or 16 (UE8M0), and Xs is 16-byte aligned, so
 *       each scale row is a valid TMA source.  Entries m >= M are not written.
 * K % 128 == 0.  M == 0 is a no-op.
 */
fgfp8_status fgfp8_quant_act(const void* X, int64_t M, int64_t K, int64_t ldx, uint8_t* Xq, void* Xs,
                             int64_t ld_s, int fmt, void* stream);

/*
 * Block-scaled FP8 GEMM, Y = X * W^T with both scales applied per 128-wide
 * K block ("Fine-grained FP8", "DeepGEMM fast path": the FP8 linear layer).
 *   Xq, Xs, ld_s  as written by fgfp8_quant_act (same fmt).
 *   Wq, Ws        as written by fgfp8_quant_weight (same fmt).
 *   Y             bf16 [M, N] row-major (row stride N), 16-byte aligned.
 * K % 128 == 0, N % 128 == 0, M >= 0 arbitrary (M == 0 is a no-op).
 * M, N, K < 2^31.
 * The GEMM kernels are launched with programmatic stream serialization: they
 * may be scheduled while the preceding kernel in `stream` finishes, and wait
 * for its completion before their first access to global memory.
 */
fgfp8_status fgfp8_gemm(const uint8_t* Xq, const void* Xs, int64_t ld_s, const uint8_t* Wq, const void* Ws,
                        void* Y, int64_t M, int64_t N, int64_t K, int fmt, void* stream);

/*
 * M-grouped GEMM for MoE experts ("Fine-grained FP8", "DeepGEMM fast path":
 * the experts backend).  The rows of Xq are grouped per expert in
 * contiguous segments: rows [group_offs[e], group_offs[e+1]) belong to
 * expert e and are multiplied by Wq[e].
 *   Xq, Xs, ld_s  as from fgfp8_quant_act over all M_total rows.
 *   Wq            [E, N, K] E4M3 (E stacked fgfp8_quant_weight outputs).
 *   Ws            [E, N/128, K/128].
 *   Y             bf16 [M_total, N].
 *   group_offs    DEVICE int32 [E+1]: group_offs[0] == 0,
 *                 group_offs[E] == M_total, non-decreasing, every entry a
 *                 multiple of 128.  Empty experts are allowed.
 * Rows a caller padded with zeros produce zeros.  M_total % 128 == 0.  The
 * offsets are checked on the device.  Inconsistent offsets leave the affected
 * tiles unwritten, and fgfp8_check_device_status then reports
 * FGFP8_ERR_DEVICE.  Both scale formats are accepted.
 */
fgfp8_status fgfp8_grouped_gemm(const uint8_t* Xq, const void* Xs, int64_t ld_s, const uint8_t* Wq,
                                const void* Ws, void* Y, const int32_t* group_offs, int32_t E,
                                int64_t M_total, int64_t N, int64_t K, int fmt, void* stream);

/*
 * Masked (batched) expert GEMM for decode-time MoE ("Fine-grained FP8",
 * "DeepGEMM fast path": the experts backends, batched and masked expert
 * layouts): every expert e owns a fixed block of cap rows, rows
 * [e*cap, e*cap + cap), of which the first counts[e] hold tokens; rows
 * [e*cap + counts[e], e*cap + cap) are padding that is never read into Y.
 *   Xq, Xs, ld_s  as from fgfp8_quant_act over all E*cap rows (padding rows
 *                 may hold anything).
 *   Wq, Ws        [E, N, K] and [E, N/128, K/128] as for fgfp8_grouped_gemm.
 *   Y             bf16 [E*cap, N]; only token rows are written.
 *   counts        DEVICE int32 [E], each in [0, cap].
 * cap % 128 == 0.  Tiles of padding rows only are skipped.  A count outside
 * [0, cap] skips that expert's tiles and fgfp8_check_device_status then
 * reports FGFP8_ERR_DEVICE.  Both scale formats are accepted.
 */
fgfp8_status fgfp8_masked_gemm(const uint8_t* Xq, const void* Xs, int64_t ld_s, const uint8_t* Wq, const void* Ws,
                               void* Y, const int32_t* counts, int32_t E, int64_t cap, int64_t N, int64_t K, int fmt,
                               void* stream);

/*
 * The dynamic 1x128 activation quantizer of fgfp8_quant_act over the token
 * rows of the masked layout only: rows [e*cap, e*cap + counts[e]) of X for
 * every expert e.  Padding rows are not read, and their codes and scales
 * are left as they are: fgfp8_masked_gemm loads them with their tile, but no
 * output row depends on another row's input and rows past a count are never
 * stored.
 *   X        DEVICE bf16 [E*cap, K], row stride ldx; Xq, Xs, ld_s as for
 *            fgfp8_quant_act with M = E*cap.
 *   counts   DEVICE int32 [E]; a count below 0 quantizes no row and one
 *            above cap quantizes cap rows; either is recorded in the device
 *            status word (fgfp8_check_device_status then returns
 *            FGFP8_ERR_DEVICE), as fgfp8_masked_gemm does.
 * cap % 128 == 0, 1 <= E <= 65535; the other checks are those of
 * fgfp8_quant_act.  No counterpart on the pages: the decode step would
 * otherwise quantize every padding row.
 */
fgfp8_status fgfp8_quant_act_masked(const void* X, int64_t ldx, const int32_t* counts, int32_t E, int64_t cap,
                                    int64_t K, uint8_t* Xq, void* Xs, int64_t ld_s, int fmt, void* stream);

/*
 * The masked expert layer in one call: fgfp8_quant_act_masked into the
 * caller's Xq / Xs, then fgfp8_masked_gemm launched as the quantizer's
 * programmatic dependent.  Every argument is checked before either launch.
 */
fgfp8_status fgfp8_masked_linear(const void* X, int64_t ldx, uint8_t* Xq, void* Xs, int64_t ld_s, const uint8_t* Wq,
                                 const void* Ws, void* Y, const int32_t* counts, int32_t E, int64_t cap, int64_t N,
                                 int64_t K, int fmt, void* stream);

/*
 * The whole W8A8 linear layer: fgfp8_quant_act of X into the caller's Xq /
 * Xs buffers followed by fgfp8_gemm ("Fine-grained FP8", introduction and
 * "DeepGEMM fast path": activations are quantized on the fly, weights are
 * pre-quantized).  Arguments mean what they mean for those two calls; every
 * argument of both is validated before anything is launched, so on an error
 * nothing has been written.  The GEMM is launched as a programmatic
 * dependent of the quantizer and may start streaming Wq while the quantizer
 * runs: the quantizer writes only Xq and Xs, and it starts only after all
 * earlier work on `stream` has completed.  Y equals fgfp8_gemm's.
 */
fgfp8_status fgfp8_linear(const void* X, int64_t ldx, uint8_t* Xq, void* Xs, int64_t ld_s, const uint8_t* Wq,
                          const void* Ws, void* Y, int64_t M, int64_t N, int64_t K, int fmt, void* stream);

/*
 * The M-grouped expert layer: fgfp8_quant_act of the expert-grouped rows X
 * [M_total, K] followed by fgfp8_grouped_gemm, with the same validation-first
 * behaviour as fgfp8_linear.
 */
fgfp8_status fgfp8_grouped_linear(const void* X, int64_t ldx, uint8_t* Xq, void* Xs, int64_t ld_s,
                                  const uint8_t* Wq, const void* Ws, void* Y, const int32_t* group_offs,
                                  int32_t E, int64_t M_total, int64_t N, int64_t K, int fmt, void* stream);

/*
 * Scale granularity per row or per tensor ("FP8 W8A8", "Applying
 * quantization": the FP8_DYNAMIC scheme quantizes weights statically per
 * output channel and activations dynamically per token; static activation
 * scales, "Fine-grained FP8", "DeepGEMM fast path"; AbsMax per-tensor
 * calibration on the OwLite FP8 page).  Scales are fp32 and follow the same
 * rules as the 1x128 groups: scale = max(amax, 1e-4) / 448, code =
 * E4M3(x / scale) rounded to nearest even and saturated.
 */

/*
 * One scale per row of X bf16 [R, K] (row stride ldx elements, ldx % 8 == 0,
 * 16-byte aligned): per-token activations (rows = tokens) or per-output-
 * channel weights (rows = output channels of W [N, K]).
 *   Xq      E4M3 codes [R, K], row stride K bytes, 16-byte aligned.
 *   scales  float [R]: scales[r] = max(amax of row r, 1e-4) / 448.
 * K % 128 == 0; R == 0 is a no-op.
 */
fgfp8_status fgfp8_quant_rows(const void* X, int64_t R, int64_t K, int64_t ldx, uint8_t* Xq, float* scales,
                              void* stream);

/*
 * Per-tensor AbsMax scale of X bf16 [R, K]: *scale = max(amax over every
 * element, 1e-4) / 448 (one float in device memory, written on `stream`; a
 * NaN element gives a NaN scale).  The float is used as the reduction's
 * working word until the final value is written.
 */
fgfp8_status fgfp8_tensor_scale(const void* X, int64_t R, int64_t K, int64_t ldx, float* scale, void* stream);

/*
 * Static quantization with a given scale: Xq = E4M3(X / *scale), where
 * *scale is one float in device memory (a calibrated activation scale, or
 * the output of fgfp8_tensor_scale).  Layouts as for fgfp8_quant_rows.
 * Any positive scale is accepted, subnormal and +inf included, and the codes
 * equal those of the IEEE fp32 quotient x / scale for every finite bf16 x
 * (a quotient beyond 448, or an infinite one, saturates to +-448).  A scale
 * <= 0 or NaN is rejected on the device: no code is written and
 * fgfp8_check_device_status returns FGFP8_ERR_DEVICE.
 */
fgfp8_status fgfp8_quant_static(const void* X, int64_t R, int64_t K, int64_t ldx, const float* scale, uint8_t* Xq,
                                void* stream);

/*
 * Row/column-scaled FP8 GEMM:
 *   Y[m, n] = bf16( sx[m] * sw[n] * sum_k Xq[m, k] * Wq[n, k] )
 *   Xq  E4M3 [M, K] row-major, 16-byte aligned.
 *   sx  float [M] per-token scales (x_per_tensor = 0) or float [1]
 *       (x_per_tensor = 1), 4-byte aligned.
 *   Wq  E4M3 [N, K] row-major, 16-byte aligned.
 *   sw  float [N] per-channel scales (w_per_tensor = 0, 16-byte aligned) or
 *       float [1] (w_per_tensor = 1).
 *   Y   bf16 [M, N] row-major, 16-byte aligned.
 * K % 128 == 0, N % 128 == 0, M >= 0 arbitrary.  The K sum accumulates in
 * fp32; the result is within |Y - Y_exact| <= 2^-7 |Y_exact| + 1e-4 sum_k
 * |x_hat w_hat|.  Launched with programmatic stream serialization like
 * fgfp8_gemm.
 */
fgfp8_status fgfp8_gemm_rowcol(const uint8_t* Xq, const float* sx, int x_per_tensor, const uint8_t* Wq,
                               const float* sw, int w_per_tensor, void* Y, int64_t M, int64_t N, int64_t K,
                               void* stream);

/*
 * The gate/up projection of a SwiGLU MLP (Llama-3-8B's MLP: gate/up
 * [2I, K], then down [K_out, I]) fused with the down projection's dynamic
 * activation quantizer ("Fine-grained FP8", introduction and "DeepGEMM fast
 * path": 1x128 per-token groups, fp32 scales).  For every token m and
 * intermediate index i:
 *   g, u   = bf16_rne of the block-scaled GEMM outputs of the gate and up rows
 *   h      = bf16_rne( silu(g) * u ),  silu(g) = g * (1 / (1 + exp(-g))) in fp32
 *   Hq, Hs = fgfp8_quant_act of h (fp32 scales): codes [M, I] row-major and
 *            MN-major scales Hs[(i / 128) * ld_h + m]
 * so Hq / Hs feed fgfp8_gemm with the down-projection weight directly and
 * the bf16 [M, 2I] output of the gate/up projection is never written.
 *   Xq, Xs, ld_s  the block-quantized input [M, K] (fp32 scales).
 *   Wq_gu         E4M3 [2I, K]: gate and up rows interleaved in 128-row
 *                 blocks, rows [256 j, 256 j + 128) = gate rows [128 j, ..),
 *                 rows [256 j + 128, 256 j + 256) = up rows [128 j, ..).
 *   Ws_gu         float [2I/128, K/128], the 128x128 block scales in the same
 *                 interleaved order.
 *   Hq            E4M3 [M, I], 16-byte aligned; Hs, ld_h as for
 *                 fgfp8_quant_act (fp32, ld_h >= M, ld_h % 4 == 0).
 * I % 128 == 0, K % 128 == 0.  The codes equal fgfp8_quant_act of the h the
 * unfused layer would compute from its bf16 gate/up output, up to that
 * output's own GEMM rounding.
 */
fgfp8_status fgfp8_gemm_swiglu_quant(const uint8_t* Xq, const float* Xs, int64_t ld_s, const uint8_t* Wq_gu,
                                     const float* Ws_gu, uint8_t* Hq, float* Hs, int64_t ld_h, int64_t M, int64_t I,
                                     int64_t K, void* stream);

/*
 * Output layout of a tensor-parallel column split (no counterpart on the
 * pages, which run the layer on one GPU): when P ranks each hold n = N/P of
 * the weight's output rows (whole 128-row blocks with their block scales)
 * and compute their part of Y with fgfp8_linear / fgfp8_gemm, an all-gather
 * stacks the parts as parts bf16 [P, M, n]; this call writes them as
 * Y bf16 [M, P * n], Y[m, p * n + j] = parts[p, m, j].  Both buffers are in
 * this device's memory (the all-gather brings remote parts in first).
 *   parts, Y  16-byte aligned, contiguous; n % 8 == 0; P * M * n / 8 < 2^32.
 * P, M or n == 0 is a no-op.
 */
fgfp8_status fgfp8_gather_cols(const void* parts, int64_t P, int64_t M, int64_t n, void* Y, void* stream);

/* Size of the static scratch of fgfp8_linear_noalloc: 32 MiB per device. */
#define FGFP8_NOALLOC_SCRATCH_BYTES (32u << 20)

/*
 * fgfp8_linear without the Xq / Xs buffers, for callers that cannot allocate
 * device memory.  The source documentation has no counterpart to this call;
 * it exists for hosts such as a plugin that receives only its input and
 * output buffers from a framework that owns all device memory, a
 * latency-critical loop that must not call cudaMalloc (which can synchronize
 * the device), or a process whose memory pool is sized once at start-up and
 * refuses further allocations.
 *
 * The quantized activations live in one scratch array that the library
 * reserves statically on every device that loads it (FGFP8_NOALLOC_SCRATCH_BYTES,
 * held until the process exits).  The codes take M*K bytes rounded up to 256,
 * followed by the scales: (K/128) * round_up(M, 16) * (4 for F32, 1 for
 * UE8M0) bytes.  A request whose total exceeds FGFP8_NOALLOC_SCRATCH_BYTES
 * returns FGFP8_ERR_SHAPE before any CUDA call (for example M = 4096 tokens
 * fits for K = 4096, M = 8192 does not).
 *   X, ldx       bf16 [M, K] as for fgfp8_quant_act.
 *   Wq, Ws, fmt  the pre-quantized weight as for fgfp8_gemm.
 *   Y            bf16 [M, N], 16-byte aligned.
 * Y equals fgfp8_linear's for the same arguments.
 *
 * This call allocates nothing, through CUDA or any library.  Its first call
 * on a device looks up the scratch array's device address (with that device
 * current) and keeps it; make that first call before any stream capture on
 * the device.  Every call on a device shares the same array and leaves its
 * contents behind; each call writes every byte it later reads, so nothing
 * needs clearing between calls.  Calls whose kernels overlap on the GPU
 * (different streams, or different host threads, without ordering between
 * them) race on the array and give wrong results: order them on one stream.
 */
fgfp8_status fgfp8_linear_noalloc(const void* X, int64_t ldx, const uint8_t* Wq, const void* Ws, void* Y, int64_t M,
                                  int64_t N, int64_t K, int fmt, void* stream);

/*
 * Diagnostic with no counterpart on the pages: a self-test of the kernels'
 * bounded barrier waits.  Launches one thread on `stream` that waits on a
 * barrier nothing completes; after the one-second limit the wait gives up,
 * the device status word records a timeout and the kernel exits.
 * fgfp8_check_device_status then returns FGFP8_ERR_TIMEOUT, and the context
 * stays usable.  Returns FGFP8_ERR_CUDA without an sm_100a device.
 */
fgfp8_status fgfp8_selftest_expired_wait(void* stream);

/*
 * Diagnostic with no counterpart on the pages: a self-test of the GEMM's own
 * unwinding.  Runs the persistent dense GEMM (fmt F32: the promotion kernel;
 * UE8M0: the block-scaled kernel) on the given operands, exactly as
 * fgfp8_gemm would, except that the CTA holding work item 0 never requests
 * the operand tiles of K block withhold_kb.  The MMA issuer's wait for them
 * expires after its one-second limit, and with it the waits of the producer,
 * the scale stager and the epilogue: each role records a timeout, stops
 * issuing, waits (bounded) for the copies and MMAs it already issued, and
 * the CTA frees TMEM and exits within a few seconds.  The other CTAs finish
 * their tiles.  fgfp8_check_device_status then returns FGFP8_ERR_TIMEOUT,
 * the context stays usable, and Y's tile 0 is left unspecified.
 * Arguments as for fgfp8_gemm, with M > 64, N % 256 == 0 and
 * 0 <= withhold_kb < K/128.
 */
fgfp8_status fgfp8_selftest_gemm_timeout(const uint8_t* Xq, const void* Xs, int64_t ld_s, const uint8_t* Wq,
                                         const void* Ws, void* Y, int64_t M, int64_t N, int64_t K, int fmt,
                                         int64_t withhold_kb, void* stream);

/*
 * Synchronizes `stream`, then reads and clears the device status word that
 * the kernels set when they give up.  It returns FGFP8_OK,
 * FGFP8_ERR_TIMEOUT (a barrier wait ran past its one-second limit),
 * FGFP8_ERR_DEVICE (inconsistent group offsets, a masked count outside
 * [0, cap], or a static scale that is not positive) or FGFP8_ERR_CUDA.
 */
fgfp8_status fgfp8_check_device_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FGFP8_H */

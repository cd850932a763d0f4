/*
 * wq.h -- C ABI of libwq, group-wise weight quantisation and the
 * dequant-fused weight-only matmul for NVIDIA B200 (sm_100a).
 *
 * The operations follow these web pages (cited by title and section):
 *  [P2] "Quantization for LLM inference: FP8, INT4 (GPTQ, AWQ) and GGUF --
 *       the model's accounting zoom", section "The minimum maths: scale and
 *       zero-point": asymmetric b-bit quantisation of a block of weights,
 *       s = (max - min) / (2^b - 1), z = round(-min / s),
 *       q = clip(round(w / s + z), 0, 2^b - 1), decode w_hat = s * (q - z);
 *       section "Numerical example": 4-bit codes, two per byte, a bf16 scale.
 *  [P3] "Quantization Methods Compared: INT8, GPTQ, AWQ, FP8, FP4 and
 *       KV-Cache Quantization", section "What quantisation does": symmetric
 *       absmax INT8, s = max|w| / 127, q = round(w / s), w_hat = q * s;
 *       one scale per tensor, per output channel or per group of 128 (or 32)
 *       consecutive weights.  Section "Hardware, formats and the roofline":
 *       a decode step reads all the weights once, and 4-bit weights are
 *       turned back into 16-bit values inside the matmul kernel.  Section
 *       "The methods compared": the AWQ example, symmetric int4 with codes
 *       -7 to 7.
 *  [P1C] "Test-time quantization: quantising on the fly with no calibration
 *       dataset", section "The error of quantising an outlier with the wrong
 *       scale": a b-bit symmetric scale s = M / (2^(b-1) - 1), M / 7 at 4 bits.
 *
 * Conventions shared by every call
 *  - Weights are stored one row per output channel: W is [N][K] with K (the
 *    reduction axis) contiguous; groups are g consecutive weights of a row.
 *    y[m][n] = sum_k x[m][k] * w_hat[n][k].
 *  - bf16 values travel as uint16_t bit patterns (the top half of an IEEE
 *    binary32).  Row-major, densely packed unless a leading dimension is given.
 *  - Every pointer is a DEVICE pointer to memory the caller owns; the library
 *    never allocates or frees device memory.  Pointers must be 16-byte
 *    aligned.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream) and never synchronises.  Argument errors are
 *    detected on the host before anything is launched and leave every output
 *    untouched.
 *  - Inputs are finite; non-finite inputs give unspecified (but in-bounds)
 *    results.
 *  - Quantisation is bit-exact against the arithmetic stated below: binary32
 *    with round-to-nearest-even for every operation, "round" = round half to
 *    even, bf16 rounding = round to nearest even.
 *
 * Return value of every int-returning call: one of the WQ_* status codes.
 */
#ifndef WQ_H
#define WQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define WQ_OK 0
#define WQ_ERR_ARG (-1)            /* null pointer, a size <= 0, or an output overlapping an input */
#define WQ_ERR_SHAPE (-2)          /* K not a multiple of 32, g does not divide K, ldw < K */
#define WQ_ERR_ALIGN (-3)          /* a pointer not 16-byte aligned, or ldw % 8 != 0      */
#define WQ_ERR_UNSUPPORTED (-4)    /* group size or dtype outside the supported set       */
#define WQ_ERR_CUDA (-5)           /* a CUDA call or launch failed; see wq_last_error()   */
#define WQ_ERR_WORKSPACE (-6)      /* workspace null or smaller than wq_gemm_workspace_bytes */
#define WQ_ERR_DEVICE_TIMEOUT (-7) /* a kernel gave up on a bounded wait (see wq_device_status) */

/* Element type of the unquantised weight given to the quantisers. */
#define WQ_F32 0
#define WQ_BF16 1

/* FP8 formats: E4M3 (range +-448) and E5M2 (range +-57,344). */
#define WQ_FP8_E4M3 0
#define WQ_FP8_E5M2 1

/* Text for a status code (static storage; never NULL). */
const char *wq_status_str(int status);

/* Detail of the last error raised by a call on this host thread ("" if none). */
const char *wq_last_error(void);

/* Library ABI version: 100 * major + minor. */
int wq_version(void);

/*
 * Asymmetric INT4 quantisation, one (scale, zero-point) per group of g
 * consecutive weights along K  ([P2] "The minimum maths", b = 4).
 *
 *   w       [N][ldw] of WQ_F32 or WQ_BF16 (wtype); only the first K columns are read
 *   qweight [N][K/2] bytes: byte j of a row holds q[2j] in bits 0-3 and
 *           q[2j+1] in bits 4-7
 *   scales  [N][K/g] bf16;  zeros [N][K/g] bf16
 *
 * Per group, in binary32 (widening a bf16 w is exact):
 *   mn, mx = min, max of the group
 *   s  = bf16((mx - mn) / 15)                 one subtraction, one division
 *   if s == 0: s = bf16(max(|mn|, |mx|)); if still 0: s = 1
 *   z  = bf16(round(-mn / s) + 0)             (+0 turns -0 into +0)
 *   q  = clip(round(w / s + z), 0, 15)        with the stored s and z
 * Requirements: N >= 1; K >= 32, K % 32 == 0; g in {32, 64, 128}, K % g == 0;
 * ldw >= K, ldw % 8 == 0; all pointers 16-byte aligned; the outputs must not
 * overlap w or one another (WQ_ERR_ARG otherwise).
 */
int wq_quantize_int4(const void *w, int wtype, int64_t N, int64_t K, int64_t ldw, int g,
                     uint8_t *qweight, uint16_t *scales, uint16_t *zeros, void *stream);

/*
 * Asymmetric INT4 quantisation of column-scaled weights: exactly
 * wq_quantize_int4 applied to w[n][k] * col_scale[k], each product rounded
 * to binary32 -- the weights an activation-aware per-input-channel scaling
 * hands the quantiser ([P3] "The methods compared": AWQ scales the salient
 * channels up before quantising; the activations are divided by the same
 * scales, so the product is unchanged up to the quantisation).
 *
 *   col_scale  [K] binary32, device, 16-byte aligned; other arguments as
 *              wq_quantize_int4
 * Requirements: as wq_quantize_int4; col_scale non-NULL.
 */
int wq_quantize_int4_scaled(const void *w, int wtype, int64_t N, int64_t K, int64_t ldw, int g,
                            const float *col_scale, uint8_t *qweight, uint16_t *scales, uint16_t *zeros,
                            void *stream);

/*
 * Symmetric INT4 quantisation, one scale per group of g consecutive weights,
 * levels -7..7  ([P1C] "The error of quantising an outlier with the wrong
 * scale"; [P3] "The methods compared").  The output is the asymmetric INT4
 * format above with every zero-point 8, so wq_gemm_w4a16 consumes it as is.
 *
 *   w, qweight, scales, zeros: as wq_quantize_int4
 *
 * Per group, in binary32:
 *   s  = bf16(max|w| / 7); if s == 0: s = 1
 *   q  = clip(round(w / s), -7, 7)            with the stored s
 *   stored code q + 8 (1..15), zero-point 8: s * (code - 8) = s * q
 * Requirements: as wq_quantize_int4.
 */
int wq_quantize_int4_sym(const void *w, int wtype, int64_t N, int64_t K, int64_t ldw, int g,
                         uint8_t *qweight, uint16_t *scales, uint16_t *zeros, void *stream);

/*
 * Symmetric absmax INT8 quantisation  ([P3] "What quantisation does").
 * One scale per group of g weights; g == K gives one scale per output
 * channel (row).
 *
 *   w       [N][ldw] of WQ_F32 or WQ_BF16
 *   qweight [N][K] int8 in -127..127
 *   scales  [N][K/g] bf16
 *
 * Per group, in binary32:
 *   s = bf16(max|w| / 127); if s == 0: s = 1
 *   q = clip(round(w / s), -127, 127)   (the clip matters when the bf16 s
 *                                        rounded below max|w| / 127)
 * Requirements: as wq_quantize_int4, with g in {32, 64, 128, K}.
 */
int wq_quantize_int8(const void *w, int wtype, int64_t N, int64_t K, int64_t ldw, int g,
                     int8_t *qweight, uint16_t *scales, void *stream);

/*
 * Bytes of device workspace wq_gemm_w4a16 (wbits = 4) or wq_gemm_w8a16
 * (wbits = 8) needs for this shape; 0 when the chosen kernel needs none.
 * The workspace holds per-tile arrival counters, in its first 64 KB (a
 * multiple of 64 KB for shapes of more than 16,384 tiles, whose counters
 * above 64 KB the call clears first), and the binary32 partial sums of a
 * K-split above them.  A call that completes normally re-zeroes its counters,
 * so a workspace must be zero-filled once before its first use and may then
 * be reused by later calls on the same stream, of this or any other shape and
 * kernel, as long as it is large enough for each.  A call whose kernel gave
 * up on a bounded wait (wq_device_status returns WQ_ERR_DEVICE_TIMEOUT) can
 * leave counters non-zero: zero-fill the workspace again before reusing it
 * after such a status.
 */
size_t wq_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int g, int wbits);

/*
 * W4A16 weight-only matmul with in-kernel dequantisation
 * ([P2] decode w_hat = s * (q - z); [P3] "Hardware, formats and the roofline":
 * the 4-bit weights are expanded inside the matmul kernel).
 *
 *   x       [M][K] bf16 activations
 *   qweight, scales, zeros: as produced by wq_quantize_int4 with group g
 *   y       [M][N] bf16, y[m][n] = sum_k x[m][k] * s[n][k/g] * (q[n][k] - z[n][k/g])
 *
 * Arithmetic: the M = 1 kernel writes x, per block of 128 inputs, as 4 planes
 * of radix-128 integer digits (x_k = 2^(E-5) * sum_c d_ck * 128^-c, |d| <= 64,
 * 2^E <= max |x| of the block: exact for every |x_k| >= 2^(E-19), others
 * rounded to a multiple of 2^(E-26)), takes the exact integer sums
 * sum_k q_k d_ck of each group on the tensor core and applies
 * s * (D_c - z * sum_k d_ck) per group in binary32.  Every other kernel forms the exact integers (q - z)
 * in bf16 (a code pair 128 + q minus the pair 128 + z), multiplies them by x
 * with binary32 accumulation (tensor cores for the decode and batched
 * kernels), applies s per group in binary32.  y is rounded to bf16 once.
 * In those kernels a zero-point outside
 * [0, 15] (a group on one side of zero, far from it) is split as
 * z = z_hi + z_lo with z_lo in [0, 16) and z_hi a multiple of 16: the
 * operand is the exact q - z_lo and -z_hi times the group's activation sum
 * is added in binary32.  No term carries an
 * offset that cancels later, so rows whose weights are all zero give exactly
 * zero and |y - y_exact| stays within 4e-3 * sum_k |x[m][k] * w_hat[n][k]|
 * on the inputs this library is tested on (including activations spanning
 * ~e^+-20).  Split-K partial sums are combined in a fixed order, so repeated
 * calls give identical bytes, except on the older 2 <= M <= 16 kernel (the
 * shapes below that the persistent one does not take), whose partials meet in
 * binary32 atomics (the last bits of y may then vary between calls).
 * Kernels: M = 1 with 1024 <= K <= 32768, K % 1024 == 0 (K <= 31744 for
 * g = 32): persistent TMA-fed kernel on integer products (exact digits of x,
 * above; groups of 32 and 64 keep their digit sums in separate MMA columns);
 * 2 <= M <= 16 with g = 128 and the same K: the persistent TMA-fed kernel
 * with the M rows as the MMA's columns (at M = 2 on the integer products of
 * the M = 1 kernel), when the activations of a CTA's share fit shared
 * memory, else a TMA-fed decode kernel (N >= 128, K >= 256); M > 16,
 * 2 <= M <= 16 with g = 32 or 64, or 9 <= M <= 16 with g = 128 and
 * K % 1024 == 0 unless M <= 12 and the persistent kernel keeps three weight
 * stages (N >= 128, K % 128 == 0): tcgen05 tensor-core kernels; other shapes:
 * a CUDA-core kernel.
 * Requirements: M, N >= 1; K % 32 == 0; g in {32, 64, 128}, K % g == 0;
 * pointers 16-byte aligned; workspace of wq_gemm_workspace_bytes(M, N, K, g, 4)
 * bytes (may be NULL when that is 0).  y must not overlap x, qweight,
 * scales or zeros (WQ_ERR_ARG otherwise).
 * The persistent M = 1 and 2 <= M <= 16 kernels and the tensor-core kernel
 * for M > 16, g = 128 and K % 1024 == 0 are launched
 * with programmatic dependent launch: they start while the previous kernel
 * on the stream finishes, read x and write only after that kernel has
 * completed, but request their qweight, scales and zeros at once -- so
 * those must not have been written by the kernel just before on the same
 * stream (the y or workspace of the previous call, or the quantiser that
 * produced them: put another operation or an event between).
 * The persistent M = 1 kernel and the tensor-core kernels (except the
 * 128-column form of the one used for g = 32 or 64, or K % 1024 != 0) run at
 * most one CTA per SM and have a tile split between CTAs combined by the CTA
 * of its first segment, which waits for the others: a kernel on another
 * stream that holds SMs for good would make that wait run out
 * (WQ_ERR_DEVICE_TIMEOUT from wq_device_status after 1 s) rather than hang.
 */
int wq_gemm_w4a16(const uint16_t *x, int64_t M, int64_t N, int64_t K, const uint8_t *qweight,
                  const uint16_t *scales, const uint16_t *zeros, int g, uint16_t *y,
                  void *workspace, size_t ws_bytes, void *stream);

/*
 * W8A16 weight-only matmul: y[m][n] = sum_k x[m][k] * s[n][k/g] * q[n][k]
 * ([P3] dequantised value q * s).  qweight [N][K] int8, scales [N][K/g]
 * bf16, g in {32, 64, 128, K}.  Kernels: 1 <= M <= 8 with g = K (per output
 * channel), K % 128 == 0 and 128 <= K <= 65536, when the digit planes of a
 * CTA's share of K fit shared memory: a persistent TMA-fed kernel
 * on exact integer products (q as signed bytes against the radix-128 digit
 * planes of x described under wq_gemm_w4a16, s applied per row in binary32),
 * launched with programmatic dependent launch (qweight must not have been
 * written by the kernel just before on the same stream); other M >= 2 with
 * N >= 128 and K % 128 == 0: the tcgen05 tensor-core kernel (q converted exactly to
 * bf16, binary32 accumulation per group of g, or per 128 k for g = K, scaled
 * and summed in binary32); otherwise a CUDA-core kernel.  Workspace of
 * wq_gemm_workspace_bytes(M, N, K, g, 8) bytes.  Other arguments and
 * guarantees as wq_gemm_w4a16 (y is deterministic for every M here), the
 * integer kernel's split tiles combined by the CTA of their first segment as
 * there.
 */
int wq_gemm_w8a16(const uint16_t *x, int64_t M, int64_t N, int64_t K, const int8_t *qweight,
                  const uint16_t *scales, int g, uint16_t *y, void *workspace, size_t ws_bytes,
                  void *stream);

/*
 * W4A16 matmul of column-scaled activations: the activation side of
 * per-input-channel (AWQ-style) scaling ([P3] "The methods compared": AWQ
 * scales the salient channels up before quantising and the activations
 * compensate; [P1C] "The idea": the activations are divided by the same
 * scales, so the product is unchanged up to the quantisation).
 *
 *   y[m][n] = sum_k bf16(x[m][k] / col_scale[k]) * w_hat[n][k]
 *
 * with the weights quantised by wq_quantize_int4_scaled with the same
 * col_scale (binary32 [K], device, 16-byte aligned) and x / col_scale an IEEE
 * binary32 quotient rounded to bf16.  The M = 1 decode kernel divides while
 * it stages x (no extra pass); other shapes first write the scaled
 * activations behind the matmul's part of the workspace.  Arguments, accuracy and the rest of the
 * contract as wq_gemm_w4a16, with a workspace of
 * wq_gemm_w4a16_colscaled_workspace_bytes(M, N, K, g) bytes that must not
 * overlap x or y.
 */
size_t wq_gemm_w4a16_colscaled_workspace_bytes(int64_t M, int64_t N, int64_t K, int g);
int wq_gemm_w4a16_colscaled(const uint16_t *x, const float *col_scale, int64_t M, int64_t N, int64_t K,
                            const uint8_t *qweight, const uint16_t *scales, const uint16_t *zeros, int g, uint16_t *y,
                            void *workspace, size_t ws_bytes, void *stream);

/*
 * Channel statistics of the offline AWQ-style scale search ([P3] "The methods
 * compared": AWQ finds the salient channels from activation magnitudes and
 * searches the scale per channel; the pages give no formula, the reading
 * here is s_c = m_c^alpha normalised to max(s) * min(s) = 1).
 *
 * wq_awq_channel_magnitudes: magnitudes[k] = mean over the M rows of
 *   |x[m][k]|, binary64, rows summed in order (x [M][K] bf16; magnitudes [K]
 *   binary64, device).
 * wq_awq_channel_scales: col_scale[k] = m'^alpha / sqrt(max m'^alpha *
 *   min m'^alpha) in binary64, rounded once to binary32, with m' = m or, where
 *   m == 0, the smallest positive magnitude (1 if none); alpha in [0, 1].
 * Requirements: sizes >= 1, pointers 16-byte aligned, outputs not overlapping
 * the inputs.
 */
int wq_awq_channel_magnitudes(const uint16_t *x, int64_t M, int64_t K, double *magnitudes, void *stream);
int wq_awq_channel_scales(const double *magnitudes, int64_t K, double alpha, float *col_scale, void *stream);

/*
 * FP8 quantisation with one binary32 scale per output channel (row)
 * ("Quantization for LLM inference: FP8, INT4 (GPTQ, AWQ) and GGUF", section
 * "FP8: the Hopper/Blackwell datacenter format": E4M3 = 4 exponent and 3
 * mantissa bits, range +-448; E5M2 = 5 and 2, range +-57,344).
 *
 *   w       [N][ldw] of WQ_F32 or WQ_BF16
 *   fmt     WQ_FP8_E4M3 or WQ_FP8_E5M2
 *   qweight [N][K] FP8 codes (sign, exponent with bias 2^(e-1) - 1, mantissa;
 *           subnormals kept; E4M3 has no infinities)
 *   scales  [N] binary32
 *
 * Per row, in binary32:
 *   s    = max|w| / max_fmt; if s == 0: s = 1
 *   code = nearest FP8 value to w / s, ties to the even code, finite values
 *          beyond the range saturated to +-max_fmt
 * Requirements: as wq_quantize_int4 (without g); fmt one of the two formats
 * (WQ_ERR_UNSUPPORTED otherwise).
 */
int wq_quantize_fp8(const void *w, int wtype, int64_t N, int64_t K, int64_t ldw, int fmt, uint8_t *qweight,
                    float *scales, void *stream);

/*
 * FP8 quantisation of a whole tensor with one scale: the dynamic per-tensor
 * scaling of the activations of an FP8 W8A8 matmul (same page and section).
 *
 *   x      [M][K] dense, WQ_F32 or WQ_BF16 (xtype)
 *   q      [M][K] FP8 codes
 *   scale  one binary32 value on the device: s = max|x| / max_fmt (1 if 0)
 * Arithmetic as wq_quantize_fp8 with the tensor as one row.  Launches a
 * clear of *scale and three kernels (maximum, encode, scale); *scale holds
 * the maximum in between, so read it only after the call's work completes.
 * Requirements: M, K >= 1, K % 32 == 0; x, q 16-byte aligned, scale 4-byte
 * aligned; q and scale must not overlap x or each other.
 */
int wq_quantize_fp8_tensor(const void *x, int xtype, int64_t M, int64_t K, int fmt, uint8_t *q, float *scale,
                           void *stream);

/* Bytes of device workspace wq_gemm_w8a8_fp8 needs for this shape (same contract as
 * wq_gemm_workspace_bytes: zero-filled once, reusable after calls that complete normally). */
size_t wq_gemm_w8a8_fp8_workspace_bytes(int64_t M, int64_t N, int64_t K);

/*
 * FP8 W8A8 matmul on the tensor cores (same page and section: FP8 weights and
 * activations, multiplied by the tensor cores directly).
 *
 *   xq, xscale   [M][K] E4M3 codes and their per-tensor scale (one binary32
 *                value on the device), as from wq_quantize_fp8_tensor
 *   wq, wscales  [N][K] E4M3 codes and [N] binary32 scales, as from
 *                wq_quantize_fp8
 *   y            [M][N] bf16,
 *                y[m][n] = bf16((sum_k e4m3(xq[m][k]) * e4m3(wq[n][k])) * xscale * wscales[n])
 * The products are exact and accumulate in binary32 (tcgen05 kind::f8f6f4);
 * split-K partials are combined in a fixed order, so repeated calls give
 * identical bytes.  |y - y_exact| <= 4e-3 * sum_k |x_hat * w_hat| on the
 * inputs this library is tested on.
 * Requirements: M, N >= 1; K >= 128, K % 128 == 0; xq, wq, wscales, y 16-byte
 * aligned, xscale 4-byte aligned; workspace of
 * wq_gemm_w8a8_fp8_workspace_bytes bytes; y must not overlap an input.
 * Split tiles are combined by the CTA of their first segment, as described
 * under wq_gemm_w4a16.
 */
int wq_gemm_w8a8_fp8(const uint8_t *xq, const float *xscale, int64_t M, int64_t N, int64_t K, const uint8_t *wq,
                     const float *wscales, uint16_t *y, void *workspace, size_t ws_bytes, void *stream);

/*
 * NVFP4 quantisation ("Quantization Methods Compared: INT8, GPTQ, AWQ, FP8,
 * FP4 and KV-Cache Quantization", section "Hardware, formats and the
 * roofline": 4-bit values, one E4M3 scale per 16 values, one fp32 tensor
 * scale, 4.5 bits per value; "Quantization for LLM inference ...", section
 * "Microscaling: NVFP4 and MXFP4").  The 4-bit values are E2M1 (0, 0.5, 1,
 * 1.5, 2, 3, 4, 6 and their negatives).  In binary32, every division IEEE:
 *   st   = max|w over the whole tensor| / (6 * 448)      (1 if that is 0)
 *   sb   = E4M3 code of ((max|w over the block of 16| / 6) / st)
 *   code = nearest E2M1 value to w / (e4m3(sb) * st), ties to the even code,
 *          saturated at +-6 (0 when e4m3(sb) * st == 0)
 *
 *   w             [N][ldw] of WQ_F32 or WQ_BF16 (weights, or activations
 *                 [M][K] for the activation operand)
 *   codes         [N][K/2] bytes, value 2j of a row in bits 0-3 of byte j
 *   block_scales  wq_nvfp4_scale_bytes(N, K) bytes: E4M3 codes in the layout
 *                 the tensor cores read (512-byte atoms of 128 rows x 64
 *                 values of K; the scale of row r, block b sits at byte
 *                 16 (r % 32) + 4 ((r % 128) / 32) + (b % 4) of atom
 *                 (r / 128) * (K / 64) + b / 4); rows past N hold 0
 *   tensor_scale  one binary32 value on the device (holds the maximum while
 *                 the call's kernels run; read it after they complete)
 * Requirements: N >= 1; K >= 64, K % 64 == 0; ldw >= K, ldw % 8 == 0; w,
 * codes and block_scales 16-byte aligned, tensor_scale 4-byte aligned; no
 * output overlaps w or another output.
 */
size_t wq_nvfp4_scale_bytes(int64_t N, int64_t K);
int wq_quantize_nvfp4(const void *w, int wtype, int64_t N, int64_t K, int64_t ldw, uint8_t *codes,
                      uint8_t *block_scales, float *tensor_scale, void *stream);

/* Bytes of device workspace wq_gemm_nvfp4 needs for this shape (contract as wq_gemm_workspace_bytes). */
size_t wq_gemm_nvfp4_workspace_bytes(int64_t M, int64_t N, int64_t K);

/*
 * NVFP4 W4A4 matmul on the tensor cores with the block scales applied inside
 * the MMA (tcgen05.mma kind::mxf4nvf4, one E4M3 scale per 16 values):
 *   y[m][n] = bf16( (sum_b bx[m][b] bw[n][b] sum_{k in block b} e2m1(x[m][k]) e2m1(w[n][k]))
 *                   * x_tensor_scale * w_tensor_scale )
 * with both operands as produced by wq_quantize_nvfp4.  Products and their
 * block scalings are exact, sums binary32; split-K partials combine in a
 * fixed order.  |y - y_exact| <= 4e-3 * sum_k |x_hat * w_hat| on the inputs
 * this library is tested on.
 * Requirements: M, N >= 1; K >= 256, K % 256 == 0; every pointer 16-byte
 * aligned except the two tensor scales (4-byte); workspace of
 * wq_gemm_nvfp4_workspace_bytes bytes; y must not overlap an input.
 * Split tiles are combined by the CTA of their first segment, as described
 * under wq_gemm_w4a16.
 */
int wq_gemm_nvfp4(const uint8_t *x_codes, const uint8_t *x_block_scales, const float *x_tensor_scale, int64_t M,
                  int64_t N, int64_t K, const uint8_t *w_codes, const uint8_t *w_block_scales,
                  const float *w_tensor_scale, uint16_t *y, void *workspace, size_t ws_bytes, void *stream);

/*
 * Decode attention over a quantised KV cache: one new query token per
 * sequence against its first lengths[b] cached tokens ("Quantization Methods
 * Compared: INT8, GPTQ, AWQ, FP8, FP4 and KV-Cache Quantization", section
 * "Hardware, formats and the roofline": every decode step reads the whole
 * cache of every sequence; "Quantization for LLM inference: FP8, INT4 (GPTQ,
 * AWQ) and GGUF", section "KV cache quantization": fp8 caches, and int4
 * caches in blocks of 128 values).  Scaled dot-product attention:
 *   score_t = (q_j . k_hat_t) / sqrt(D), p = softmax over t < lengths[b],
 *   o_j = sum_t p_t v_hat_t,   query head j reading KV head j / (Hq / H);
 *   lengths[b] == 0 gives o_j = 0 (lengths are clamped to [0, T]).
 *
 *   q        [B][Hq][D] bf16
 *   int4 cache (K and V alike, each vector one block of 128 in the format of
 *            wq_quantize_int4 with g = 128 applied to the cache viewed as
 *            [B*T*H][D] rows): codes [B][T][H][D/2] bytes, scales and
 *            zero-points [B][T][H] bf16; v_hat = s (q - z)
 *   fp8 cache: E4M3 codes [B][T][H][D] and one binary32 scale per tensor on
 *            the device, as from wq_quantize_fp8_tensor; v_hat = s e4m3(code)
 *   lengths  [B] int32 on the device
 *   o        [B][Hq][D] binary32
 * Arithmetic: int4 keys and values enter the tensor cores as the exact
 * integers q - z (bf16), fp8 ones as exact f16 values; scores and sums are
 * binary32; p times the token's V scale (int4) or p (fp8) is rounded to
 * bf16 / f16 as the MMA operand.  |o - o_exact| <= 4e-3 * sum_t p_t |v_hat_t|
 * on the inputs this library is tested on.
 * Requirements: D == 128 and Hq % H == 0 with Hq / H <= 8
 * (WQ_ERR_UNSUPPORTED otherwise); B, T, H >= 1; every pointer 16-byte
 * aligned (the fp8 scales 4-byte); workspace of
 * wq_decode_attention_workspace_bytes(B, T, H) bytes (no zero-fill needed);
 * o must not overlap an input.
 */
size_t wq_decode_attention_workspace_bytes(int64_t B, int64_t T, int64_t H);
int wq_decode_attention_int4(const uint16_t *q, const uint8_t *k_codes, const uint16_t *k_scales,
                             const uint16_t *k_zeros, const uint8_t *v_codes, const uint16_t *v_scales,
                             const uint16_t *v_zeros, const int32_t *lengths, int64_t B, int64_t T, int64_t H,
                             int64_t Hq, int64_t D, float *o, void *workspace, size_t ws_bytes, void *stream);
int wq_decode_attention_fp8(const uint16_t *q, const uint8_t *k_codes, const float *k_scale, const uint8_t *v_codes,
                            const float *v_scale, const int32_t *lengths, int64_t B, int64_t T, int64_t H, int64_t Hq,
                            int64_t D, float *o, void *workspace, size_t ws_bytes, void *stream);

/*
 * W4A16 matmul for callers that cannot allocate device memory.  The pages
 * have no counterpart: this is an interface variant, not part of the method.
 *
 * Same operation, arguments and accuracy as wq_gemm_w4a16, but no workspace
 * argument: the split-K partial sums and tile counters live in a fixed 2 MiB
 * array inside the library (held on every GPU that loads the library until
 * the process exits).  For callers that cannot call cudaMalloc -- it
 * synchronises the device, and runtimes or plug-in hosts that own all device
 * memory, or fixed-budget deployments, forbid allocation after start-up.
 *
 *   Accepted shapes: g == 128, 2 <= M <= 16, N >= 128, K >= 256, K % 128 == 0
 *   (WQ_ERR_UNSUPPORTED otherwise), and M * N * 4 bytes plus one int per 128
 *   rows of N must fit in the 2 MiB array (WQ_ERR_WORKSPACE otherwise).
 *   The first call with a given device current looks up the array's device
 *   address (cudaGetSymbolAddress); make it before any stream capture.
 *   Each call clears the part of the array it uses on `stream` before its
 *   kernel runs.  All calls share the array: calls whose executions overlap on
 *   the GPU (other streams, other host threads) race on it.
 *   Allocates nothing; calls no cudaMalloc or cudaFree.
 */
int wq_gemm_w4a16_noalloc(const uint16_t *x, int64_t M, int64_t N, int64_t K, const uint8_t *qweight,
                          const uint16_t *scales, const uint16_t *zeros, int g, uint16_t *y, void *stream);

/*
 * Device status word.  Kernels with waits on barriers bound every wait; a
 * wait that runs out records a code on the device and the kernel returns
 * early instead of hanging.  This call synchronises `stream`, returns
 * WQ_ERR_DEVICE_TIMEOUT if any kernel of this library recorded a timeout on
 * the current device since the last call (and clears it), WQ_ERR_CUDA if the
 * stream reports an error, else WQ_OK.  After WQ_ERR_DEVICE_TIMEOUT the
 * outputs of the calls since the last check are unspecified and every
 * workspace they used must be zero-filled again before its next use.
 *
 * The device addresses of the status word and of the no-allocation scratch
 * array are looked up once per device and cached: do not keep using the
 * library after cudaDeviceReset in the same process.
 */
int wq_device_status(void *stream);

/*
 * Test hook of the failure path, for the library's own tests: the next
 * tensor-core W4A16 launch (wq_gemm_w4a16 with M > 16) never requests the
 * weight copy of its stream-K unit `unit` (tile * (K / 128) + stage), so
 * the waits on that copy run out after the bounded-wait limit (about 1 s):
 * the call returns, wq_device_status reports WQ_ERR_DEVICE_TIMEOUT and the
 * library stays usable.  No copy is left in flight.  Pass -1 to disarm.
 */
void wq_test_skip_weight_copy(int64_t unit);

#ifdef __cplusplus
}
#endif

#endif /* WQ_H */

// wq_internal.h -- host-side launchers behind the C ABI (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace wq {

// Workspace layout of every kernel that splits tiles between CTAs: the per-tile arrival counters first, in a
// region of counter_region_bytes(tiles) (4 bytes a tile, rounded up to 64 KB), then the binary32 partial sums.
// A call that completes normally re-zeroes its counters and leaves its partial sums behind; since every shape
// with up to 16,384 tiles keeps its counters below 64 KB and its partial sums above, one workspace can serve
// calls of any shapes in turn.  A shape with more tiles has counters above 64 KB, where another shape's partial
// sums may lie: clear_extra_counters() zeroes them on the stream before its launch.
constexpr size_t kCounterRegion = 65536;
inline size_t counter_region_bytes(int64_t tiles)
{
    return ((size_t)tiles * 4 + kCounterRegion - 1) / kCounterRegion * kCounterRegion;
}
inline cudaError_t clear_extra_counters(void *workspace, int64_t tiles, cudaStream_t st)
{
    const size_t region = counter_region_bytes(tiles);
    if (region <= kCounterRegion) return cudaSuccess;
    return cudaMemsetAsync(static_cast<uint8_t *>(workspace) + kCounterRegion, 0, region - kCounterRegion, st);
}

// y [M][N] bf16 overlaps x [M][K] bf16, the codes, the scales or the zero-points (wq_api.cu).
bool output_overlaps_inputs(const void *x, int64_t M, int64_t N, int64_t K, const void *q, const void *s,
                            const void *z, int g, const void *y, bool int8);

// Quantisers (wq_quant.cu).  Arguments are validated by the caller.
void launch_quantize_int4(const void *w, int wtype, int64_t N, int64_t K, int64_t ldw, int g, uint8_t *q,
                          uint16_t *s, uint16_t *z, cudaStream_t st);
void launch_quantize_int4_scaled(const void *w, int wtype, int64_t N, int64_t K, int64_t ldw, int g,
                                 const float *col_scale, uint8_t *q, uint16_t *s, uint16_t *z, cudaStream_t st);
void launch_quantize_int4_sym(const void *w, int wtype, int64_t N, int64_t K, int64_t ldw, int g, uint8_t *q,
                              uint16_t *s, uint16_t *z, cudaStream_t st);
void launch_quantize_int8(const void *w, int wtype, int64_t N, int64_t K, int64_t ldw, int g, int8_t *q,
                          uint16_t *s, cudaStream_t st);

// CUDA-core matmul for small M (wq_gemv.cu).  Any M >= 1 is accepted; rows of
// x are processed in tiles of up to 16.
void launch_gemv_w4a16(const uint16_t *x, int64_t M, int64_t N, int64_t K, const uint8_t *q, const uint16_t *s,
                       const uint16_t *z, int g, uint16_t *y, cudaStream_t st);
void launch_gemv_w8a16(const uint16_t *x, int64_t M, int64_t N, int64_t K, const int8_t *q, const uint16_t *s,
                       int g, uint16_t *y, cudaStream_t st);

// W4A16 for M = 1, group 128 (wq_gemv_m1.cu): persistent stream-K over
// (256-row tile, group pair) units, one TMA producer warp per CTA feeding
// 16 mma.sync consumer warps, a combiner warp for split tiles.  Needs a
// workspace of gemv_m1_workspace_bytes() (zero-filled before first use; the
// kernel leaves its counters zeroed) and the device status word for its
// bounded waits.  Returns 0, -1 if a tensor map cannot be encoded, -2 if the
// launch fails.
bool gemv_m1_eligible(int64_t M, int64_t N, int64_t K, int g);
size_t gemv_m1_workspace_bytes(int64_t M, int64_t N, int64_t K, int g);
// col_scale (optional, binary32 [K]): the kernel stages bf16(x / col_scale) instead of x.
int launch_gemv_w4a16_m1(const uint16_t *x, int64_t N, int64_t K, const uint8_t *q, const uint16_t *s,
                         const uint16_t *z, int g, uint16_t *y, void *workspace, int *status, cudaStream_t st,
                         const float *col_scale = nullptr);

// W4A16 for group 128 and M = 2 on integer products (wq_gemv_i4mt.cu): the M = 1 kernel with 2 rows x 4 digits
// in the MMA's B columns.  Eligible for 1024 <= K <= 32768, K % 1024 == 0 when a CTA's digit planes and
// two stages fit shared memory.  Workspace of gemv_i4mt_workspace_bytes() (zero-filled before first use; the
// kernel leaves its counters zeroed); the device status word.  Returns 0, -1 if a tensor map cannot be
// encoded, -2 if the launch fails.
bool gemv_i4mt_eligible(int64_t M, int64_t N, int64_t K, int g);
size_t gemv_i4mt_workspace_bytes(int64_t M, int64_t N, int64_t K, int g);
int launch_gemv_w4a16_i4mt(const uint16_t *x, int64_t M, int64_t N, int64_t K, const uint8_t *q, const uint16_t *s,
                           const uint16_t *z, uint16_t *y, void *workspace, int *status, cudaStream_t st,
                           const float *col_scale = nullptr);

// W4A16 for group 128 and 2 <= M <= 16 (wq_gemv_mt.cu): the M = 1 kernel's weight stream with the M
// activation rows as the bf16 columns of mma.sync and exact bf16 q - z operands.  Eligible when, in addition,
// 1024 <= K <= 32768, K % 1024 == 0 and the CTA's activation pairs fit shared memory.  Workspace of
// gemv_mt_workspace_bytes() (zero-filled before first use; the kernel leaves its counters zeroed); the device
// status word for its bounded waits.  Returns 0, -1 if a tensor map cannot be encoded, -2 if the launch fails.
bool gemv_mt_eligible(int64_t M, int64_t N, int64_t K, int g);
int gemv_mt_stages(int64_t M, int64_t N, int64_t K, int g);  // weight stages in flight; 0 when not eligible
size_t gemv_mt_workspace_bytes(int64_t M, int64_t N, int64_t K, int g);
int launch_gemv_w4a16_mt(const uint16_t *x, int64_t M, int64_t N, int64_t K, const uint8_t *q, const uint16_t *s,
                         const uint16_t *z, uint16_t *y, void *workspace, int *status, cudaStream_t st);

// W8A16 per output channel at 1 <= M <= 8 (wq_gemv_w8int.cu): persistent TMA-fed stream of the int8 codes,
// integer mma.sync s8 x s8 against exact digit planes of x.  Eligible for g == K, K % 128 == 0,
// 128 <= K <= 65536 when a CTA's digit planes and two stages fit shared memory.  Workspace of
// gemv_w8int_workspace_bytes() (zero-filled before first use; the kernel leaves its counters zeroed); the
// device status word for its bounded waits.  Returns 0, -1 if the tensor map cannot be encoded, -2 if the
// launch fails.
bool gemv_w8int_eligible(int64_t M, int64_t N, int64_t K, int g);
size_t gemv_w8int_workspace_bytes(int64_t M, int64_t N, int64_t K, int g);
int launch_gemv_w8a16_int(const uint16_t *x, int64_t M, int64_t N, int64_t K, const int8_t *q, const uint16_t *s,
                          uint16_t *y, void *workspace, int *status, cudaStream_t st);

// TMA-pipelined W4A16 for group 128 and M <= 16 (wq_gemv_tma.cu).  Needs a
// workspace of gemv_tma_workspace_bytes() (counters first, zero-filled before
// first use; the launcher clears the partial sums, which meet in atomics),
// or, compact = true, a private scratch area of gemv_tma_compact_bytes()
// cleared before every call (partial sums first).  Returns 0, -1 if the tensor map could not be
// encoded, -2 if clearing counters failed.
bool gemv_tma_eligible(int64_t M, int64_t N, int64_t K, int g);
size_t gemv_tma_workspace_bytes(int64_t M, int64_t N, int64_t K, int g);
size_t gemv_tma_compact_bytes(int64_t M, int64_t N, int64_t K, int g);
int launch_gemv_w4a16_tma(const uint16_t *x, int64_t M, int64_t N, int64_t K, const uint8_t *q, const uint16_t *s,
                          const uint16_t *z, uint16_t *y, void *workspace, int *status, cudaStream_t st,
                          bool compact = false);

// tcgen05 W4A16 for M > 16 (wq_gemm_tc.cu): N >= 128, K % 128 == 0.  Workspace
// of gemm_tc_workspace_bytes(): per-segment binary32 partials and per-tile
// counters (zero-filled before first use; the kernel leaves the counters zeroed).
int gemm_tc_bn(int64_t M, int g);
int64_t gemm_tc_max_segments(int64_t total, int64_t grid, int64_t spt);
int gemm_tc_w4_bn(int64_t M, int64_t K, int g);
size_t gemm_tc_partials_bytes(int64_t M, int64_t N, int64_t K, int BN);
bool gemm_tc_eligible(int64_t M, int64_t N, int64_t K, int g);
size_t gemm_tc_workspace_bytes(int64_t M, int64_t N, int64_t K, int g);
int launch_gemm_w4a16_tc(const uint16_t *x, int64_t M, int64_t N, int64_t K, const uint8_t *q, const uint16_t *s,
                         const uint16_t *z, int g, uint16_t *y, void *workspace, int *status, cudaStream_t st);
// W8A16 on the same tensor-core kernel (int8 codes converted exactly to bf16 in the dequant warps):
// M >= 2, N >= 128, K % 128 == 0, g in {32, 64, 128, K}.  Workspace as the W4A16 form's.
bool gemm_tc_w8_eligible(int64_t M, int64_t N, int64_t K, int g);
size_t gemm_tc_w8_workspace_bytes(int64_t M, int64_t N, int64_t K, int g);
int launch_gemm_w8a16_tc(const uint16_t *x, int64_t M, int64_t N, int64_t K, const int8_t *q, const uint16_t *s,
                         int g, uint16_t *y, void *workspace, int *status, cudaStream_t st);
// The 128 x 128-tile, g = 128 form with dequantisation and promotion in separate warps (wq_gemm_tc2.cu): the
// same workspace layout as gemm_tc_workspace_bytes(M, N, K, 128) with BN = 128.  skip_unit: failure-path
// tests only (-1 otherwise).
int launch_gemm_w4a16_tc2(const uint16_t *x, int64_t M, int64_t N, int64_t K, const uint8_t *q, const uint16_t *s,
                          const uint16_t *z, uint16_t *y, void *workspace, int *status, cudaStream_t st,
                          int64_t skip_unit);

// FP8 quantisers (wq_quant_fp8.cu): per output channel, and per tensor (the latter returns -1 if the
// scale cannot be cleared before its grid-wide maximum).
void launch_quantize_fp8_rows(const void *w, int wtype, int64_t N, int64_t K, int64_t ldw, int fmt, uint8_t *q,
                              float *s, cudaStream_t st);
int launch_quantize_fp8_tensor(const void *x, int xtype, int64_t count, int fmt, uint8_t *q, float *scale,
                               cudaStream_t st);

// FP8 W8A8 tcgen05 matmul (wq_gemm_lowp.cu): K % 128 == 0.  Workspace of gemm_fp8_workspace_bytes():
// per-segment binary32 partials and per-tile counters (zero-filled before first use; the kernel leaves the
// counters zeroed).  Returns 0, or -1 if a tensor map cannot be encoded.
size_t gemm_fp8_workspace_bytes(int64_t M, int64_t N, int64_t K);
int launch_gemm_w8a8_fp8(const uint8_t *xq, const float *xscale, int64_t M, int64_t N, int64_t K, const uint8_t *wq,
                         const float *wscale, uint16_t *y, void *workspace, int *status, cudaStream_t st);

// NVFP4 quantiser (wq_quant_nvfp4.cu): codes [N][K/2], block scales in the tensor-core atom layout
// (nvfp4_scale_bytes(N, K) bytes, rows padded to 128), binary32 tensor scale.  Returns -1 if a clear fails.
size_t nvfp4_scale_bytes(int64_t N, int64_t K);
int launch_quantize_nvfp4(const void *w, int wtype, int64_t N, int64_t K, int64_t ldw, uint8_t *codes, uint8_t *sf,
                          float *tscale, cudaStream_t st);

// NVFP4 W4A4 tcgen05 matmul (wq_gemm_lowp.cu): K % 256 == 0.  Workspace as the FP8 matmul's.
size_t gemm_nvfp4_workspace_bytes(int64_t M, int64_t N, int64_t K);
int launch_gemm_nvfp4(const uint8_t *xc, const uint8_t *xsf, const float *xts, int64_t M, int64_t N, int64_t K,
                      const uint8_t *wc, const uint8_t *wsf, const float *wts, uint16_t *y, void *workspace,
                      int *status, cudaStream_t st);

// Decode attention over an int4 or fp8 KV cache (wq_kv_attn.cu): D = 128, Hq / H <= 8.  Workspace of
// kv_attn_workspace_bytes() binary32 chunk partials (no zero-fill needed).
size_t kv_attn_workspace_bytes(int64_t B, int64_t T, int64_t H);
int launch_kv_attn(bool fp8, const uint16_t *q, const uint8_t *kc, const uint16_t *ks, const uint16_t *kz,
                   const float *k8s, const uint8_t *vc, const uint16_t *vs, const uint16_t *vz, const float *v8s,
                   const int *lengths, int64_t B, int64_t T, int64_t H, int64_t Hq, float *o, void *workspace,
                   cudaStream_t st);

// x_out[m][k] = bf16(x[m][k] / col_scale[k]) (IEEE binary32 quotient), M rows of K (wq_colscale.cu).
void launch_colscale_x(const uint16_t *x, int64_t M, int64_t K, const float *col_scale, uint16_t *x_out,
                       cudaStream_t st);
// mag64[k] = mean over the M rows of |x[m][k]| (binary64, rows in order; mag, if not null, its binary32
// rounding), and s[k] = m'[k]^alpha / sqrt(max_k m'^alpha * min_k m'^alpha) in binary64 rounded to binary32,
// m' = m or the smallest positive m where m == 0 (wq_colscale.cu).
void launch_channel_magnitudes(const uint16_t *x, int64_t M, int64_t K, double *mag64, float *mag, cudaStream_t st);
void launch_channel_scales(const double *mag64, int64_t K, double alpha, float *s, cudaStream_t st);

// Error reporting and the bounded-wait status word, for entry points outside wq_api.cu.
int record_error(int status, const char *msg);
void clear_error();
int *device_status_word();

}  // namespace wq

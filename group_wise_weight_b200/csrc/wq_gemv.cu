// wq_gemv.cu -- weight-only matmul for the decode regime (few activation
// rows), on CUDA cores.
//
// "Quantization Methods Compared: INT8, GPTQ, AWQ, FP8, FP4 and KV-Cache
// Quantization", section "Hardware, formats and the roofline": a decode step
// reads every weight once and does 2 x batch flops per weight, so at small
// batch the matmul is bound by the weight stream from HBM, and a real 4-bit
// kernel dequantises inside the kernel.  The decode is
// w_hat = s * (q - z) ("Quantization for LLM inference: FP8, INT4 (GPTQ, AWQ)
// and GGUF", "The minimum maths").
//
// Work layout.  A warp owns R consecutive weight rows n and walks the whole
// K axis; lane l takes the 16-byte slices l, l + 32, l + 64, ... of every
// one of its rows, so each warp load is 512 contiguous bytes of one row
// (128-bit coalesced, streamed past L1).  The slice's activations are loaded
// once (through L1, shared by every warp of the SM) and reused for the R
// rows.  At the end the R x MT partial sums are reduced across the warp with
// xor shuffles (a split-K over the 32 lanes) and lane 0 writes y.
//
// INT4 arithmetic.  A slice is 32 codes of one group (g >= 32).  The codes
// become bf16 values 128 + q with one LOP3 per pair; subtracting the pair
// (128 + z, 128 + z) leaves the exact integers q - z, and the products
// x * (q - z) are formed with the mixed-precision FMA (bf16 x bf16 into a
// binary32 accumulator; the product is exact); s is applied once per slice
// in binary32.  No term carries an offset that would have to cancel later,
// so rows of zeros give exactly zero and the rounding error stays
// proportional to sum |x w_hat|; the only rounding beyond binary32
// accumulation is the final bf16 store of y.  A zero-point outside [0, 15]
// is split (zp_split in wq_common.cuh): the products use q - z_lo and the
// slice adds -z_hi times its activation sum.
//
// INT8 arithmetic.  A slice is 16 codes.  Each code byte is flipped to
// q + 128, placed under the exponent of 2^23 by a byte permute and shifted
// back with one exact binary32 subtraction, then multiplied in packed
// binary32 pairs.
#include "wq_common.cuh"
#include "wq_internal.h"

namespace wq {

namespace {

constexpr int kGemvThreads = 256;

// Activation pairs matching the code pairs of nib_pair_bf16: for 8
// activations x0..x7 held as bf16x2 words (x0,x1) (x2,x3) (x4,x5) (x6,x7),
// return (x0,x4) (x1,x5) (x2,x6) (x3,x7).
__device__ __forceinline__ void pair_activations(const uint4 xv, uint32_t xp[4])
{
    xp[0] = __byte_perm(xv.x, xv.z, 0x5410);
    xp[1] = __byte_perm(xv.x, xv.z, 0x7632);
    xp[2] = __byte_perm(xv.y, xv.w, 0x5410);
    xp[3] = __byte_perm(xv.y, xv.w, 0x7632);
}

// Rows of a CTA: kGemvThreads / 32 / KSPLIT row groups of R rows; the KSPLIT
// warps of a group interleave over the K slices of the same rows and their
// partial sums meet in shared memory at the end.  With PF the next slice's
// weights, scales and zero-points are loaded before the current slice is
// consumed (two slices in flight per lane).
template <int MT, int R, int KSPLIT, bool PF>
__global__ void __launch_bounds__(kGemvThreads)
gemv_w4a16_kernel(const uint16_t *__restrict__ x, int64_t M, int64_t N, int64_t K,
                  const uint8_t *__restrict__ qw, const uint16_t *__restrict__ sc,
                  const uint16_t *__restrict__ zp, int g_shift, uint16_t *__restrict__ y)
{
    constexpr int kWarps = kGemvThreads / 32;
    constexpr int kGroups = kWarps / KSPLIT;
    __shared__ float red[KSPLIT > 1 ? kWarps : 1][R][MT];
    const int lane = threadIdx.x & 31;
    const int wid = threadIdx.x >> 5;
    const int kp = wid % KSPLIT;
    const int64_t n0 = ((int64_t)blockIdx.x * kGroups + wid / KSPLIT) * R;
    const bool live = n0 < N;  // warp-uniform; dead warps still join the final barrier
    const int64_t m0 = (int64_t)blockIdx.y * MT;
    const int64_t slices = K >> 5;
    const int64_t G = K >> g_shift;
    const int64_t row_bytes = K >> 1;

    int64_t nr[R];
#pragma unroll
    for (int r = 0; r < R; ++r) nr[r] = (n0 + r < N) ? n0 + r : N - 1;  // duplicates are not stored
    const uint16_t *xr[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) xr[m] = x + ((m0 + m < M) ? m0 + m : M - 1) * K;

    float acc[R][MT];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[r][m] = 0.0f;

    const int64_t step = 32 * KSPLIT;
    int64_t j = (int64_t)kp * 32 + lane;

    uint4 wq[R];
    uint16_t sb[R], zb[R];
    auto fetch = [&](int64_t jj) {
        const int64_t gi = (jj << 5) >> g_shift;
#pragma unroll
        for (int r = 0; r < R; ++r) wq[r] = ld_stream_v4(qw + nr[r] * row_bytes + (jj << 4));
#pragma unroll
        for (int r = 0; r < R; ++r) {
            sb[r] = ld_nc_u16(sc + nr[r] * G + gi);
            zb[r] = ld_nc_u16(zp + nr[r] * G + gi);
        }
    };
    if (live && PF && j < slices) fetch(j);

    for (; live && j < slices; j += step) {
        if (!PF) fetch(j);
        uint4 cw[R];
        float s[R], zh[R];
        uint32_t zz[R];  // bf16 pairs (128 + z, 128 + z), z split by zp_split when outside [0, 15]
        bool wide = false;
#pragma unroll
        for (int r = 0; r < R; ++r) {
            cw[r] = wq[r];
            s[r] = bf16_to_f32(sb[r]);
            float zl = bf16_to_f32(zb[r]);
            zh[r] = 0.0f;
            if (!(zl >= 0.0f && zl <= 15.0f)) {
                zl = zp_split(zl, zh[r]);
                wide = true;
            }
            zz[r] = bf16_pair_128_plus(zl);
        }
        float xs[MT];  // activation sums of the slice, needed when a zero-point was split
#pragma unroll
        for (int m = 0; m < MT; ++m) xs[m] = 0.0f;
        if (PF && j + step < slices) fetch(j + step);
        const int64_t k0 = j << 5;
        float part[R][MT];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m) part[r][m] = 0.0f;
#pragma unroll
        for (int wd = 0; wd < 4; ++wd) {
            uint32_t xp[MT][4];
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const uint4 xv = ld_nc_v4(xr[m] + k0 + 8 * wd);
                pair_activations(xv, xp[m]);
                if (wide) xs[m] += sum_bf16x8(xv);
            }
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const uint32_t v = wd == 0 ? cw[r].x : wd == 1 ? cw[r].y : wd == 2 ? cw[r].z : cw[r].w;
                uint32_t b[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) b[i] = sub_bf16x2(nib_pair_bf16(v, 4 * i), zz[r]);  // exact q - z
#pragma unroll
                for (int m = 0; m < MT; ++m)
#pragma unroll
                    for (int i = 0; i < 4; ++i) part[r][m] = fma_bf16x2(b[i], xp[m][i], part[r][m]);
            }
        }
        if (wide) {
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int m = 0; m < MT; ++m) part[r][m] = fmaf(-zh[r], xs[m], part[r][m]);
        }
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m) acc[r][m] = fmaf(s[r], part[r][m], acc[r][m]);
    }

#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[r][m] = warp_sum(acc[r][m]);
    if (KSPLIT > 1) {
        if (lane == 0) {
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int m = 0; m < MT; ++m) red[wid][r][m] = acc[r][m];
        }
        __syncthreads();
        if (kp != 0 || !live) return;
        if (lane == 0) {
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    float t = red[wid][r][m];
#pragma unroll
                    for (int p = 1; p < KSPLIT; ++p) t += red[wid + p][r][m];
                    acc[r][m] = t;
                }
        }
    }
    if (live && lane == 0) {
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m)
                if (n0 + r < N && m0 + m < M) y[(m0 + m) * N + n0 + r] = f32_to_bf16(acc[r][m]);
    }
}

// int8 bytes -> exact binary32 pairs: (q0, q1), (q2, q3) of one word.
__device__ __forceinline__ void int8_word_to_f32(uint32_t v, f32x2 &p01, f32x2 &p23)
{
    const uint32_t u = v ^ 0x80808080u;  // q + 128 in each byte
    const float b = 8388736.0f;          // 2^23 + 128
    p01 = add2(f32x2{__uint_as_float(__byte_perm(u, 0x4b000000u, 0x7540)),
                     __uint_as_float(__byte_perm(u, 0x4b000000u, 0x7541))},
               f32x2{-b, -b});
    p23 = add2(f32x2{__uint_as_float(__byte_perm(u, 0x4b000000u, 0x7542)),
                     __uint_as_float(__byte_perm(u, 0x4b000000u, 0x7543))},
               f32x2{-b, -b});
}

// W8A16 on CUDA cores, laid out like the INT4 kernel above: KSPLIT warps share R rows and interleave over
// their 16-byte K slices (partial sums meet in shared memory), and with PF each lane requests its next
// slice's codes and scales before it consumes the current one.
template <int MT, int R, int KSPLIT, bool PF>
__global__ void __launch_bounds__(kGemvThreads)
gemv_w8a16_kernel(const uint16_t *__restrict__ x, int64_t M, int64_t N, int64_t K,
                  const int8_t *__restrict__ qw, const uint16_t *__restrict__ sc, int64_t g,
                  uint16_t *__restrict__ y)
{
    constexpr int kWarps = kGemvThreads / 32;
    constexpr int kGroups = kWarps / KSPLIT;
    __shared__ float red[KSPLIT > 1 ? kWarps : 1][R][MT];
    const int lane = threadIdx.x & 31;
    const int wid = threadIdx.x >> 5;
    const int kp = wid % KSPLIT;
    const int64_t n0 = ((int64_t)blockIdx.x * kGroups + wid / KSPLIT) * R;
    const bool live = n0 < N;  // warp-uniform; dead warps still join the final barrier
    const int64_t m0 = (int64_t)blockIdx.y * MT;
    const int64_t slices = K >> 4;
    const int64_t G = K / g;

    int64_t nr[R];
#pragma unroll
    for (int r = 0; r < R; ++r) nr[r] = (n0 + r < N) ? n0 + r : N - 1;
    const uint16_t *xr[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) xr[m] = x + ((m0 + m < M) ? m0 + m : M - 1) * K;

    float acc[R][MT];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[r][m] = 0.0f;

    const int64_t step = 32 * KSPLIT;
    int64_t j = (int64_t)kp * 32 + lane;
    uint4 wq[R];
    uint16_t sb[R];
    auto fetch = [&](int64_t jj) {
        const int64_t k0 = jj << 4;
        const int64_t gi = k0 / g;
#pragma unroll
        for (int r = 0; r < R; ++r) wq[r] = ld_stream_v4(qw + nr[r] * K + k0);
#pragma unroll
        for (int r = 0; r < R; ++r) sb[r] = ld_nc_u16(sc + nr[r] * G + gi);
    };
    if (live && PF && j < slices) fetch(j);

    for (; live && j < slices; j += step) {
        if (!PF) fetch(j);
        uint4 cw[R];
        float s[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            cw[r] = wq[r];
            s[r] = bf16_to_f32(sb[r]);
        }
        if (PF && j + step < slices) fetch(j + step);
        const int64_t k0 = j << 4;
        f32x2 part[R][MT];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m) part[r][m] = f32x2{0.0f, 0.0f};
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // 8 activations at a time
            f32x2 xf[MT][4];
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const uint4 xv = ld_nc_v4(xr[m] + k0 + 8 * h);
                const uint32_t u[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    xf[m][i] = f32x2{__uint_as_float(u[i] << 16), __uint_as_float(u[i] & 0xffff0000u)};
            }
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const uint32_t w0 = h == 0 ? cw[r].x : cw[r].z;
                const uint32_t w1 = h == 0 ? cw[r].y : cw[r].w;
                f32x2 q[4];
                int8_word_to_f32(w0, q[0], q[1]);
                int8_word_to_f32(w1, q[2], q[3]);
#pragma unroll
                for (int m = 0; m < MT; ++m)
#pragma unroll
                    for (int i = 0; i < 4; ++i) part[r][m] = fma2(q[i], xf[m][i], part[r][m]);
            }
        }
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m) acc[r][m] = fmaf(s[r], part[r][m].x + part[r][m].y, acc[r][m]);
    }

#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[r][m] = warp_sum(acc[r][m]);
    if (KSPLIT > 1) {
        if (lane == 0) {
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int m = 0; m < MT; ++m) red[wid][r][m] = acc[r][m];
        }
        __syncthreads();
        if (kp != 0 || !live) return;
        if (lane == 0) {
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    float t = red[wid][r][m];
#pragma unroll
                    for (int p = 1; p < KSPLIT; ++p) t += red[wid + p][r][m];
                    acc[r][m] = t;
                }
        }
    }
    if (live && lane == 0) {
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m)
                if (n0 + r < N && m0 + m < M) y[(m0 + m) * N + n0 + r] = f32_to_bf16(acc[r][m]);
    }
}

int log2_int(int v)
{
    int s = 0;
    while ((1 << s) < v) ++s;
    return s;
}

template <int MT, int R, int KSPLIT, bool PF>
void run_w4(const uint16_t *x, int64_t M, int64_t N, int64_t K, const uint8_t *q, const uint16_t *s,
            const uint16_t *z, int g, uint16_t *y, cudaStream_t st)
{
    constexpr int rows_per_block = (kGemvThreads / 32 / KSPLIT) * R;
    const unsigned blocks = (unsigned)((N + rows_per_block - 1) / rows_per_block);
    const unsigned mtiles = (unsigned)((M + MT - 1) / MT);
    gemv_w4a16_kernel<MT, R, KSPLIT, PF><<<dim3(blocks, mtiles), kGemvThreads, 0, st>>>(x, M, N, K, q, s, z,
                                                                                       log2_int(g), y);
}

template <int MT, int R, int KSPLIT, bool PF>
void run_w8(const uint16_t *x, int64_t M, int64_t N, int64_t K, const int8_t *q, const uint16_t *s, int g,
            uint16_t *y, cudaStream_t st)
{
    constexpr int rows_per_block = (kGemvThreads / 32 / KSPLIT) * R;
    const unsigned blocks = (unsigned)((N + rows_per_block - 1) / rows_per_block);
    const unsigned mtiles = (unsigned)((M + MT - 1) / MT);
    gemv_w8a16_kernel<MT, R, KSPLIT, PF><<<dim3(blocks, mtiles), kGemvThreads, 0, st>>>(x, M, N, K, q, s, g, y);
}

}  // namespace

void launch_gemv_w4a16(const uint16_t *x, int64_t M, int64_t N, int64_t K, const uint8_t *q, const uint16_t *s,
                       const uint16_t *z, int g, uint16_t *y, cudaStream_t st)
{
    // The shapes the TMA kernels do not take come here (other group sizes, small N or K, M = 1 with
    // K outside the persistent kernel's range, M > 16 when the tensor-core kernel cannot run).
    if (M == 1) {
        // enough warps per SM to keep the weight stream busy: split K when rows are few
        if (N >= 32768) run_w4<1, 4, 2, false>(x, M, N, K, q, s, z, g, y, st);
        else run_w4<1, 4, 4, false>(x, M, N, K, q, s, z, g, y, st);
    }
    else if (M == 2) run_w4<2, 4, 2, false>(x, M, N, K, q, s, z, g, y, st);
    else if (M <= 4) run_w4<4, 2, 2, false>(x, M, N, K, q, s, z, g, y, st);
    else if (M <= 8) run_w4<8, 2, 1, false>(x, M, N, K, q, s, z, g, y, st);
    else run_w4<16, 1, 1, false>(x, M, N, K, q, s, z, g, y, st);
}

void launch_gemv_w8a16(const uint16_t *x, int64_t M, int64_t N, int64_t K, const int8_t *q, const uint16_t *s,
                       int g, uint16_t *y, cudaStream_t st)
{
    // M = 1: the next slice in flight per lane; many rows keep one warp per row group, fewer rows split K
    // over four warps (measured at K = N = 8192, N = 57,344 and K = 28,672: within 1% of the best layout
    // for each, where a one-warp, one-slice layout left the weight stream latency-bound)
    if (M == 1) {
        if (N >= 32768) run_w8<1, 4, 1, true>(x, M, N, K, q, s, g, y, st);
        else run_w8<1, 4, 4, true>(x, M, N, K, q, s, g, y, st);
    }
    else if (M == 2) run_w8<2, 4, 1, false>(x, M, N, K, q, s, g, y, st);
    else if (M <= 4) run_w8<4, 2, 1, false>(x, M, N, K, q, s, g, y, st);
    else if (M <= 8) run_w8<8, 2, 1, false>(x, M, N, K, q, s, g, y, st);
    else run_w8<16, 1, 1, false>(x, M, N, K, q, s, g, y, st);
}

}  // namespace wq

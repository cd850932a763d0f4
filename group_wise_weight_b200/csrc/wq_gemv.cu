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
// become bf16 values 128 + q with one LOP3 per pair, exact; the products
// x * (128 + q) are formed with the mixed-precision FMA (bf16 x bf16 into a
// binary32 accumulator; the product is exact) and the group's affine part is
// removed once per slice:
//     sum_k x_k s (q_k - z) = s * (sum_k x_k (128 + q_k) - (128 + z) sum_k x_k).
// (q - z) is never rounded and s is applied in binary32; the only rounding
// beyond binary32 accumulation is the final bf16 store of y.
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

    const uint32_t one2 = 0x3f803f80u;  // bf16x2 (1, 1)
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
        float s[R], zc[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            cw[r] = wq[r];
            s[r] = bf16_to_f32(sb[r]);
            zc[r] = 128.0f + bf16_to_f32(zb[r]);
        }
        if (PF && j + step < slices) fetch(j + step);
        const int64_t k0 = j << 5;
        float part[R][MT], xsum[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) xsum[m] = 0.0f;
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
#pragma unroll
                for (int i = 0; i < 4; ++i) xsum[m] = fma_bf16x2(xp[m][i], one2, xsum[m]);
            }
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const uint32_t v = wd == 0 ? cw[r].x : wd == 1 ? cw[r].y : wd == 2 ? cw[r].z : cw[r].w;
                uint32_t b[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) b[i] = nib_pair_bf16(v, 4 * i);
#pragma unroll
                for (int m = 0; m < MT; ++m)
#pragma unroll
                    for (int i = 0; i < 4; ++i) part[r][m] = fma_bf16x2(b[i], xp[m][i], part[r][m]);
            }
        }
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m) acc[r][m] = fmaf(s[r], fmaf(-zc[r], xsum[m], part[r][m]), acc[r][m]);
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

// ---------------------------------------------------------------------------
// Group-128 W4A16 for M <= 16 on the tensor pipe, operands straight from
// registers (mma.sync m16n8k16, bf16 in, binary32 accumulate).
//
// The CUDA-core form above spends ~4 instructions per weight (measured:
// ALU pipe ~70% busy at ~55% of HBM bandwidth), so here the multiply-adds
// move to the tensor pipe and only the nibble extraction stays on the ALU
// (3 shifts + 4 LOP3 per 8 weights).  The weight tile is the 16-row A
// operand, the activations are the 8-column B operand (M padded to 8 or 16).
//
// k permutation.  Lane (r, c) = (lane / 4, lane % 4) loads the 16 bytes
// covering k = 32c .. 32c + 31 of a 128-k chunk from rows n and n + 8.  A
// 32-bit word of those bytes (8 codes, k = 8i .. 8i + 7) yields the bf16x2
// pairs (c0,c4) (c1,c5) (c2,c6) (c3,c7) (128 + code, exact); pairs 2h and
// 2h+1 fill the lane's A slots of MMA (i, h), so MMA (i, h) sums over the
// 16 physical k = 32c' + 8i + {2h, 2h+1, 2h+4, 2h+5}, c' = 0..3.  The B
// fragment of the same lane holds the activations at the same physical k
// (bytes permuted the same way), so every product pairs the right x with
// the right code; the sum over all 8 MMAs of a chunk covers its 128 k once.
//
// Zero-point and scale.  One chunk is one group.  Its MMAs accumulate
// C[n][m] = sum_k (128 + q[n][k]) x[m][k] from zero; then, in binary32,
// y[m][n] += s[n] * (C[n][m] - (128 + z[n]) * X[m]) with
// X[m] = sum_k x[m][k] over the group, computed once per CTA into shared
// memory.  (q - z) is never rounded and s is applied in binary32.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_bf16_16816(float c[4], const uint32_t a[4], uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
                 "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t word_of(const uint4 &v, int i)
{
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// NT: 8-column activation tiles (M <= 8 * NT); R: 16-row weight tiles per
// warp; KSPLIT: warps sharing a row tile, interleaved over its chunks; U:
// chunks whose loads are all issued before any of them is consumed.
template <int NT, int R, int KSPLIT, int U>
__global__ void __launch_bounds__(kGemvThreads)
gemv_w4a16_g128_mma_kernel(const uint16_t *__restrict__ x, int64_t M, int64_t N, int64_t K,
                           const uint8_t *__restrict__ qw, const uint16_t *__restrict__ sc,
                           const uint16_t *__restrict__ zp, uint16_t *__restrict__ y)
{
    constexpr int kWarps = kGemvThreads / 32;
    constexpr int kGroups = kWarps / KSPLIT;
    constexpr int MP = 8 * NT;
    constexpr int kAcc = R * 2 * NT * 2;  // (row tile, row n / n+8, column tile, m / m+1)
    extern __shared__ float smem[];
    const int64_t G = K >> 7;
    float *Xs = smem;                                   // [MP][G]
    float *red = smem + MP * G;                         // [kGroups][KSPLIT-1][kAcc][32]
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int r4 = lane >> 2, c = lane & 3;
    const int kp = wid % KSPLIT, grp = wid / KSPLIT;
    const int64_t m0 = (int64_t)blockIdx.y * MP;
    const int64_t row_bytes = K >> 1;

    // group sums of the activations, once per CTA
    for (int64_t t = wid; t < MP * G; t += kWarps) {
        const int64_t m = t / G, gi = t - m * G;
        float v = 0.0f;
        if (m0 + m < M) {
            const uint2 p = *reinterpret_cast<const uint2 *>(x + (m0 + m) * K + gi * 128 + lane * 4);
            v = (__uint_as_float(p.x << 16) + __uint_as_float(p.x & 0xffff0000u)) +
                (__uint_as_float(p.y << 16) + __uint_as_float(p.y & 0xffff0000u));
        }
        v = warp_sum(v);
        if (lane == 0) Xs[t] = v;
    }
    __syncthreads();

    const uint16_t *xrow[NT];
    bool xok[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int64_t m = m0 + nt * 8 + r4;
        xok[nt] = m < M;
        xrow[nt] = x + (xok[nt] ? m : 0) * K;
    }

    const int64_t rows_per_tile = 16 * R * kGroups;
    const int64_t tiles = (N + rows_per_tile - 1) / rows_per_tile;
    for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
        const int64_t n0 = tile * rows_per_tile + (int64_t)grp * 16 * R;
        int64_t na[R], nb[R];
#pragma unroll
        for (int rr = 0; rr < R; ++rr) {
            const int64_t a = n0 + 16 * rr + r4;
            na[rr] = a < N ? a : N - 1;
            nb[rr] = a + 8 < N ? a + 8 : N - 1;
        }
        float acc[kAcc];
#pragma unroll
        for (int i = 0; i < kAcc; ++i) acc[i] = 0.0f;

        for (int64_t ch0 = kp; ch0 < G; ch0 += KSPLIT * U) {
            uint4 wa[U][R], wb[U][R];
            uint16_t sa[U][R], za[U][R], sbb[U][R], zbb[U][R];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t ch = ch0 + (int64_t)u * KSPLIT;
                if (ch < G) {
#pragma unroll
                    for (int rr = 0; rr < R; ++rr) {
                        wa[u][rr] = ld_stream_v4(qw + na[rr] * row_bytes + ch * 64 + c * 16);
                        wb[u][rr] = ld_stream_v4(qw + nb[rr] * row_bytes + ch * 64 + c * 16);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t ch = ch0 + (int64_t)u * KSPLIT;
                if (ch < G) {
#pragma unroll
                    for (int rr = 0; rr < R; ++rr) {
                        sa[u][rr] = ld_nc_u16(sc + na[rr] * G + ch);
                        za[u][rr] = ld_nc_u16(zp + na[rr] * G + ch);
                        sbb[u][rr] = ld_nc_u16(sc + nb[rr] * G + ch);
                        zbb[u][rr] = ld_nc_u16(zp + nb[rr] * G + ch);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t ch = ch0 + (int64_t)u * KSPLIT;
                if (ch >= G) break;
                uint32_t P[NT][4][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        if (xok[nt]) {
                            const uint4 xv = ld_nc_v4(xrow[nt] + ch * 128 + c * 32 + 8 * i);
                            pair_activations(xv, P[nt][i]);
                        } else {
                            P[nt][i][0] = P[nt][i][1] = P[nt][i][2] = P[nt][i][3] = 0u;
                        }
                    }
                float C[R][NT][4];
#pragma unroll
                for (int rr = 0; rr < R; ++rr)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        C[rr][nt][0] = C[rr][nt][1] = C[rr][nt][2] = C[rr][nt][3] = 0.0f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
#pragma unroll
                    for (int rr = 0; rr < R; ++rr) {
                        const uint32_t va = word_of(wa[u][rr], i), vb = word_of(wb[u][rr], i);
                        uint32_t RA[4], RB[4];
#pragma unroll
                        for (int t = 0; t < 4; ++t) {
                            RA[t] = nib_pair_bf16(va, 4 * t);
                            RB[t] = nib_pair_bf16(vb, 4 * t);
                        }
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const uint32_t a[4] = {RA[2 * h], RB[2 * h], RA[2 * h + 1], RB[2 * h + 1]};
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt)
                                mma_bf16_16816(C[rr][nt], a, P[nt][i][2 * h], P[nt][i][2 * h + 1]);
                        }
                    }
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const float x0 = Xs[(nt * 8 + 2 * c) * G + ch], x1 = Xs[(nt * 8 + 2 * c + 1) * G + ch];
#pragma unroll
                    for (int rr = 0; rr < R; ++rr) {
                        const float s_a = bf16_to_f32(sa[u][rr]), z_a = 128.0f + bf16_to_f32(za[u][rr]);
                        const float s_b = bf16_to_f32(sbb[u][rr]), z_b = 128.0f + bf16_to_f32(zbb[u][rr]);
                        float *A = acc + ((rr * 2) * NT + nt) * 2;
                        float *B = acc + ((rr * 2 + 1) * NT + nt) * 2;
                        A[0] = fmaf(s_a, fmaf(-z_a, x0, C[rr][nt][0]), A[0]);
                        A[1] = fmaf(s_a, fmaf(-z_a, x1, C[rr][nt][1]), A[1]);
                        B[0] = fmaf(s_b, fmaf(-z_b, x0, C[rr][nt][2]), B[0]);
                        B[1] = fmaf(s_b, fmaf(-z_b, x1, C[rr][nt][3]), B[1]);
                    }
                }
            }
        }

        if (KSPLIT > 1) {
            if (kp > 0) {
                float *dst = red + ((int64_t)(grp * (KSPLIT - 1) + kp - 1) * kAcc) * 32 + lane;
#pragma unroll
                for (int i = 0; i < kAcc; ++i) dst[i * 32] = acc[i];
            }
            __syncthreads();
            if (kp == 0) {
#pragma unroll
                for (int p = 1; p < KSPLIT; ++p) {
                    const float *src = red + ((int64_t)(grp * (KSPLIT - 1) + p - 1) * kAcc) * 32 + lane;
#pragma unroll
                    for (int i = 0; i < kAcc; ++i) acc[i] += src[i * 32];
                }
            }
            __syncthreads();
        }
        if (kp == 0) {
#pragma unroll
            for (int rr = 0; rr < R; ++rr)
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int64_t n = n0 + 16 * rr + r4 + 8 * half;
                    if (n >= N) continue;
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int64_t m = m0 + nt * 8 + 2 * c + e;
                            if (m < M) y[m * N + n] = f32_to_bf16(acc[((rr * 2 + half) * NT + nt) * 2 + e]);
                        }
                }
        }
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

template <int MT, int R>
__global__ void __launch_bounds__(kGemvThreads)
gemv_w8a16_kernel(const uint16_t *__restrict__ x, int64_t M, int64_t N, int64_t K,
                  const int8_t *__restrict__ qw, const uint16_t *__restrict__ sc, int64_t g,
                  uint16_t *__restrict__ y)
{
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t n0 = warp * R;
    if (n0 >= N) return;
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

    for (int64_t j = lane; j < slices; j += 32) {
        const int64_t k0 = j << 4;
        const int64_t gi = k0 / g;
        uint4 wq[R];
        float s[R];
#pragma unroll
        for (int r = 0; r < R; ++r) wq[r] = ld_stream_v4(qw + nr[r] * K + k0);
#pragma unroll
        for (int r = 0; r < R; ++r) s[r] = bf16_to_f32(ld_nc_u16(sc + nr[r] * G + gi));
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
                const uint32_t w0 = h == 0 ? wq[r].x : wq[r].z;
                const uint32_t w1 = h == 0 ? wq[r].y : wq[r].w;
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
    if (lane == 0) {
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

template <int MT, int R>
void run_w8(const uint16_t *x, int64_t M, int64_t N, int64_t K, const int8_t *q, const uint16_t *s, int g,
            uint16_t *y, cudaStream_t st)
{
    const int64_t warps = (N + R - 1) / R;
    const unsigned blocks = (unsigned)((warps * 32 + kGemvThreads - 1) / kGemvThreads);
    const unsigned mtiles = (unsigned)((M + MT - 1) / MT);
    gemv_w8a16_kernel<MT, R><<<dim3(blocks, mtiles), kGemvThreads, 0, st>>>(x, M, N, K, q, s, g, y);
}

}  // namespace

template <int NT, int R, int KSPLIT, int U>
void run_w4_mma(const uint16_t *x, int64_t M, int64_t N, int64_t K, const uint8_t *q, const uint16_t *s,
                const uint16_t *z, uint16_t *y, cudaStream_t st)
{
    auto kern = gemv_w4a16_g128_mma_kernel<NT, R, KSPLIT, U>;
    constexpr int kGroups = kGemvThreads / 32 / KSPLIT;
    const int64_t G = K / 128;
    const size_t smem = sizeof(float) * (8 * NT * G + (size_t)kGroups * (KSPLIT - 1) * R * 2 * NT * 2 * 32);
    if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    int dev = 0, sms = 148, per_sm = 1;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kGemvThreads, smem);
    if (per_sm < 1) per_sm = 1;
    const int64_t rows_per_tile = 16 * R * kGroups;
    const int64_t tiles = (N + rows_per_tile - 1) / rows_per_tile;
    const int64_t cap = (int64_t)sms * per_sm;
    const unsigned blocks = (unsigned)(tiles < cap ? tiles : cap);
    const unsigned mtiles = (unsigned)((M + 8 * NT - 1) / (8 * NT));
    kern<<<dim3(blocks, mtiles), kGemvThreads, smem, st>>>(x, M, N, K, q, s, z, y);
}

void launch_gemv_w4a16(const uint16_t *x, int64_t M, int64_t N, int64_t K, const uint8_t *q, const uint16_t *s,
                       const uint16_t *z, int g, uint16_t *y, cudaStream_t st)
{
    // M = 1: the CUDA-core form below measured fastest.  2 <= M <= 16 normally takes the TMA
    // pipeline (wq_gemv_tma.cu); shapes it does not take (N < 128, K < 256) come here.
    if (g == 128 && M >= 2 && M <= 16) {
        if (M <= 8) run_w4_mma<1, 1, 4, 2>(x, M, N, K, q, s, z, y, st);
        else run_w4_mma<2, 1, 4, 2>(x, M, N, K, q, s, z, y, st);
        return;
    }
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
    if (M == 1) run_w8<1, 4>(x, M, N, K, q, s, g, y, st);
    else if (M == 2) run_w8<2, 4>(x, M, N, K, q, s, g, y, st);
    else if (M <= 4) run_w8<4, 2>(x, M, N, K, q, s, g, y, st);
    else if (M <= 8) run_w8<8, 2>(x, M, N, K, q, s, g, y, st);
    else run_w8<16, 1>(x, M, N, K, q, s, g, y, st);
}

}  // namespace wq

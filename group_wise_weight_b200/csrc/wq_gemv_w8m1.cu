// wq_gemv_w8m1.cu -- W8A16 per output channel, a single activation row
// (M = 1): the decode step over symmetric INT8 weights, bound by streaming
// one byte per weight from HBM.
//
// "Quantization Methods Compared: INT8, GPTQ, AWQ, FP8, FP4 and KV-Cache
// Quantization", section "What quantisation does": symmetric absmax INT8,
// w_hat = s q with s = max |w| / 127 per output channel; section "Hardware,
// formats and the roofline": at batch 1 the decode step reads every weight
// once.
//
// The products are exact integer ones, as in the INT4 decode kernel
// (wq_gemv_m1.cu): x is written once per CTA as 4 planes of radix-128 digits
// per group of 128 inputs (x_k = 2^(E_g - 5) sum_c d_ck 128^-c, |d| <= 64;
// exact for every |x_k| >= 2^(E_g - 19), the rest rounded to a multiple of
// 2^(E_g - 26)), and the codes q, signed bytes as stored, are the A operand
// of mma.sync m16n8k32 s8 x s8 -> s32 against the digit planes in its B
// columns with no conversion at all.  Per group the lane adds 2^(E_g - 5) D_c
// (D_c = sum_k q_k d_ck, exact) to its column's binary32 sum; the columns
// meet, weighted by 128^-c, and s multiplies the row once per segment.
//
// Structure: a persistent grid, one CTA per SM; 16 consumer warps, a TMA
// producer warp and a combiner warp.  A unit is (256-row tile, group of 128
// inputs): one 32 KB stage, a 2-D box of 256 rows x 128 bytes loaded with the
// 128-byte swizzle (the 16-byte chunk c of row r lands at c ^ (r mod 8), so the
// consumers' 16-byte reads of two rows per quarter-warp do not collide).
// Stream-K over units, split tiles combined in segment order by the combiner
// warp, programmatic dependent launch, bounded waits -- all as in the INT4
// decode kernel.
#include <algorithm>
#include <map>
#include <mutex>

#include "wq_common.cuh"
#include "wq_internal.h"
#include "wq_sm100.cuh"

namespace wq {

namespace {

constexpr int kC = 16;                         // consumer warps
constexpr int kProducer = kC;
constexpr int kCombiner = kC + 1;
constexpr int kT = (kC + 2) * 32;
constexpr int kTile = 16 * kC;                 // rows per tile (256)
constexpr int kStages = 3;
constexpr uint32_t kStageBytes = kTile * 128;  // 256 rows x 128 codes
constexpr int kDigits = 4;
constexpr uint32_t kDigitGroupBytes = 2 * 4 * kDigits * 16;  // [half][t][digit][16 B] per group of 128
constexpr float kMagic = 12582912.0f;          // 1.5 * 2^23
constexpr uint32_t kMagicBits = 0x4B400000u;

// shared memory: [stages][2 partial tiles][digit planes][group factors][barriers]
struct W8Layout {
    size_t part, dig, gfac, bar, total;
    __host__ __device__ explicit W8Layout(int nslots)
    {
        part = (size_t)kStages * kStageBytes;
        dig = part + 2 * kTile * 4;
        gfac = dig + (size_t)nslots * kDigitGroupBytes;
        bar = (gfac + (size_t)nslots * 4 + 7) & ~(size_t)7;
        total = bar + (2 * kStages + 4 + 2) * 8 + 1024;
    }
};

__device__ __forceinline__ void mma_s8s8(uint32_t d[4], const uint32_t c[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%10, %11, %12, %13};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(c[0]), "r"(c[1]), "r"(c[2]), "r"(c[3]));
}

__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ uint4 lds128(uint32_t addr)
{
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(addr));
    return r;
}

__device__ __forceinline__ float lds_f32(uint32_t addr)
{
    float r;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(r) : "r"(addr));
    return r;
}

__device__ __forceinline__ uint32_t word_of(const uint4 &v, int i)
{
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

__device__ __forceinline__ int atom_add_acq_rel(int *p, int v)
{
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

__host__ __device__ __forceinline__ int cta_of(int64_t u, int64_t units, int64_t B)
{
    return (int)(((u + 1) * B - 1) / units);
}

__device__ __forceinline__ void wait_drain(uint64_t *bar, uint32_t parity, int *status)
{
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_ns() - t0 > kWaitLimitNs) { record_timeout(status); return; }
}

__device__ __forceinline__ float exp2i(int e) { return __uint_as_float((uint32_t)(e + 127) << 23); }

// The digit planes and the scale factor of one group of x (one warp).  Lane L holds word L / 2 of the group
// (inputs 8 (L / 2) .. + 7) and takes of it the four inputs 4 (L % 2) .. + 3, the byte order of the A
// operand's words: codes k .. k + 3 of the first word of a step, k + 4 .. k + 7 of the second.
__device__ __forceinline__ void make_digits8(uint4 v, uint32_t dig_g, uint32_t gfac_g, int lane)
{
    const int wq_ = lane >> 1, par = lane & 1;
    float e[4];
    const uint32_t w0 = par ? v.z : v.x, w1 = par ? v.w : v.y;
    e[0] = __uint_as_float(w0 << 16);
    e[1] = __uint_as_float(w0 & 0xffff0000u);
    e[2] = __uint_as_float(w1 << 16);
    e[3] = __uint_as_float(w1 & 0xffff0000u);
    float m = fmaxf(fmaxf(fabsf(e[0]), fabsf(e[1])), fmaxf(fabsf(e[2]), fabsf(e[3])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    // an infinite or NaN activation makes the group's factor NaN, so y is not finite, as x * w_hat would be
    const bool nonfinite = __any_sync(0xffffffffu, !(fabsf(e[0]) < INFINITY && fabsf(e[1]) < INFINITY &&
                                                     fabsf(e[2]) < INFINITY && fabsf(e[3]) < INFINITY));
    if (nonfinite) m = 0.0f;
    int E = m > 0.0f ? (int)((__float_as_uint(m) >> 23) & 0xff) - 127 : 0;
    if (m > 0.0f && E == -127) E = -127 + (31 - __clz((int)(__float_as_uint(m) & 0x7fffff))) - 22;  // subnormal
    const int a1 = (5 - E) / 2, a2 = (5 - E) - a1;
    const float sc1 = exp2i(a1), sc2 = exp2i(a2);
    uint32_t t[4][kDigits];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float X = (e[i] * sc1) * sc2;
#pragma unroll
        for (int c = 0; c < kDigits; ++c) {
            const float tt = X + kMagic;
            t[i][c] = __float_as_uint(tt);
            X = (X - (tt - kMagic)) * 128.0f;
        }
    }
    const int t_ = wq_ >> 2, w = wq_ & 3, half = w >> 1;
    const uint32_t dst = dig_g + (uint32_t)((half * 4 + t_) * (kDigits * 16) + (w & 1) * 8 + par * 4);
#pragma unroll
    for (int c = 0; c < kDigits; ++c) {
        const uint32_t lo = __byte_perm(t[0][c], t[1][c], 0x0040), hi = __byte_perm(t[2][c], t[3][c], 0x0040);
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(dst + (uint32_t)c * 16u), "r"(__byte_perm(lo, hi, 0x5410)) : "memory");
    }
    if (lane == 0) {
        const int ef = E - 5;
        float f = ef >= -126 ? exp2i(ef) : exp2i(ef + 64) * 5.421010862427522e-20f;  // 2^-64
        if (nonfinite) f = __int_as_float(0x7fc00000);                                 // NaN
        asm volatile("st.shared.f32 [%0], %1;" ::"r"(gfac_g), "f"(f) : "memory");
    }
}

__global__ void __maxnreg__(96)
gemv_w8a16_m1_kernel(const __grid_constant__ CUtensorMap wmap, const uint16_t *__restrict__ x,
                     const uint16_t *__restrict__ sc, int N, int K, uint16_t *__restrict__ y, float *__restrict__ ws,
                     int *__restrict__ cnt, int max_segs, int *__restrict__ status, int nslots_max)
{
    extern __shared__ __align__(1024) uint8_t w8_raw[];
    uint8_t *sm = w8_raw + ((1024u - (smem_u32(w8_raw) & 1023u)) & 1023u);
    const W8Layout L(nslots_max);
    uint8_t *ring = sm;
    float *part = reinterpret_cast<float *>(sm + L.part);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L.bar);
    uint64_t *full = bars, *empty = bars + kStages;
    uint64_t *pfull = bars + 2 * kStages, *pempty = pfull + 2;
    volatile int *flags = reinterpret_cast<volatile int *>(pempty + 2);
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int G = K >> 7;  // groups (units) per tile

    pdl_launch_dependents();
    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kC);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&pfull[i], kC);
            mbar_init(&pempty[i], 1);
        }
        flags[0] = 0;
        flags[1] = 0;
        fence_mbar_init();
    }
    __syncthreads();

    const int ntiles = (N + kTile - 1) / kTile;
    const int64_t units = (int64_t)ntiles * G;
    const int64_t B = min((int64_t)gridDim.x, units);
    const int64_t bid = blockIdx.x;
    const int64_t beg = bid < B ? units * bid / B : units, end = bid < B ? units * (bid + 1) / B : units;
    const int n = (int)(end - beg);
    const int tile0 = (int)(beg / G), grp0 = (int)(beg - (int64_t)tile0 * G);

    // The codes are inputs the preceding call does not write: the first stages are requested before the
    // grid-dependency wait; x and the scales wait.
    int pt = tile0, pg = grp0, pi = 0;
    if (wid == kProducer && lane == 0) {
        for (; pi < kStages && pi < n; ++pi) {
            mbar_arrive_expect_tx(&full[pi], kStageBytes);
            tma_load_2d(ring + (uint32_t)pi * kStageBytes, &wmap, &full[pi], pg * 128, pt * kTile);
            if (++pg == G) { pg = 0; ++pt; }
        }
    }
    pdl_wait();

    if (wid == kProducer) {
        // ================================ producer ================================
        if (lane == 0 && n > 0) {
            int i = pi;
            for (; i < n; ++i) {
                const int s = i % kStages;
                if (!mbar_wait(&empty[s], (uint32_t)(i / kStages - 1) & 1u, status, flags)) break;
                mbar_arrive_expect_tx(&full[s], kStageBytes);
                tma_load_2d(ring + (uint32_t)s * kStageBytes, &wmap, &full[s], pg * 128, pt * kTile);
                if (++pg == G) { pg = 0; ++pt; }
            }
            for (int j = max(0, i - kStages); j < i; ++j) wait_drain(&full[j % kStages], (uint32_t)(j / kStages) & 1u, status);
        }
        __syncthreads();
        return;
    }

    if (wid == kCombiner) {
        // ================================ combiner ================================
        int pseg = 0;
        for (int64_t tt = beg / G; tt * G < end; ++tt) {
            if (tt * G >= beg && tt * G + G <= end) continue;  // whole tile: the consumers wrote y
            const int b = pseg & 1;
            const bool ok = __all_sync(0xffffffffu, mbar_wait(&pfull[b], (uint32_t)(pseg >> 1) & 1u, status, flags));
            if (!ok) break;
            const float4 v0 = *reinterpret_cast<const float4 *>(part + b * kTile + 8 * lane);
            const float4 v1 = *reinterpret_cast<const float4 *>(part + b * kTile + 8 * lane + 4);
            __syncwarp();
            if (lane == 0) mbar_arrive(&pempty[b]);
            ++pseg;
            const int c_first = cta_of(tt * G, units, B);
            const int nseg = cta_of(tt * G + G - 1, units, B) - c_first + 1;
            float *slots = ws + (size_t)tt * max_segs * kTile;
            float4 *mine = reinterpret_cast<float4 *>(slots + (bid - c_first) * kTile + 8 * lane);
            mine[0] = v0;
            mine[1] = v1;
            __syncwarp();
            int last = 0;
            if (lane == 0) last = (atom_add_acq_rel(cnt + tt, 1) + 1 == nseg) ? 1 : 0;
            last = __shfl_sync(0xffffffffu, last, 0);
            if (last) {
                float v[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
                const float4 *q = reinterpret_cast<const float4 *>(slots + 8 * lane);
                int o = 0;
                for (; o + 4 <= nseg; o += 4) {
                    float4 a[8];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        a[2 * j] = __ldcg(q + (size_t)(o + j) * (kTile / 4));
                        a[2 * j + 1] = __ldcg(q + (size_t)(o + j) * (kTile / 4) + 1);
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        v[0] += a[2 * j].x; v[1] += a[2 * j].y; v[2] += a[2 * j].z; v[3] += a[2 * j].w;
                        v[4] += a[2 * j + 1].x; v[5] += a[2 * j + 1].y; v[6] += a[2 * j + 1].z; v[7] += a[2 * j + 1].w;
                    }
                }
                for (; o < nseg; ++o) {
                    const float4 a0 = __ldcg(q + (size_t)o * (kTile / 4)), a1 = __ldcg(q + (size_t)o * (kTile / 4) + 1);
                    v[0] += a0.x; v[1] += a0.y; v[2] += a0.z; v[3] += a0.w;
                    v[4] += a1.x; v[5] += a1.y; v[6] += a1.z; v[7] += a1.w;
                }
                const int64_t row = tt * kTile + 8 * lane;
                if (row + 8 <= N) {
                    uint4 pk;
                    pk.x = (uint32_t)f32_to_bf16(v[0]) | ((uint32_t)f32_to_bf16(v[1]) << 16);
                    pk.y = (uint32_t)f32_to_bf16(v[2]) | ((uint32_t)f32_to_bf16(v[3]) << 16);
                    pk.z = (uint32_t)f32_to_bf16(v[4]) | ((uint32_t)f32_to_bf16(v[5]) << 16);
                    pk.w = (uint32_t)f32_to_bf16(v[6]) | ((uint32_t)f32_to_bf16(v[7]) << 16);
                    *reinterpret_cast<uint4 *>(y + row) = pk;
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        if (row + j < N) y[row + j] = f32_to_bf16(v[j]);
                }
                __syncwarp();
                if (lane == 0) atomicExch(cnt + tt, 0);
            }
        }
        __syncthreads();
        return;
    }

    // ================================ consumers ================================
    if (n > 0) {
        const uint32_t dig_u32 = smem_u32(sm + L.dig), gfac_u32 = smem_u32(sm + L.gfac);
        // ---- digit planes of the groups this CTA touches: group (grp0 + j) mod G in slot j, x loads of a
        // warp's groups in batches of 4 ----
        const int nslots = min(n, G);
        for (int j0 = wid; j0 < nslots; j0 += 4 * kC) {
            uint4 xv[4];
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int j = j0 + b * kC;
                if (j < nslots) {
                    int gj = grp0 + j;
                    if (gj >= G) gj -= G;
                    xv[b] = *reinterpret_cast<const uint4 *>(x + (size_t)gj * 128 + 8 * (lane >> 1));
                }
            }
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int j = j0 + b * kC;
                if (j < nslots) make_digits8(xv[b], dig_u32 + (uint32_t)j * kDigitGroupBytes, gfac_u32 + (uint32_t)j * 4u, lane);
            }
        }
        named_bar_sync(1, kC * 32);

        const int gq = lane >> 2, tq = lane & 3;
        const uint32_t ring_u32 = smem_u32(ring);
        const int r0 = 16 * wid + gq;  // rows r0 and r0 + 8; r0 mod 8 = (r0 + 8) mod 8 = gq
        const bool bcol = gq < kDigits, ccol = 2 * tq < kDigits;
        const float cw0 = ccol ? exp2i(-14 * tq) : 0.0f, cw1 = ccol ? exp2i(-14 * tq - 7) : 0.0f;  // 128^-c
        const uint32_t cmag[4] = {kMagicBits, kMagicBits, kMagicBits, kMagicBits};
        // this lane's 32 codes of a row: 16-byte chunks 2 tq and 2 tq + 1, swizzled by the row (mod 8 = gq)
        const uint32_t a_lane0 = ring_u32 + (uint32_t)r0 * 128u + (uint32_t)(((2 * tq) ^ gq) * 16);
        const uint32_t a_lane1 = ring_u32 + (uint32_t)r0 * 128u + (uint32_t)(((2 * tq + 1) ^ gq) * 16);
        const uint32_t b_lane = dig_u32 + (uint32_t)(tq * (kDigits * 16) + gq * 16);
        float acc[2][2] = {{0.0f, 0.0f}, {0.0f, 0.0f}};
        int t = tile0, gg = grp0, seg_first = grp0;
        int pseg = 0, s = 0, di = 0;
        uint32_t ph = 0, w_off = 0;
        for (int i = 0; i < n; ++i) {
            mbar_wait(&full[s], ph, status, flags);
            uint4 wa[2], wb[2];  // rows r0, r0 + 8: codes 32 tq .. 32 tq + 31
            wa[0] = lds128(a_lane0 + w_off);
            wa[1] = lds128(a_lane1 + w_off);
            wb[0] = lds128(a_lane0 + w_off + 8u * 128u);
            wb[1] = lds128(a_lane1 + w_off + 8u * 128u);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            if (++s == kStages) { s = 0; ph ^= 1u; w_off = 0; } else { w_off += kStageBytes; }
            const uint32_t bsrc = b_lane + (uint32_t)di * kDigitGroupBytes;
            uint4 Bv[2];
#pragma unroll
            for (int hf = 0; hf < 2; ++hf)
                Bv[hf] = bcol ? lds128(bsrc + (uint32_t)(hf * 4) * (kDigits * 16)) : make_uint4(0u, 0u, 0u, 0u);
            uint32_t C[4];
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                // step w: codes 32 tq + 8 w .. + 3 (first word) and + 4 .. + 7 (second word) of each row
                const uint32_t a0 = word_of(wa[w >> 1], 2 * (w & 1)), a2 = word_of(wa[w >> 1], 2 * (w & 1) + 1);
                const uint32_t a1 = word_of(wb[w >> 1], 2 * (w & 1)), a3 = word_of(wb[w >> 1], 2 * (w & 1) + 1);
                const uint32_t b0 = word_of(Bv[w >> 1], (w & 1) * 2), b1 = word_of(Bv[w >> 1], (w & 1) * 2 + 1);
                mma_s8s8(C, w == 0 ? cmag : C, a0, a1, a2, a3, b0, b1);
            }
            const float F = lds_f32(gfac_u32 + (uint32_t)di * 4u);
            acc[0][0] = fmaf(F, __uint_as_float(C[0]) - kMagic, acc[0][0]);
            acc[0][1] = fmaf(F, __uint_as_float(C[1]) - kMagic, acc[0][1]);
            acc[1][0] = fmaf(F, __uint_as_float(C[2]) - kMagic, acc[1][0]);
            acc[1][1] = fmaf(F, __uint_as_float(C[3]) - kMagic, acc[1][1]);
            if (++di == G) di = 0;
            const bool tile_done = (gg + 1 == G);
            if (tile_done || i + 1 == n) {
                const int row0 = t * kTile + r0;
                // the row's scale multiplies its sum of columns (rows past N read row N - 1's scale)
                const float s0 = bf16_to_f32(sc[min(row0, N - 1)]), s1 = bf16_to_f32(sc[min(row0 + 8, N - 1)]);
                float rs[2];
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                    float v = fmaf(acc[a][1], cw1, acc[a][0] * cw0);
                    v += __shfl_xor_sync(0xffffffffu, v, 1);
                    v += __shfl_xor_sync(0xffffffffu, v, 2);
                    rs[a] = v * (a ? s1 : s0);
                    acc[a][0] = acc[a][1] = 0.0f;
                }
                if (seg_first == 0 && tile_done) {
                    if (tq == 0) {
                        if (row0 < N) y[row0] = f32_to_bf16(rs[0]);
                        if (row0 + 8 < N) y[row0 + 8] = f32_to_bf16(rs[1]);
                    }
                } else {
                    const int b = pseg & 1;
                    if (pseg >= 2) mbar_wait(&pempty[b], (uint32_t)((pseg >> 1) - 1) & 1u, status, flags);
                    if (tq == 0) {
                        part[b * kTile + r0] = rs[0];
                        part[b * kTile + r0 + 8] = rs[1];
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&pfull[b]);
                    ++pseg;
                }
            }
            if (++gg == G) { gg = 0; ++t; seg_first = 0; }
        }
    }
    __syncthreads();
}

struct W8Config {
    int grid, nslots;
    size_t smem;
};

W8Config w8m1_config(int64_t N, int64_t K)
{
    static std::mutex mu;
    static std::map<int, int> sms_of;
    int dev = 0;
    cudaGetDevice(&dev);
    int sms;
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = sms_of.find(dev);
        if (it == sms_of.end()) {
            int v = 148, o = 232448;
            cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
            cudaDeviceGetAttribute(&o, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
            cudaGetLastError();
            cudaFuncSetAttribute(gemv_w8a16_m1_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, o);
            cudaGetLastError();
            it = sms_of.emplace(dev, v).first;
        }
        sms = it->second;
    }
    const int64_t G = K / 128;
    const int64_t units = ((N + kTile - 1) / kTile) * G;
    W8Config c;
    c.grid = (int)std::max<int64_t>(1, std::min<int64_t>(units, sms));
    c.nslots = (int)std::min<int64_t>((units + c.grid - 1) / c.grid, G);
    c.smem = W8Layout(c.nslots).total;
    return c;
}

int w8m1_max_segments(int64_t N, int64_t K, int grid)
{
    const int64_t G = K / 128;
    const int64_t units = ((N + kTile - 1) / kTile) * G;
    const int64_t per = units / std::min<int64_t>(grid, units);
    return (int)std::min<int64_t>((G + per - 1) / per + 1, G);
}

size_t w8m1_slots_bytes(int64_t N, int64_t K, int grid)
{
    const int64_t ntiles = (N + kTile - 1) / kTile;
    return ((size_t)ntiles * w8m1_max_segments(N, K, grid) * kTile * 4 + 255) / 256 * 256;
}

}  // namespace

bool gemv_w8m1_eligible(int64_t M, int64_t N, int64_t K, int g)
{
    // per output channel; K % 128 for the units, K <= 65536 for the digit planes of 512 groups (worst case
    // 258 KB is never reached: a CTA holds at most its own share of groups, bounded below by the check)
    if (!(M == 1 && g == K && K >= 128 && K % 128 == 0 && K <= 65536 && N >= 1 && N <= 0x7fffffffLL)) return false;
    return W8Layout(w8m1_config(N, K).nslots).total <= 232448;
}

size_t gemv_w8m1_workspace_bytes(int64_t M, int64_t N, int64_t K, int g)
{
    if (!gemv_w8m1_eligible(M, N, K, g)) return 0;
    const int64_t ntiles = (N + kTile - 1) / kTile;
    return w8m1_slots_bytes(N, K, w8m1_config(N, K).grid) + ((size_t)ntiles * 4 + 255) / 256 * 256;
}

int launch_gemv_w8a16_m1(const uint16_t *x, int64_t N, int64_t K, const int8_t *q, const uint16_t *s, uint16_t *y,
                         void *workspace, int *status, cudaStream_t st)
{
    CUtensorMap wmap;
    // codes [N][K] bytes: boxes of 128 bytes x 256 rows, 128-byte swizzle
    if (!encode_tmap_2d(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, (uint64_t)K, (uint64_t)N, (uint64_t)K, 128, kTile,
                        CU_TENSOR_MAP_SWIZZLE_128B))
        return -1;
    const W8Config c = w8m1_config(N, K);
    const int max_segs = w8m1_max_segments(N, K, c.grid);
    uint8_t *w8 = static_cast<uint8_t *>(workspace);
    float *ws = reinterpret_cast<float *>(w8);
    int *cnt = reinterpret_cast<int *>(w8 + w8m1_slots_bytes(N, K, c.grid));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)c.grid);
    cfg.blockDim = dim3(kT);
    cfg.dynamicSmemBytes = c.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemv_w8a16_m1_kernel, wmap, x, s, (int)N, (int)K, y, ws, cnt, max_segs, status,
                              c.nslots) == cudaSuccess
               ? 0
               : -2;
}

}  // namespace wq

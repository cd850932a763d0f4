// wq_gemv_w8int.cu -- W8A16 per output channel at 1 <= M <= 8 activation
// rows: the decode step over symmetric INT8 weights, bound by streaming one
// byte per weight from HBM.
//
// "Quantization Methods Compared: INT8, GPTQ, AWQ, FP8, FP4 and KV-Cache
// Quantization", section "What quantisation does": symmetric absmax INT8,
// w_hat = s q with s = max |w| / 127 per output channel; section "Hardware,
// formats and the roofline": at decode batch sizes the step reads every
// weight once.
//
// The products are exact integer ones, as in the INT4 decode kernel
// (wq_gemv_m1.cu): each activation row is written once per CTA as 4 planes of
// radix-128 digits per group of 128 inputs (x_k = 2^(E_g - 5) sum_c d_ck
// 128^-c, |d| <= 64; exact for every |x_k| >= 2^(E_g - 19), the rest rounded
// to a multiple of 2^(E_g - 26)), and the codes q, signed bytes as stored,
// are the A operand of mma.sync m16n8k32 s8 x s8 -> s32 with no conversion at
// all.  The B operand's columns hold (row m, digit c) at column 4 m + c, 8 per
// MMA, so M rows take ceil(M / 2) MMAs per code word.  A lane's accumulator
// columns are two digits of one row: per group it adds
// 2^(E_g - 5) (D_c 128^-c + D_c+1 128^-(c+1)) (D = sum_k q_k d_k, exact) to
// that row's binary32 sum; the other two digits sit in the neighbouring lane,
// and s multiplies the row once per segment.
//
// Structure: a persistent grid, one CTA per SM; 16 consumer warps, a TMA
// producer warp and a combiner warp.  A unit is (256-row tile, group of 128
// inputs): one 32 KB stage, a 2-D box of 256 rows x 128 bytes loaded with the
// 128-byte swizzle (the 16-byte chunk c of row r lands at c ^ (r mod 8), so the
// consumers' 16-byte reads of two rows per quarter-warp do not collide).
// Stream-K over units, split tiles combined in segment order by the combiner
// warp, programmatic dependent launch, bounded waits -- all as in the INT4
// decode kernel.  Shapes whose digit planes do not fit shared memory with two
// stages go to the other W8A16 kernels.
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
constexpr int kMaxStages = 3;
constexpr uint32_t kStageBytes = kTile * 128;  // 256 rows x 128 codes
constexpr int kDigits = 4;
// digit planes of a group of 128 inputs for one 8-column tile: [half][t][column][16 B]; NT tiles per group
constexpr uint32_t kDigitGroupBytes = 2 * 4 * 8 * 16;
constexpr float kMagic = 12582912.0f;          // 1.5 * 2^23
constexpr uint32_t kMagicBits = 0x4B400000u;

// shared memory: [stages][2 partial tiles of M x 256][digit planes][group factors][barriers]
struct W8Layout {
    size_t part, dig, gfac, bar, total;
    __host__ __device__ W8Layout(int stages, int M, int NT, int nslots)
    {
        part = (size_t)stages * kStageBytes;
        dig = part + (size_t)2 * M * kTile * 4;
        gfac = dig + (size_t)nslots * kDigitGroupBytes * NT;
        bar = (gfac + (size_t)nslots * 16 * 4 + 7) & ~(size_t)7;
        total = bar + (2 * kMaxStages + 4 + 2) * 8 + 1024;
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

// Device-scope add with release semantics (no value returned): the writes that happen before it (this
// thread's, and through the preceding warp barrier the other lanes') are visible before the add is.
__device__ __forceinline__ void red_add_release(int *p, int v)
{
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Device-scope load with acquire semantics: later reads see what was written before the matching release.
__device__ __forceinline__ int ld_acquire(const int *p)
{
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
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
// cols: the columns of the group's tile layout (8 per tile); column 4 row + c holds digit c of that row, stored
// at (4 row + c) ^ 2 t so that the 8 lanes of a shared-memory phase (two columns, four quads) read 8 bank groups.
__device__ __forceinline__ void make_digits8(uint4 v, uint32_t dig_g, int cols, int row, uint32_t gfac_g, int lane)
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
    const uint32_t dst0 = dig_g + (uint32_t)(((half * 4 + t_) * cols) * 16 + (w & 1) * 8 + par * 4);
#pragma unroll
    for (int c = 0; c < kDigits; ++c) {
        const uint32_t lo = __byte_perm(t[0][c], t[1][c], 0x0040), hi = __byte_perm(t[2][c], t[3][c], 0x0040);
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(dst0 + (uint32_t)(((4 * row + c) ^ (2 * t_)) * 16)),
                     "r"(__byte_perm(lo, hi, 0x5410))
                     : "memory");
    }
    if (lane == 0) {
        const int ef = E - 5;
        float f = ef >= -126 ? exp2i(ef) : exp2i(ef + 64) * 5.421010862427522e-20f;  // 2^-64
        if (nonfinite) f = __int_as_float(0x7fc00000);                                 // NaN
        asm volatile("st.shared.f32 [%0], %1;" ::"r"(gfac_g), "f"(f) : "memory");
    }
}

// 18 warps put five on one SM sub-partition, whose register file holds 16K registers: at most 96 each.
template <int NT, int STAGES>
__global__ void __maxnreg__(96)
gemv_w8a16_int_kernel(const __grid_constant__ CUtensorMap wmap, const uint16_t *__restrict__ x,
                      const uint16_t *__restrict__ sc, int M, int N, int K, uint16_t *__restrict__ y,
                      float *__restrict__ ws, int *__restrict__ cnt, int max_segs, int *__restrict__ status,
                      int nslots_max)
{
    extern __shared__ __align__(1024) uint8_t w8_raw[];
    uint8_t *sm = w8_raw + ((1024u - (smem_u32(w8_raw) & 1023u)) & 1023u);
    const W8Layout L(STAGES, M, NT, nslots_max);
    uint8_t *ring = sm;
    float *part = reinterpret_cast<float *>(sm + L.part);  // [2][M][256 rows]
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L.bar);
    uint64_t *full = bars, *empty = bars + kMaxStages;
    uint64_t *pfull = bars + 2 * kMaxStages, *pempty = pfull + 2;
    volatile int *flags = reinterpret_cast<volatile int *>(pempty + 2);
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int G = K >> 7;  // groups (units) per tile

    pdl_launch_dependents();
    if (tid == 0) {
        for (int i = 0; i < STAGES; ++i) {
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
        for (; pi < STAGES && pi < n; ++pi) {
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
                const int s = i % STAGES;
                if (!mbar_wait(&empty[s], (uint32_t)(i / STAGES - 1) & 1u, status, flags)) break;
                mbar_arrive_expect_tx(&full[s], kStageBytes);
                tma_load_2d(ring + (uint32_t)s * kStageBytes, &wmap, &full[s], pg * 128, pt * kTile);
                if (++pg == G) { pg = 0; ++pt; }
            }
            for (int j = max(0, i - STAGES); j < i; ++j) wait_drain(&full[j % STAGES], (uint32_t)(j / STAGES) & 1u, status);
        }
        __syncthreads();
        return;
    }

    if (wid == kCombiner) {
        // ================================ combiner ================================
        // Split tiles in the consumers' order.  Lane l handles rows 8l .. 8l + 7 of the tile, for every m.
        int pseg = 0;
        for (int64_t tt = beg / G; tt * G < end; ++tt) {
            if (tt * G >= beg && tt * G + G <= end) continue;  // whole tile: the consumers wrote y
            const int b = pseg & 1;
            const bool ok = __all_sync(0xffffffffu, mbar_wait(&pfull[b], (uint32_t)(pseg >> 1) & 1u, status, flags));
            if (!ok) break;
            const int c_first = cta_of(tt * G, units, B);
            const int nseg = cta_of(tt * G + G - 1, units, B) - c_first + 1;
            float *slots = ws + (size_t)tt * max_segs * M * kTile;  // [segment][m][256]
            const float *src = part + (size_t)b * M * kTile + 8 * lane;
            ++pseg;
            // The CTA of the tile's first segment combines it: that segment ends its range (so it is this CTA's
            // last), while the tile's last segment starts the next CTA's.  The others copy their sums to their
            // slots and publish them with a release add (no round trip); the first keeps its own in the shared
            // tile and waits (bounded) until the counter shows the others.
            if (bid != c_first) {
                float *mine = slots + (size_t)(bid - c_first) * M * kTile + 8 * lane;
                for (int m = 0; m < M; ++m) {
                    const float4 v0 = *reinterpret_cast<const float4 *>(src + m * kTile);
                    const float4 v1 = *reinterpret_cast<const float4 *>(src + m * kTile + 4);
                    reinterpret_cast<float4 *>(mine + m * kTile)[0] = v0;
                    reinterpret_cast<float4 *>(mine + m * kTile)[1] = v1;
                }
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&pempty[b]);  // the shared tile is copied out: free it
                    red_add_release(cnt + tt, 1);
                }
                continue;
            }
            int arrived = 1;
            if (lane == 0) {
                const uint64_t t0 = global_ns();
                while (ld_acquire(cnt + tt) != nseg - 1) {
                    if (flags[0] != 0) { arrived = 0; break; }
                    if (global_ns() - t0 > kWaitLimitNs) {
                        record_timeout(status);
                        flags[0] = 1;
                        arrived = 0;
                        break;
                    }
                }
            }
            // the other lanes read the slots after lane 0's acquire (ordered by the warp barrier)
            if (!__shfl_sync(0xffffffffu, arrived, 0)) {
                if (lane == 0) mbar_arrive(&pempty[b]);
                break;
            }
            {
                // sum the segments in segment order, from 0: this CTA's own (segment 0, in the shared tile), then
                // the slots of the others
                const int64_t row = tt * kTile + 8 * lane;
                const size_t sstride = (size_t)M * (kTile / 4);  // float4 between segments
                for (int m = 0; m < M; ++m) {
                    const float4 s0 = *reinterpret_cast<const float4 *>(src + m * kTile);
                    const float4 s1 = *reinterpret_cast<const float4 *>(src + m * kTile + 4);
                    float v[8] = {0.0f + s0.x, 0.0f + s0.y, 0.0f + s0.z, 0.0f + s0.w,
                                  0.0f + s1.x, 0.0f + s1.y, 0.0f + s1.z, 0.0f + s1.w};
                    const float4 *q = reinterpret_cast<const float4 *>(slots + (size_t)m * kTile + 8 * lane);
                    int o = 1;
                    for (; o + 4 <= nseg; o += 4) {
                        float4 a[8];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            a[2 * j] = __ldcg(q + (size_t)(o + j) * sstride);
                            a[2 * j + 1] = __ldcg(q + (size_t)(o + j) * sstride + 1);
                        }
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            v[0] += a[2 * j].x; v[1] += a[2 * j].y; v[2] += a[2 * j].z; v[3] += a[2 * j].w;
                            v[4] += a[2 * j + 1].x; v[5] += a[2 * j + 1].y; v[6] += a[2 * j + 1].z; v[7] += a[2 * j + 1].w;
                        }
                    }
                    for (; o < nseg; ++o) {
                        const float4 a0 = __ldcg(q + (size_t)o * sstride), a1 = __ldcg(q + (size_t)o * sstride + 1);
                        v[0] += a0.x; v[1] += a0.y; v[2] += a0.z; v[3] += a0.w;
                        v[4] += a1.x; v[5] += a1.y; v[6] += a1.z; v[7] += a1.w;
                    }
                    uint16_t *yr = y + (size_t)m * N;
                    if (row + 8 <= N && (N & 7) == 0) {
                        uint4 pk;
                        pk.x = (uint32_t)f32_to_bf16(v[0]) | ((uint32_t)f32_to_bf16(v[1]) << 16);
                        pk.y = (uint32_t)f32_to_bf16(v[2]) | ((uint32_t)f32_to_bf16(v[3]) << 16);
                        pk.z = (uint32_t)f32_to_bf16(v[4]) | ((uint32_t)f32_to_bf16(v[5]) << 16);
                        pk.w = (uint32_t)f32_to_bf16(v[6]) | ((uint32_t)f32_to_bf16(v[7]) << 16);
                        *reinterpret_cast<uint4 *>(yr + row) = pk;
                    } else {
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            if (row + j < N) yr[row + j] = f32_to_bf16(v[j]);
                    }
                }
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&pempty[b]);  // the shared tile is summed: free it
                    atomicExch(cnt + tt, 0);
                }
            }
        }
        __syncthreads();
        return;
    }

    // ================================ consumers ================================
    if (n > 0) {
        const uint32_t dig_u32 = smem_u32(sm + L.dig), gfac_u32 = smem_u32(sm + L.gfac);
        constexpr int kCols = 8 * NT;  // digit columns per group: 4 per activation row
        const uint32_t slot_bytes = kDigitGroupBytes * NT;
        // ---- digit planes of (group, row) for the groups this CTA touches: group (grp0 + j) mod G in slot j;
        // a warp's jobs load x in batches of 4 before converting ----
        const int nslots = min(n, G);
        const int njobs = nslots * M;
        for (int j0 = wid; j0 < njobs; j0 += 4 * kC) {
            uint4 xv[4];
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int j = j0 + b * kC;
                if (j < njobs) {
                    const int js = j / M, m = j - js * M;
                    int gj = grp0 + js;
                    if (gj >= G) gj -= G;
                    xv[b] = *reinterpret_cast<const uint4 *>(x + (size_t)m * K + (size_t)gj * 128 + 8 * (lane >> 1));
                }
            }
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int j = j0 + b * kC;
                if (j < njobs) {
                    const int js = j / M, m = j - js * M;
                    make_digits8(xv[b], dig_u32 + (uint32_t)js * slot_bytes, kCols, m,
                                 gfac_u32 + (uint32_t)(js * 16 + m) * 4u, lane);
                }
            }
        }
        named_bar_sync(1, kC * 32);

        const int gq = lane >> 2, tq = lane & 3;
        const uint32_t ring_u32 = smem_u32(ring);
        const int r0 = 16 * wid + gq;  // rows r0 and r0 + 8; r0 mod 8 = (r0 + 8) mod 8 = gq
        // this lane's accumulator columns 2 tq, 2 tq + 1 of tile nt: row m = 2 nt + tq / 2, digits d, d + 1
        const int dlo = 2 * (tq & 1);
        const float cw0 = exp2i(-7 * dlo), cw1 = exp2i(-7 * dlo - 7);  // 128^-d, 128^-(d + 1)
        const uint32_t cmag[4] = {kMagicBits, kMagicBits, kMagicBits, kMagicBits};
        const uint32_t a_lane0 = ring_u32 + (uint32_t)r0 * 128u + (uint32_t)(((2 * tq) ^ gq) * 16);
        const uint32_t a_lane1 = ring_u32 + (uint32_t)r0 * 128u + (uint32_t)(((2 * tq + 1) ^ gq) * 16);
        float acc[2][NT];  // [row r0, r0 + 8][tile]: this lane's two digit columns of row 2 nt + tq / 2, weighted
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) acc[0][nt] = acc[1][nt] = 0.0f;
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
            if (++s == STAGES) { s = 0; ph ^= 1u; w_off = 0; } else { w_off += kStageBytes; }
            const uint32_t slot = dig_u32 + (uint32_t)di * slot_bytes;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int col = 8 * nt + gq;  // this lane's B column: row col / 4, digit col % 4
                const bool bok = (col >> 2) < M;
                uint4 Bv[2];
#pragma unroll
                for (int hf = 0; hf < 2; ++hf)
                    Bv[hf] = bok ? lds128(slot + (uint32_t)(((hf * 4 + tq) * kCols + (col ^ (2 * tq))) * 16))
                                 : make_uint4(0u, 0u, 0u, 0u);
                uint32_t C[4];
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const uint32_t a0 = word_of(wa[w >> 1], 2 * (w & 1)), a2 = word_of(wa[w >> 1], 2 * (w & 1) + 1);
                    const uint32_t a1 = word_of(wb[w >> 1], 2 * (w & 1)), a3 = word_of(wb[w >> 1], 2 * (w & 1) + 1);
                    const uint32_t b0 = word_of(Bv[w >> 1], (w & 1) * 2), b1 = word_of(Bv[w >> 1], (w & 1) * 2 + 1);
                    mma_s8s8(C, w == 0 ? cmag : C, a0, a1, a2, a3, b0, b1);
                }
                // C: (row r0, digit dlo), (r0, dlo + 1), (r0 + 8, dlo), (r0 + 8, dlo + 1) of activation row m
                const int m = 2 * nt + (tq >> 1);
                if (m < M) {
                    const float F = lds_f32(gfac_u32 + (uint32_t)(di * 16 + m) * 4u);
                    acc[0][nt] = fmaf(F, fmaf(__uint_as_float(C[1]) - kMagic, cw1, (__uint_as_float(C[0]) - kMagic) * cw0), acc[0][nt]);
                    acc[1][nt] = fmaf(F, fmaf(__uint_as_float(C[3]) - kMagic, cw1, (__uint_as_float(C[2]) - kMagic) * cw0), acc[1][nt]);
                }
            }
            if (++di == G) di = 0;
            const bool tile_done = (gg + 1 == G);
            if (tile_done || i + 1 == n) {
                const int row0 = t * kTile + r0;
                // the row's scale multiplies its sum (rows past N read row N - 1's scale)
                const float s0 = bf16_to_f32(sc[min(row0, N - 1)]), s1 = bf16_to_f32(sc[min(row0 + 8, N - 1)]);
                const int b = pseg & 1;
                const bool whole = (seg_first == 0 && tile_done);
                if (!whole && pseg >= 2) mbar_wait(&pempty[b], (uint32_t)((pseg >> 1) - 1) & 1u, status, flags);
                float *pb = part + (size_t)b * M * kTile;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    // the row's four digits: this lane's two and its neighbour's (tq ^ 1)
                    float v0 = acc[0][nt], v1 = acc[1][nt];
                    v0 += __shfl_xor_sync(0xffffffffu, v0, 1);
                    v1 += __shfl_xor_sync(0xffffffffu, v1, 1);
                    acc[0][nt] = acc[1][nt] = 0.0f;
                    const int m = 2 * nt + (tq >> 1);
                    if ((tq & 1) == 0 && m < M) {
                        if (whole) {
                            if (row0 < N) y[(size_t)m * N + row0] = f32_to_bf16(v0 * s0);
                            if (row0 + 8 < N) y[(size_t)m * N + row0 + 8] = f32_to_bf16(v1 * s1);
                        } else {
                            pb[m * kTile + r0] = v0 * s0;
                            pb[m * kTile + r0 + 8] = v1 * s1;
                        }
                    }
                }
                if (!whole) {
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
    int grid, nslots, stages;
    size_t smem;
};

int nt_of(int64_t M) { return M <= 2 ? 1 : M <= 4 ? 2 : 4; }

W8Config w8_config(int64_t M, int64_t N, int64_t K)
{
    static std::mutex mu;
    static std::map<int, std::pair<int, int>> dev_of;  // SMs, opt-in shared memory per block
    int dev = 0;
    cudaGetDevice(&dev);
    int sms, optin;
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = dev_of.find(dev);
        if (it == dev_of.end()) {
            // without a device (a workspace query on a build host) assume a B200: 148 SMs, 227 KB per block
            int v = 148, o = 232448;
            cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
            cudaDeviceGetAttribute(&o, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
            cudaGetLastError();
#define WQ_W8_ATTR(NT_, S_) cudaFuncSetAttribute(gemv_w8a16_int_kernel<NT_, S_>, cudaFuncAttributeMaxDynamicSharedMemorySize, o)
            WQ_W8_ATTR(1, 3); WQ_W8_ATTR(1, 2); WQ_W8_ATTR(2, 3); WQ_W8_ATTR(2, 2);
            WQ_W8_ATTR(4, 3); WQ_W8_ATTR(4, 2);
#undef WQ_W8_ATTR
            cudaGetLastError();
            it = dev_of.emplace(dev, std::make_pair(v, o)).first;
        }
        sms = it->second.first;
        optin = it->second.second;
    }
    const int64_t G = K / 128;
    const int64_t units = ((N + kTile - 1) / kTile) * G;
    const int NT = nt_of(M);
    W8Config c;
    c.grid = (int)std::max<int64_t>(1, std::min<int64_t>(units, sms));
    c.nslots = (int)std::min<int64_t>((units + c.grid - 1) / c.grid, G);
    c.stages = W8Layout(3, (int)M, NT, c.nslots).total <= (size_t)optin ? 3
               : W8Layout(2, (int)M, NT, c.nslots).total <= (size_t)optin ? 2
                                                                           : 0;
    c.smem = c.stages ? W8Layout(c.stages, (int)M, NT, c.nslots).total : 0;
    return c;
}

int w8_max_segments(int64_t N, int64_t K, int grid)
{
    const int64_t G = K / 128;
    const int64_t units = ((N + kTile - 1) / kTile) * G;
    const int64_t per = units / std::min<int64_t>(grid, units);
    return (int)std::min<int64_t>((G + per - 1) / per + 1, G);
}

size_t w8_slots_bytes(int64_t M, int64_t N, int64_t K, int grid)
{
    const int64_t ntiles = (N + kTile - 1) / kTile;
    return ((size_t)ntiles * w8_max_segments(N, K, grid) * M * kTile * 4 + 255) / 256 * 256;
}

}  // namespace

bool gemv_w8int_eligible(int64_t M, int64_t N, int64_t K, int g)
{
    // per output channel, 1 <= M <= 8 (at 16 rows, 8 MMAs per code word and the B loads of every warp made it
    // slower than the tensor-core kernel), K % 128 for the units; a CTA's digit planes and at least two stages
    // must fit shared memory
    if (!(M >= 1 && M <= 8 && g == K && K >= 128 && K % 128 == 0 && K <= 65536 && N >= 1 && N <= 0x7fffffffLL))
        return false;
    return w8_config(M, N, K).stages != 0;
}

size_t gemv_w8int_workspace_bytes(int64_t M, int64_t N, int64_t K, int g)
{
    if (!gemv_w8int_eligible(M, N, K, g)) return 0;
    const int64_t ntiles = (N + kTile - 1) / kTile;
    return counter_region_bytes(ntiles) + w8_slots_bytes(M, N, K, w8_config(M, N, K).grid);
}

int launch_gemv_w8a16_int(const uint16_t *x, int64_t M, int64_t N, int64_t K, const int8_t *q, const uint16_t *s,
                          uint16_t *y, void *workspace, int *status, cudaStream_t st)
{
    CUtensorMap wmap;
    // codes [N][K] bytes: boxes of 128 bytes x 256 rows, 128-byte swizzle
    if (!encode_tmap_2d(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, (uint64_t)K, (uint64_t)N, (uint64_t)K, 128, kTile,
                        CU_TENSOR_MAP_SWIZZLE_128B))
        return -1;
    const W8Config c = w8_config(M, N, K);
    const int max_segs = w8_max_segments(N, K, c.grid);
    const int64_t ntiles = (N + kTile - 1) / kTile;
    uint8_t *w8 = static_cast<uint8_t *>(workspace);
    int *cnt = reinterpret_cast<int *>(w8);
    float *ws = reinterpret_cast<float *>(w8 + counter_region_bytes(ntiles));
    if (clear_extra_counters(workspace, ntiles, st) != cudaSuccess) return -2;
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
    const int Mi = (int)M, Ni = (int)N, Ki = (int)K;
    cudaError_t e = cudaErrorInvalidValue;
#define WQ_W8_LAUNCH(NT_)                                                                                          \
    e = c.stages == 3 ? cudaLaunchKernelEx(&cfg, gemv_w8a16_int_kernel<NT_, 3>, wmap, x, s, Mi, Ni, Ki, y, ws, cnt,  \
                                           max_segs, status, c.nslots)                                              \
                      : cudaLaunchKernelEx(&cfg, gemv_w8a16_int_kernel<NT_, 2>, wmap, x, s, Mi, Ni, Ki, y, ws, cnt,  \
                                           max_segs, status, c.nslots)
    switch (nt_of(M)) {
    case 1: WQ_W8_LAUNCH(1); break;
    case 2: WQ_W8_LAUNCH(2); break;
    default: WQ_W8_LAUNCH(4); break;
    }
#undef WQ_W8_LAUNCH
    return e == cudaSuccess ? 0 : -2;
}

}  // namespace wq

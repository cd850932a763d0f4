// wq_gemv_i4mt.cu -- W4A16, group 128, M = 2 activation rows on the
// integer products of the M = 1 kernel (wq_gemv_m1.cu): the decode step at a
// small batch, bound by streaming the packed weights from HBM once.
//
// "Quantization Methods Compared: INT8, GPTQ, AWQ, FP8, FP4 and KV-Cache
// Quantization", section "Hardware, formats and the roofline": at decode
// batch sizes one pass over the weights serves every row.  w_hat = s (q - z)
// ("Quantization for LLM inference: FP8, INT4 (GPTQ, AWQ) and GGUF", "The
// minimum maths").
//
// (The kernel is written for up to 8 rows -- NT column tiles -- but at 3 to 8 rows, with 2 or 4 MMAs per code
// word, the bf16 small-batch kernel measured faster, so only NT = 1 is instantiated.)
// Everything is the M = 1 kernel's -- weight stream, s/z windows, stream-K,
// combiner warp, programmatic dependent launch, bounded waits, exact integer
// products s (sum_k q_k x_k - z sum_k x_k) with x as 4 planes of radix-128
// digits per group -- except that each of the M rows has its own digit planes
// and the B operand's 8 columns hold (row m, digit c) at column 4 m + c: M rows
// take ceil(M / 2) MMAs per code word.  A lane's two accumulator columns are
// two digits of one row, folded per group as s 2^(E_mg - 5) ((D_c - z S_mc)
// 128^-c + (D_c+1 - z S_mc+1) 128^-(c+1)); the neighbouring lane holds the
// other two digits.  Shapes whose digit planes do not fit shared memory with
// two stages take the bf16 small-batch kernel (wq_gemv_mt.cu).

#include "wq_common.cuh"
#include "wq_internal.h"
#include "wq_sm100.cuh"

#include <algorithm>
#include <map>
#include <mutex>

namespace wq {

namespace {

constexpr int kC = 16;                            // consumer warps
constexpr int kProducer = kC;                     // warp roles: consumers 0 .. kC-1, then these two
constexpr int kCombiner = kC + 1;
constexpr int kT = (kC + 2) * 32;                 // threads
constexpr int kTile = 16 * kC;                    // rows per tile (256)
constexpr int kMaxStages = 3;                     // weight stages in flight (2 for the longest K)
constexpr uint32_t kStageBytes = kTile * 128;     // 256 rows x 2 groups x 64 B
constexpr uint32_t kSzBytes = kTile * 16;         // 256 rows x 8 groups x 2 B (one of s or z)
constexpr int kPairsPerWindow = 4;                // 8 groups of s/z = 4 units
constexpr int kDigits = 4;                        // radix-128 digit planes of x
// digit planes of a group pair: [group][half][t][column (8 per tile of two rows)][16 B]; column j of quad t
// is stored at j ^ 2 t, so the 8 lanes of a shared-memory phase (two columns, four quads) read 8 bank groups
constexpr float kMagic = 12582912.0f;             // 1.5 * 2^23
constexpr uint32_t kMagicBits = 0x4B400000u;

// shared memory: [stages][s/z windows][2 partial tiles][digit planes][S sums][group factors][barriers]
struct M1Layout {
    size_t sz, part, dig, gsum, gfac, bar, total;
    __host__ __device__ M1Layout(int stages, int M, int npairs)
    {
        sz = (size_t)stages * kStageBytes;
        part = sz + 2 * 2 * kSzBytes;
        dig = part + (size_t)2 * M * kTile * 4;
        gsum = dig + (size_t)npairs * 2048 * (M <= 2 ? 1 : M <= 4 ? 2 : 4);
        gfac = gsum + (size_t)npairs * 2 * M * kDigits * 4;
        bar = (gfac + (size_t)npairs * 2 * M * 4 + 7) & ~(size_t)7;
        total = bar + (2 * kMaxStages + 4 + 4 + 2) * 8 + 1024;
    }
};

// D += A B for one m16n8k32 step (A unsigned bytes, B signed bytes, exact 32-bit integer accumulation), with the
// accumulator's input given separately.
__device__ __forceinline__ void mma_u8s8(uint32_t d[4], const uint32_t c[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%10, %11, %12, %13};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(c[0]), "r"(c[1]), "r"(c[2]), "r"(c[3]));
}

__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar, int x, int y, int z)
{
    asm volatile("cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];"
                 :: "r"(smem_u32(dst)), "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
                 : "memory");
}

// Programmatic dependent launch: let the next kernel in the stream start launching now, and wait until
// the previous kernel has completed and its writes are visible (no-ops for a normal launch).
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ uint4 lds128(uint32_t addr)
{
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(addr));
    return r;
}

__device__ __forceinline__ uint32_t lds_u32(uint32_t addr)
{
    uint32_t r;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(r) : "r"(addr));
    return r;
}

__device__ __forceinline__ float2 lds_f2(uint32_t addr)
{
    float2 r;
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(r.x), "=f"(r.y) : "r"(addr));
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

// Device-scope add with acquire-release semantics: orders the writes that happen before it (this thread's,
// and through the preceding CTA barrier the other consumers') before the add, and later reads after it.
__device__ __forceinline__ int atom_add_acq_rel(int *p, int v)
{
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// The CTA whose equal share [units * b / B, units * (b + 1) / B) holds unit u.
__host__ __device__ __forceinline__ int cta_of(int64_t u, int64_t units, int64_t B)
{
    return (int)(((u + 1) * B - 1) / units);
}

// Eight activations divided by their input channels' scales: bf16(x / s) with an IEEE binary32 quotient
// (the activation side of per-input-channel scaling, wq_gemm_w4a16_colscaled).
__device__ __forceinline__ uint4 colscale8(uint4 v, const float *s)
{
    const float4 s0 = __ldg(reinterpret_cast<const float4 *>(s)), s1 = __ldg(reinterpret_cast<const float4 *>(s) + 1);
    const float sc[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
        w[i] = pack_bf16x2(__fdiv_rn(__uint_as_float(w[i] << 16), sc[2 * i]),
                           __fdiv_rn(__uint_as_float(w[i] & 0xffff0000u), sc[2 * i + 1]));
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Bounded wait used on the drain path (ignores the abort flag).
__device__ __forceinline__ void wait_drain(uint64_t *bar, uint32_t parity, int *status)
{
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_ns() - t0 > kWaitLimitNs) { record_timeout(status); return; }
}

// 2^e as binary32 for e in [-126, 127].
__device__ __forceinline__ float exp2i(int e) { return __uint_as_float((uint32_t)(e + 127) << 23); }

// The digit planes, column sums and scale factor of one group of one row of x (one warp).  Lane L holds word
// L / 2 of the group (inputs 8 (L / 2) .. + 7, loaded by the caller) and takes of it the inputs of parity L % 2:
// 2 i + L % 2, i = 0 .. 3, the byte order of the A operand's even (L % 2 = 0) and odd code words.
// cols = 8 NT columns per (group, half, t); column 4 row + c holds digit c of that row, stored at (4 row + c) ^ 2 t.
__device__ __forceinline__ void make_digits(uint4 v, const float *__restrict__ csg, uint32_t dig_pair, int cols,
                                            int row, uint32_t gsum_g, uint32_t gfac_g, int h, int lane)
{
    const int wq_ = lane >> 1, par = lane & 1;
    if (csg) v = colscale8(v, csg + 8 * wq_);
    float e[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t wd = word_of(v, i);
        e[i] = __uint_as_float(par ? (wd & 0xffff0000u) : (wd << 16));
    }
    float m = fmaxf(fmaxf(fabsf(e[0]), fabsf(e[1])), fmaxf(fabsf(e[2]), fabsf(e[3])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    // an infinite or NaN activation makes the group's factor NaN, so y is not finite, as x * w_hat would be
    const bool nonfinite = __any_sync(0xffffffffu, !(fabsf(e[0]) < INFINITY && fabsf(e[1]) < INFINITY &&
                                                     fabsf(e[2]) < INFINITY && fabsf(e[3]) < INFINITY));
    if (nonfinite) m = 0.0f;
    // 2^E <= m < 2^(E + 1); a group of zeros gets E = 0 (all digits 0)
    int E = m > 0.0f ? (int)((__float_as_uint(m) >> 23) & 0xff) - 127 : 0;
    if (m > 0.0f && E == -127) E = -127 + (31 - __clz((int)(__float_as_uint(m) & 0x7fffff))) - 22;  // subnormal
    // X = x 2^(5 - E) in (-64, 64), applied in two exact power-of-two steps
    const int a1 = (5 - E) / 2, a2 = (5 - E) - a1;
    const float sc1 = exp2i(a1), sc2 = exp2i(a2);
    uint32_t t[4][kDigits];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float X = (e[i] * sc1) * sc2;
#pragma unroll
        for (int c = 0; c < kDigits; ++c) {
            const float tt = X + kMagic;            // the nearest integer sits in the low bits
            t[i][c] = __float_as_uint(tt);
            X = (X - (tt - kMagic)) * 128.0f;      // exact
        }
    }
    const int t_ = wq_ >> 2, w = wq_ & 3, half = w >> 1;
    const uint32_t dst0 = dig_pair + (uint32_t)((((h * 2 + half) * 4 + t_) * cols) * 16 + (w & 1) * 8 + par * 4);
#pragma unroll
    for (int c = 0; c < kDigits; ++c) {
        const uint32_t lo = __byte_perm(t[0][c], t[1][c], 0x0040), hi = __byte_perm(t[2][c], t[3][c], 0x0040);
        const uint32_t packed = __byte_perm(lo, hi, 0x5410);
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(dst0 + (uint32_t)(((4 * row + c) ^ (2 * t_)) * 16)), "r"(packed)
                     : "memory");
        // the digit values (wrapping 32-bit arithmetic: the four magic offsets cancel)
        const int sum = (int)(t[0][c] + t[1][c] + t[2][c] + t[3][c] - 4u * kMagicBits);
        const int tot = __reduce_add_sync(0xffffffffu, sum);
        if (lane == 0) asm volatile("st.shared.f32 [%0], %1;" ::"r"(gsum_g + (uint32_t)c * 4u), "f"((float)tot) : "memory");
    }
    // weight of digit 0: 2^(E - 5) (binary32 loses precision only below 2^-126)
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
gemv_w4a16_i4mt_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap smap,
                       const __grid_constant__ CUtensorMap zmap, const uint16_t *__restrict__ x, int M, int N, int K,
                     uint16_t *__restrict__ y, float *__restrict__ ws, int *__restrict__ cnt, int max_segs,
                     int *__restrict__ status, int npairs, const float *__restrict__ col_scale)
{
    extern __shared__ __align__(1024) uint8_t i4_raw[];
    // TMA destinations want 128-byte (we keep 1024-byte) alignment: align the base explicitly
    uint8_t *sm = i4_raw + ((1024u - (smem_u32(i4_raw) & 1023u)) & 1023u);
    const M1Layout L(STAGES, M, npairs);
    uint8_t *ring = sm;
    uint8_t *szr = sm + L.sz;                                     // [2 windows][s, z][256 rows][8 groups]
    float *part = reinterpret_cast<float *>(sm + L.part);         // [2][M][256 rows] partial sums
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L.bar);
    uint64_t *full = bars, *empty = bars + kMaxStages;
    uint64_t *szfull = bars + 2 * kMaxStages, *szempty = szfull + 2;
    uint64_t *pfull = szempty + 2, *pempty = pfull + 2;
    volatile int *flags = reinterpret_cast<volatile int *>(pempty + 2);  // [0] abort, [1] unused
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int G = K >> 7;
    const int P = G >> 1;  // group pairs (units) per tile

    pdl_launch_dependents();
    if (tid == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kC);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&szfull[i], 1);
            mbar_init(&szempty[i], kC);
            mbar_init(&pfull[i], kC);
            mbar_init(&pempty[i], 1);
        }
        flags[0] = 0;
        flags[1] = 0;
        fence_mbar_init();
    }
    __syncthreads();

    // ---- this CTA's equal share of the units ----
    const int ntiles = (N + kTile - 1) / kTile;
    const int64_t units = (int64_t)ntiles * P;
    const int64_t B = min((int64_t)gridDim.x, units);  // participating CTAs, each with >= 1 unit
    const int64_t bid = blockIdx.x;
    const int64_t beg = bid < B ? units * bid / B : units, end = bid < B ? units * (bid + 1) / B : units;
    const int n = (int)(end - beg);  // a CTA's share stays far below 2^31
    const int tile0 = (int)(beg / P), pair0 = (int)(beg - (int64_t)tile0 * P);

    // Under programmatic dependent launch the previous kernel may still be running.  Nothing it writes may
    // be read before pdl_wait().  The packed weights, scales and zero-points are inputs that the preceding
    // call does not write (a call of this kernel writes only y and its workspace; the library's other
    // kernels do not launch dependents early), so the producer issues the first stages and the first s/z
    // window into shared memory now; only the activations wait.  (Requesting further units into L2 here as
    // well made a stream of linears slower: 8 units per CTA cost 9%.)
    int pt = tile0, pp = pair0;  // producer position: tile, group pair
    int wins = 0;                // s/z windows issued
    int pi = 0;                  // stages issued
    auto issue_window = [&](int slot) {
        mbar_arrive_expect_tx(&szfull[slot], 2 * kSzBytes);
        uint8_t *d = szr + (uint32_t)slot * 2u * kSzBytes;
        const int g8 = (2 * pp) & ~7;
        tma_load_2d(d, &smap, &szfull[slot], g8, pt * kTile);
        tma_load_2d(d + kSzBytes, &zmap, &szfull[slot], g8, pt * kTile);
        ++wins;
    };
    if (wid == kProducer && lane == 0) {
        // at most two windows start within the first STAGES pairs, so no window slot needs a wait here
        for (; pi < STAGES && pi < n; ++pi) {
            if (pi == 0 || (pp & (kPairsPerWindow - 1)) == 0) issue_window(wins & 1);
            mbar_arrive_expect_tx(&full[pi], kStageBytes);
            tma_load_3d(ring + (uint32_t)pi * kStageBytes, &wmap, &full[pi], 0, pt * kTile, 2 * pp);
            if (++pp == P) { pp = 0; ++pt; }
        }
    }
    pdl_wait();

    if (wid == kProducer) {
        // ================================ producer ================================
        if (lane == 0 && n > 0) {
            int i = pi;
            for (; i < n; ++i) {
                // s/z window: at every 4th pair of a tile
                if ((pp & (kPairsPerWindow - 1)) == 0) {
                    const int slot = wins & 1;
                    if (wins >= 2 && !mbar_wait(&szempty[slot], (uint32_t)((wins >> 1) - 1) & 1u, status, flags)) break;
                    issue_window(slot);
                }
                const int s = i % STAGES;
                if (!mbar_wait(&empty[s], (uint32_t)(i / STAGES - 1) & 1u, status, flags)) break;
                mbar_arrive_expect_tx(&full[s], kStageBytes);
                tma_load_3d(ring + (uint32_t)s * kStageBytes, &wmap, &full[s], 0, pt * kTile, 2 * pp);
                if (++pp == P) { pp = 0; ++pt; }
            }
            // drain: the copies issued last must land before the CTA can end (bounded, ignores abort)
            for (int j = max(0, i - STAGES); j < i; ++j) wait_drain(&full[j % STAGES], (uint32_t)(j / STAGES) & 1u, status);
            for (int j = max(0, wins - 2); j < wins; ++j) wait_drain(&szfull[j & 1], (uint32_t)(j >> 1) & 1u, status);
        }
        __syncthreads();
        return;
    }

    if (wid == kCombiner) {
        // ================================ combiner ================================
        // Split tiles in the consumers' order.  Lane l handles rows 8l .. 8l + 7 of the tile, for every m.
        int pseg = 0;
        for (int64_t tt = beg / P; tt * P < end; ++tt) {
            if (tt * P >= beg && tt * P + P <= end) continue;  // whole tile: the consumers wrote y
            const int b = pseg & 1;
            const bool ok = __all_sync(0xffffffffu, mbar_wait(&pfull[b], (uint32_t)(pseg >> 1) & 1u, status, flags));
            if (!ok) break;
            const int c_first = cta_of(tt * P, units, B);
            const int nseg = cta_of(tt * P + P - 1, units, B) - c_first + 1;
            float *slots = ws + (size_t)tt * max_segs * M * kTile;  // [segment][m][256]
            float *mine = slots + (size_t)(bid - c_first) * M * kTile + 8 * lane;
            const float *src = part + (size_t)b * M * kTile + 8 * lane;
            for (int m = 0; m < M; ++m) {
                const float4 v0 = *reinterpret_cast<const float4 *>(src + m * kTile);
                const float4 v1 = *reinterpret_cast<const float4 *>(src + m * kTile + 4);
                reinterpret_cast<float4 *>(mine + m * kTile)[0] = v0;
                reinterpret_cast<float4 *>(mine + m * kTile)[1] = v1;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&pempty[b]);  // the shared tile is copied out: free it
            ++pseg;
            int last = 0;
            if (lane == 0) last = (atom_add_acq_rel(cnt + tt, 1) + 1 == nseg) ? 1 : 0;
            last = __shfl_sync(0xffffffffu, last, 0);
            if (last) {
                // sum the segments' slots in segment order (independent of which CTA arrived last)
                const int64_t row = tt * kTile + 8 * lane;
                const size_t sstride = (size_t)M * (kTile / 4);  // float4 between segments
                for (int m = 0; m < M; ++m) {
                    float v[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
                    const float4 *q = reinterpret_cast<const float4 *>(slots + (size_t)m * kTile + 8 * lane);
                    int o = 0;
                    for (; o + 4 <= nseg; o += 4) {
                        float4 a4[8];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            a4[2 * j] = __ldcg(q + (size_t)(o + j) * sstride);
                            a4[2 * j + 1] = __ldcg(q + (size_t)(o + j) * sstride + 1);
                        }
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            v[0] += a4[2 * j].x; v[1] += a4[2 * j].y; v[2] += a4[2 * j].z; v[3] += a4[2 * j].w;
                            v[4] += a4[2 * j + 1].x; v[5] += a4[2 * j + 1].y; v[6] += a4[2 * j + 1].z; v[7] += a4[2 * j + 1].w;
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
                if (lane == 0) atomicExch(cnt + tt, 0);
            }
        }
        __syncthreads();
        return;
    }

    // ================================ consumers ================================
    if (n > 0) {
        const uint32_t dig_u32 = smem_u32(sm + L.dig), gsum_u32 = smem_u32(sm + L.gsum), gfac_u32 = smem_u32(sm + L.gfac);
        constexpr int cols = 8 * NT;                  // digit columns per (group, half, t)
        constexpr uint32_t pair_bytes = 2048u * NT;
        // ---- digit planes of (group, row) for the group pairs this CTA touches: pair (pair0 + j) mod P in
        // slot j ----
        // a warp's jobs load their x words in batches of 4 before any is converted
        const int nslots = min(n, P);
        const int njobs = 2 * nslots * M;
        for (int j0 = wid; j0 < njobs; j0 += 4 * kC) {
            uint4 xv[4];
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int j = j0 + b * kC;
                if (j < njobs) {
                    const int m = j % M, jh = j / M, js = jh >> 1, h = jh & 1;
                    int pj = pair0 + js;
                    if (pj >= P) pj -= P;
                    xv[b] = *reinterpret_cast<const uint4 *>(x + (size_t)m * K + (size_t)(2 * pj + h) * 128 +
                                                             8 * (lane >> 1));
                }
            }
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int j = j0 + b * kC;
                if (j < njobs) {
                    const int m = j % M, jh = j / M, js = jh >> 1, h = jh & 1;
                    int pj = pair0 + js;
                    if (pj >= P) pj -= P;
                    const int kg = 2 * pj + h;
                    make_digits(xv[b], col_scale ? col_scale + (size_t)kg * 128 : nullptr,
                                dig_u32 + (uint32_t)js * pair_bytes, cols, m,
                                gsum_u32 + (uint32_t)(((js * 2 + h) * M + m) * kDigits) * 4u,
                                gfac_u32 + (uint32_t)((js * 2 + h) * M + m) * 4u, h, lane);
                }
            }
        }
        named_bar_sync(1, kC * 32);

        const int gq = lane >> 2, tq = lane & 3;
        const uint32_t ring_u32 = smem_u32(ring), szr_u32 = smem_u32(szr);
        const int r0 = 16 * wid + gq;  // this lane's rows in the tile: r0 and r0 + 8
        // accumulator columns 2 tq, 2 tq + 1 of tile nt: row 2 nt + tq / 2, digits dlo, dlo + 1
        const int dlo = 2 * (tq & 1);
        const float cw0 = exp2i(-7 * dlo), cw1 = exp2i(-7 * dlo - 7);  // 128^-c
        float acc[2][NT];  // [row r0, r0 + 8][tile]
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) acc[0][nt] = acc[1][nt] = 0.0f;
        const uint32_t cmag[4] = {kMagicBits, kMagicBits, kMagicBits, kMagicBits};
        int t = tile0, p = pair0, seg_first = pair0;
        int win = -1;
        int pseg = 0;  // partial segments handed to the combiner
        int s = 0;     // stage slot of unit i, and the parity of its fill
        int di = 0;    // digit slot of pair p
        uint32_t ph = 0, w_off = 0;
        const uint32_t w_lane = ring_u32 + (uint32_t)r0 * 64u + (uint32_t)tq * 16u;
        const uint32_t sz_lane = szr_u32 + (uint32_t)r0 * 16u;
        // A wait that runs out sets the abort flag and every later wait returns at once: the loop then runs
        // to its end on garbage, with the same control flow in every warp, so the barriers below still meet.
        for (int i = 0; i < n; ++i) {
            // ---- s/z window ----
            if (i == 0 || (p & (kPairsPerWindow - 1)) == 0) {
                if (win >= 0) {  // the previous window is consumed
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&szempty[win & 1]);
                }
                ++win;
                mbar_wait(&szfull[win & 1], (uint32_t)(win >> 1) & 1u, status, flags);
            }
            mbar_wait(&full[s], ph, status, flags);
            const uint32_t wsrc = w_lane + w_off;
            uint4 wv[2][2];  // [group h][row r0, row r0 + 8]
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int a = 0; a < 2; ++a) wv[h][a] = lds128(wsrc + (uint32_t)h * (kTile * 64u) + (uint32_t)a * 8u * 64u);
            const int kg = 2 * p;
            const uint32_t szsrc = sz_lane + (uint32_t)(win & 1) * 2u * kSzBytes + (uint32_t)(kg & 7) * 2u;
            float sv[2][2], zv[2][2];
#pragma unroll
            for (int a = 0; a < 2; ++a) {
                const uint32_t o = szsrc + (uint32_t)a * 8u * 16u;
                const uint32_t s2 = lds_u32(o), z2 = lds_u32(o + kSzBytes);
                sv[0][a] = __uint_as_float(s2 << 16);
                sv[1][a] = __uint_as_float(s2 & 0xffff0000u);
                zv[0][a] = __uint_as_float(z2 << 16);
                zv[1][a] = __uint_as_float(z2 & 0xffff0000u);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            if (++s == STAGES) { s = 0; ph ^= 1u; w_off = 0; } else { w_off += kStageBytes; }
            const uint32_t slot = dig_u32 + (uint32_t)di * pair_bytes;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                // the A operand of the group's four k32 steps: even and odd codes as unsigned bytes
                uint32_t Alo[4][2], Ahi[4][2];
#pragma unroll
                for (int w = 0; w < 4; ++w)
#pragma unroll
                    for (int a = 0; a < 2; ++a) {
                        const uint32_t v = word_of(wv[h][a], w);
                        Alo[w][a] = v & 0x0F0F0F0Fu;
                        Ahi[w][a] = (v >> 4) & 0x0F0F0F0Fu;
                    }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int col = 8 * nt + gq;  // this lane's B column: row col / 4, digit col % 4
                    const bool bok = col < 4 * M;
                    uint4 Bv[2];
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf)
                        Bv[hf] = bok ? lds128(slot + (uint32_t)((((h * 2 + hf) * 4 + tq) * cols + (col ^ (2 * tq))) * 16))
                                     : make_uint4(0u, 0u, 0u, 0u);
                    uint32_t C[4];
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const uint32_t b0 = word_of(Bv[w >> 1], (w & 1) * 2), b1 = word_of(Bv[w >> 1], (w & 1) * 2 + 1);
                        mma_u8s8(C, w == 0 ? cmag : C, Alo[w][0], Alo[w][1], Ahi[w][0], Ahi[w][1], b0, b1);
                    }
                    // C: (row r0, digit dlo), (r0, dlo + 1), (r0 + 8, dlo), (r0 + 8, dlo + 1) of activation row m
                    const int m = 2 * nt + (tq >> 1);
                    if (m < M) {
                        const int gi = (di * 2 + h) * M + m;
                        const float2 S = lds_f2(gsum_u32 + (uint32_t)(gi * kDigits + dlo) * 4u);
                        const float F = lds_f32(gfac_u32 + (uint32_t)gi * 4u);
#pragma unroll
                        for (int a = 0; a < 2; ++a) {
                            const float d0 = fmaf(-zv[h][a], S.x, __uint_as_float(C[2 * a]) - kMagic);
                            const float d1 = fmaf(-zv[h][a], S.y, __uint_as_float(C[2 * a + 1]) - kMagic);
                            acc[a][nt] = fmaf(sv[h][a] * F, fmaf(d1, cw1, d0 * cw0), acc[a][nt]);
                        }
                    }
                }
            }
            if (++di == P) di = 0;
            // ---- end of a segment: the tile's last pair, or the end of this CTA's range ----
            const bool tile_done = (p + 1 == P);
            if (tile_done || i + 1 == n) {
                const int row0 = t * kTile + r0;
                const bool whole = (seg_first == 0 && tile_done);
                const int b = pseg & 1;
                if (!whole && pseg >= 2) mbar_wait(&pempty[b], (uint32_t)((pseg >> 1) - 1) & 1u, status, flags);
                float *pb = part + (size_t)b * M * kTile;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    // the row's four digit columns: this lane's two and its neighbour's (tq ^ 1)
                    float v0 = acc[0][nt], v1 = acc[1][nt];
                    v0 += __shfl_xor_sync(0xffffffffu, v0, 1);
                    v1 += __shfl_xor_sync(0xffffffffu, v1, 1);
                    acc[0][nt] = acc[1][nt] = 0.0f;
                    const int m = 2 * nt + (tq >> 1);
                    if ((tq & 1) == 0 && m < M) {
                        if (whole) {
                            if (row0 < N) y[(size_t)m * N + row0] = f32_to_bf16(v0);
                            if (row0 + 8 < N) y[(size_t)m * N + row0 + 8] = f32_to_bf16(v1);
                        } else {
                            pb[m * kTile + r0] = v0;
                            pb[m * kTile + r0 + 8] = v1;
                        }
                    }
                }
                if (!whole) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&pfull[b]);
                    ++pseg;
                }
            }
            if (++p == P) { p = 0; ++t; seg_first = 0; }
        }
    }
    __syncthreads();
}

// Launch parameters per (device, M, N, K): grid (one CTA per SM, fewer when there is less work), the digit
// slots a CTA needs, the stage count that fits shared memory (0: the shape does not fit).
struct I4Config {
    int grid, npairs, stages;
    size_t smem;
};

I4Config i4_config(int64_t M, int64_t N, int64_t K)
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
#define WQ_I4_ATTR(NT_, S_) cudaFuncSetAttribute(gemv_w4a16_i4mt_kernel<NT_, S_>, cudaFuncAttributeMaxDynamicSharedMemorySize, o)
            WQ_I4_ATTR(1, 3); WQ_I4_ATTR(1, 2);
#undef WQ_I4_ATTR
            cudaGetLastError();
            it = dev_of.emplace(dev, std::make_pair(v, o)).first;
        }
        sms = it->second.first;
        optin = it->second.second;
    }
    const int64_t P = K / 256;
    const int64_t units = ((N + kTile - 1) / kTile) * P;
    I4Config c;
    c.grid = (int)std::max<int64_t>(1, std::min<int64_t>(units, sms));
    c.npairs = (int)std::min<int64_t>((units + c.grid - 1) / c.grid, P);
    c.stages = M1Layout(3, (int)M, c.npairs).total <= (size_t)optin ? 3
               : M1Layout(2, (int)M, c.npairs).total <= (size_t)optin ? 2
                                                                       : 0;
    c.smem = c.stages ? M1Layout(c.stages, (int)M, c.npairs).total : 0;
    return c;
}

int i4_max_segments(int64_t N, int64_t K, int grid)
{
    const int64_t P = K / 256;
    const int64_t units = ((N + kTile - 1) / kTile) * P;
    const int64_t per = units / std::min<int64_t>(grid, units);
    return (int)std::min<int64_t>((P + per - 1) / per + 1, P);
}

size_t i4_slots_bytes(int64_t M, int64_t N, int64_t K, int grid)
{
    const int64_t ntiles = (N + kTile - 1) / kTile;
    return ((size_t)ntiles * i4_max_segments(N, K, grid) * M * kTile * 4 + 255) / 256 * 256;
}

}  // namespace

bool gemv_i4mt_eligible(int64_t M, int64_t N, int64_t K, int g)
{
    // M = 2 only: at 3 to 8 rows (2 or 4 MMAs per code word) the bf16 small-batch kernel measured faster.
    // K % 1024: the s/z row stride must be a multiple of 16 bytes for their tensor maps; a CTA's digit planes
    // and at least two stages must fit shared memory
    if (!(M == 2 && g == 128 && K >= 1024 && K % 1024 == 0 && K <= 32768 && N >= 1 && N <= 0x7fffffffLL))
        return false;
    return i4_config(M, N, K).stages != 0;
}

size_t gemv_i4mt_workspace_bytes(int64_t M, int64_t N, int64_t K, int g)
{
    if (!gemv_i4mt_eligible(M, N, K, g)) return 0;
    const int64_t ntiles = (N + kTile - 1) / kTile;
    return counter_region_bytes(ntiles) + i4_slots_bytes(M, N, K, i4_config(M, N, K).grid);
}

int launch_gemv_w4a16_i4mt(const uint16_t *x, int64_t M, int64_t N, int64_t K, const uint8_t *q, const uint16_t *s,
                           const uint16_t *z, uint16_t *y, void *workspace, int *status, cudaStream_t st,
                           const float *col_scale)
{
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qr) != cudaSuccess ||
            qr != cudaDriverEntryPointSuccess || fn == nullptr)
            return -1;
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    CUtensorMap wmap, smap, zmap;
    const uint64_t G = (uint64_t)K / 128;
    cuuint64_t dims[3] = {64, (cuuint64_t)N, G};
    cuuint64_t strides[2] = {(cuuint64_t)K / 2, 64};
    cuuint32_t box[3] = {64, (cuuint32_t)kTile, 2};
    cuuint32_t estr[3] = {1, 1, 1};
    if (encode(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t *>(q), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return -1;
    if (!encode_tmap_2d(&smap, CU_TENSOR_MAP_DATA_TYPE_UINT16, s, G, (uint64_t)N, G * 2, 8, kTile,
                        CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_tmap_2d(&zmap, CU_TENSOR_MAP_DATA_TYPE_UINT16, z, G, (uint64_t)N, G * 2, 8, kTile,
                        CU_TENSOR_MAP_SWIZZLE_NONE))
        return -1;
    const I4Config c = i4_config(M, N, K);
    const int max_segs = i4_max_segments(N, K, c.grid);
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
#define WQ_I4_LAUNCH(NT_)                                                                                         \
    e = c.stages == 3 ? cudaLaunchKernelEx(&cfg, gemv_w4a16_i4mt_kernel<NT_, 3>, wmap, smap, zmap, x, Mi, Ni, Ki, y, \
                                           ws, cnt, max_segs, status, c.npairs, col_scale)                           \
                      : cudaLaunchKernelEx(&cfg, gemv_w4a16_i4mt_kernel<NT_, 2>, wmap, smap, zmap, x, Mi, Ni, Ki, y, \
                                           ws, cnt, max_segs, status, c.npairs, col_scale)
    WQ_I4_LAUNCH(1);
#undef WQ_I4_LAUNCH
    return e == cudaSuccess ? 0 : -2;
}

}  // namespace wq

// wq_gemv_m1.cu -- W4A16, group 128, a single activation row (M = 1): the
// decode step of an LLM, bound by streaming the packed weights from HBM once.
//
// "Quantization Methods Compared: INT8, GPTQ, AWQ, FP8, FP4 and KV-Cache
// Quantization", section "Hardware, formats and the roofline": at batch 1 a
// decode step reads every weight once and does two flops per weight, so the
// kernel has to keep HBM streaming while spending as few issue slots per
// weight as possible on the dequantisation w_hat = s (q - z) ("Quantization
// for LLM inference: FP8, INT4 (GPTQ, AWQ) and GGUF", "The minimum maths").
//
// Integer products.  Per group g of 128 inputs,
//     sum_k w_hat_k x_k = s (sum_k q_k x_k - z sum_k x_k),
// and both sums are computed exactly in integers:
//  * x is written, once per CTA, as D = 4 planes of signed radix-128 digits
//    per group: x_k = 2^(E_g - 5) sum_c d_ck 128^-c, |d_ck| <= 64, where 2^E_g
//    <= max |x| of the group < 2^(E_g + 1).  bf16 has 8 significant bits, so
//    every x_k of magnitude at least 2^(E_g - 19) is represented exactly;
//    smaller ones are rounded to the nearest multiple of 2^(E_g - 26), far
//    below the binary32 rounding of the sums they enter.
//  * The codes enter the tensor core as they are: a 32-bit word of 8 nibbles
//    becomes two words of 4 unsigned bytes (one LOP3 for the even codes, a
//    shift and a LOP3 for the odd ones; 3 instructions per 8 codes, against
//    11 for an exact bf16 q - z), and mma.sync m16n8k32 u8 x s8 -> s32 takes
//    512 codes of 16 rows per instruction against the digit planes in its B
//    columns.  The column sums D_c = sum_k q_k d_ck are exact integers.
//  * The accumulator starts at the bits of 1.5 * 2^23, so the result read as
//    binary32 minus 1.5 * 2^23 is D_c itself (|D_c| < 2^17) with no
//    conversion instruction.  The lane then forms D_c - z S_c (S_c = sum_k
//    d_ck, exact for any zero-point up to 2^11 in magnitude, one rounding
//    beyond) and adds s 2^(E_g - 5) (D_c - z S_c) to the binary32 sum of
//    its column; the columns meet, weighted by 128^-c, once per segment.
//  The legacy mma.sync integer path issues at the rate of the bf16 one on
//  B200, so the tensor core has room to spare; the point is the ALU: the
//  exact-bf16 form of this kernel was bound by its LOP3/shift rate near 75% of
//  HBM bandwidth in steady state.  Rows whose weights are all zero (q = z)
//  still give exactly zero, and zero-points far outside [0, 15] need no
//  special path.
//
// Memory pipeline.  TMA throughput on B200 depends on the size of each copy:
// copies of 2 KB stream at about 4 TB/s, copies of 8 KB and more at over
// 6 TB/s.  So one producer warp per CTA moves 32 KB per copy: a stage is 256
// rows x 2 groups, fetched through a 3-D view of the packed codes (64-byte
// group slices, rows, groups; the group stride is 64 bytes) that lands in
// shared memory as [group][row][64 B], so the consumers' 16-byte reads are
// free of bank conflicts.  Three stages are in flight (two when the digit
// planes of a long K need the room); the scales and zero-points follow in
// [256 rows x 8 groups] boxes, double buffered.
//
// Work layout.
//  * A unit is (tile of 256 rows, pair of groups).  The grid is persistent
//    (one CTA per SM) and every CTA takes an equal contiguous range of units,
//    tile by tile along K (stream-K), so no SM idles behind a short last wave.
//    A CTA's range touches at most min(n, K / 256) distinct group pairs of x,
//    and only their digit planes are made and kept.
//  * Consumer warp w (16 of them) owns rows 16w .. 16w+15 of the tile.  Lane
//    (g, t) (g = lane / 4, t = lane % 4) reads 16 bytes -- codes 32t .. 32t+31
//    of the group -- of rows g and g + 8; word w of them is the A operand of
//    the group's w-th k32 step (even codes in the first k half, odd codes in
//    the second), and the digit planes are laid out in the same k order, one
//    16-byte load per lane and two steps.
//  * A tile split between CTAs leaves one binary32 partial per segment in the
//    workspace.  The consumers never wait on global memory for this: each
//    warp drops its 16 row sums into a double-buffered shared-memory tile and
//    moves on, and a separate combiner warp takes it from there.  The CTA
//    holding the tile's first segment combines it: that segment is the end of
//    its range, while the tile's last segment is the start of the next CTA's,
//    so it is usually among the last to finish.  The other segments write
//    their slots and bump the tile's arrival counter (a release add, no round
//    trip); the first segment's combiner keeps its own sums in registers,
//    waits (bounded) until the counter shows the others, adds their slots in
//    segment order, writes y and re-zeroes the counter -- a fixed order, so
//    results do not depend on timing.
//  * Launched with programmatic dependent launch: in a stream of linears the
//    next kernel's CTAs start as SMs free up, initialise their barriers and
//    load their first weight stages into shared memory while this one
//    finishes; they read x and write anything only after griddepcontrol.wait.
//  * Every mbarrier wait is bounded; on a timeout the kernel records it in the
//    status word, the producer stops issuing, and every later wait returns at
//    once: the consumers finish their loop (on garbage) with unchanged control
//    flow, the producer waits (bounded) for its copies in flight, and the CTA
//    exits.  The workspace must then be zero-filled again before reuse.

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
constexpr int kDigits = 4;                        // radix-128 digit planes of x
constexpr uint32_t kDigitPairBytes = 2 * 2 * 4 * kDigits * 16;  // [group][half][t][digit][16 B]
constexpr float kMagic = 12582912.0f;             // 1.5 * 2^23
constexpr uint32_t kMagicBits = 0x4B400000u;

// shared memory: [stages][s/z windows][2 partial tiles][digit planes][S sums][group factors][barriers]
struct M1Layout {
    size_t sz, part, dig, gsum, gfac, bar, total;
    __host__ __device__ M1Layout(int stages, int npairs, int sub)
    {
        sz = (size_t)stages * kStageBytes;
        part = sz + 2 * 2 * kSzBytes;
        dig = part + 2 * kTile * 4;
        gsum = dig + (size_t)npairs * kDigitPairBytes;
        gfac = gsum + (size_t)npairs * 2 * sub * kDigits * 4;
        bar = (gfac + (size_t)npairs * 2 * 4 + 7) & ~(size_t)7;
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

__device__ __forceinline__ uint16_t lds_u16(uint32_t addr)
{
    uint16_t r;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(r) : "r"(addr));
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

// The digit planes, column sums and scale factor of one group of x (one warp).  Lane L takes word L / 2 of
// the group (inputs 8 (L / 2) .. + 7) and of it the inputs of parity L % 2: 2 i + L % 2, i = 0 .. 3, the byte
// order of the A operand's even (L % 2 = 0) and odd code words.
// SUB quantisation groups share the 128 inputs (groups of 128 / SUB): their column sums are kept apart, each
// over the lanes that hold its inputs (32 / SUB consecutive lanes).
template <int SUB>
__device__ __forceinline__ void make_digits(const uint16_t *__restrict__ xg, const float *__restrict__ csg,
                                            uint32_t dig_pair, uint32_t gsum_g, uint32_t gfac_g, int h, int lane)
{
    const int wq_ = lane >> 1, par = lane & 1;
    uint4 v = *reinterpret_cast<const uint4 *>(xg + 8 * wq_);
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
    const uint32_t dst = dig_pair + (uint32_t)(((h * 2 + half) * 4 + t_) * (kDigits * 16) + (w & 1) * 8 + par * 4);
#pragma unroll
    for (int c = 0; c < kDigits; ++c) {
        const uint32_t lo = __byte_perm(t[0][c], t[1][c], 0x0040), hi = __byte_perm(t[2][c], t[3][c], 0x0040);
        const uint32_t packed = __byte_perm(lo, hi, 0x5410);
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(dst + (uint32_t)c * 16u), "r"(packed) : "memory");
        // the digit values (wrapping 32-bit arithmetic: the four magic offsets cancel)
        const int sum = (int)(t[0][c] + t[1][c] + t[2][c] + t[3][c] - 4u * kMagicBits);
        if constexpr (SUB == 1) {
            const int tot = __reduce_add_sync(0xffffffffu, sum);
            if (lane == 0) asm volatile("st.shared.f32 [%0], %1;" ::"r"(gsum_g + (uint32_t)c * 4u), "f"((float)tot) : "memory");
        } else {
            int tot = sum;  // over the 32 / SUB lanes of this lane's group
#pragma unroll
            for (int o = 1; o < 32 / SUB; o <<= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
            if ((lane & (32 / SUB - 1)) == 0)
                asm volatile("st.shared.f32 [%0], %1;" ::"r"(gsum_g + (uint32_t)((lane / (32 / SUB)) * kDigits + c) * 4u),
                             "f"((float)tot)
                             : "memory");
        }
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
template <int GROUP, int STAGES>
__global__ void __maxnreg__(96)
gemv_w4a16_m1_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap smap,
                     const __grid_constant__ CUtensorMap zmap, const uint16_t *__restrict__ x, int N, int K,
                     uint16_t *__restrict__ y, float *__restrict__ ws, int *__restrict__ cnt, int max_segs,
                     int *__restrict__ status, int npairs, const float *__restrict__ col_scale)
{
    extern __shared__ __align__(1024) uint8_t m1_raw[];
    // TMA destinations want 128-byte (we keep 1024-byte) alignment: align the base explicitly
    uint8_t *sm = m1_raw + ((1024u - (smem_u32(m1_raw) & 1023u)) & 1023u);
    constexpr int SUB = 128 / GROUP;  // quantisation groups per 128 inputs
    constexpr int UPW = GROUP / 32;   // units per s/z window of 8 groups
    const M1Layout L(STAGES, npairs, SUB);
    uint8_t *ring = sm;
    uint8_t *szr = sm + L.sz;                                     // [2 windows][s, z][256 rows][8 groups]
    float *part = reinterpret_cast<float *>(sm + L.part);         // [2][256 rows] partial sums
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
        const int g8 = (2 * SUB * pp) & ~7;  // the window's first group
        tma_load_2d(d, &smap, &szfull[slot], g8, pt * kTile);
        tma_load_2d(d + kSzBytes, &zmap, &szfull[slot], g8, pt * kTile);
        ++wins;
    };
    if (wid == kProducer && lane == 0) {
        // the prologue issues at most two windows (the ring's slots) and leaves a third to the main loop
        for (; pi < STAGES && pi < n; ++pi) {
            const bool nw = pi == 0 || (pp & (UPW - 1)) == 0;
            if (nw && wins >= 2) break;
            if (nw) issue_window(wins & 1);
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
                // s/z window: at the first unit and at every UPW-th pair of a tile
                if (i == 0 || (pp & (UPW - 1)) == 0) {
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
        // The CTA's range splits a tile wherever it starts or ends inside one; walk those tiles in the
        // consumers' order.  Lane l handles rows 8l .. 8l + 7 of the tile.
        int pseg = 0;
        for (int64_t tt = beg / P; tt * P < end; ++tt) {
            if (tt * P >= beg && tt * P + P <= end) continue;  // whole tile: the consumers wrote y
            const int b = pseg & 1;
            const bool ok = __all_sync(0xffffffffu, mbar_wait(&pfull[b], (uint32_t)(pseg >> 1) & 1u, status, flags));
            if (!ok) break;
            const float4 v0 = *reinterpret_cast<const float4 *>(part + b * kTile + 8 * lane);
            const float4 v1 = *reinterpret_cast<const float4 *>(part + b * kTile + 8 * lane + 4);
            __syncwarp();
            if (lane == 0) mbar_arrive(&pempty[b]);  // the shared tile is in registers: free it
            ++pseg;
            const int c_first = cta_of(tt * P, units, B);
            const int nseg = cta_of(tt * P + P - 1, units, B) - c_first + 1;
            float *slots = ws + (size_t)tt * max_segs * kTile;
            if (bid != c_first) {
                float4 *mine = reinterpret_cast<float4 *>(slots + (bid - c_first) * kTile + 8 * lane);
                mine[0] = v0;
                mine[1] = v1;
                // the release of the add below covers every lane's slot writes (ordered by the warp barrier)
                __syncwarp();
                if (lane == 0) red_add_release(cnt + tt, 1);
                continue;
            }
            // the tile's first segment: wait (bounded) for the other nseg - 1 to arrive
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
            if (!__shfl_sync(0xffffffffu, arrived, 0)) break;
            {
                // sum the segments in segment order, from 0: this CTA's own (segment 0, in registers), then the
                // slots of the others
                float v[8] = {0.0f + v0.x, 0.0f + v0.y, 0.0f + v0.z, 0.0f + v0.w,
                              0.0f + v1.x, 0.0f + v1.y, 0.0f + v1.z, 0.0f + v1.w};
                const float4 *q = reinterpret_cast<const float4 *>(slots + 8 * lane);
                int o = 1;
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
        const uint32_t dig_u32 = smem_u32(sm + L.dig), gsum_u32 = smem_u32(sm + L.gsum), gfac_u32 = smem_u32(sm + L.gfac);
        // ---- digit planes of the group pairs this CTA touches: pair (pair0 + j) mod P in slot j ----
        const int nslots = min(n, P);
        for (int j = wid; j < 2 * nslots; j += kC) {
            const int js = j >> 1, h = j & 1;
            int pj = pair0 + js;
            if (pj >= P) pj -= P;
            const int kg = 2 * pj + h;
            make_digits<SUB>(x + (size_t)kg * 128, col_scale ? col_scale + (size_t)kg * 128 : nullptr,
                             dig_u32 + (uint32_t)js * kDigitPairBytes,
                             gsum_u32 + (uint32_t)(js * 2 + h) * (SUB * kDigits * 4), gfac_u32 + (uint32_t)(js * 2 + h) * 4u,
                             h, lane);
        }
        named_bar_sync(1, kC * 32);

        const int gq = lane >> 2, tq = lane & 3;
        const uint32_t ring_u32 = smem_u32(ring), szr_u32 = smem_u32(szr);
        const int r0 = 16 * wid + gq;  // this lane's rows in the tile: r0 and r0 + 8
        // this lane's B columns are digits gq (all k) and its accumulator columns 2 tq, 2 tq + 1
        const bool bcol = gq < kDigits, ccol = 2 * tq < kDigits;
        const float cw0 = ccol ? exp2i(-14 * tq) : 0.0f, cw1 = ccol ? exp2i(-14 * tq - 7) : 0.0f;  // 128^-c
        float acc[2][2] = {{0.0f, 0.0f}, {0.0f, 0.0f}};  // [row r0, r0 + 8][column 2 tq, 2 tq + 1]
        const uint32_t cmag[4] = {kMagicBits, kMagicBits, kMagicBits, kMagicBits};
        int t = tile0, p = pair0, seg_first = pair0;
        int win = -1;
        int pseg = 0;  // partial segments handed to the combiner
        int s = 0;     // stage slot of unit i, and the parity of its fill
        int di = 0;    // digit slot of pair p
        uint32_t ph = 0, w_off = 0;
        const uint32_t w_lane = ring_u32 + (uint32_t)r0 * 64u + (uint32_t)tq * 16u;
        const uint32_t sz_lane = szr_u32 + (uint32_t)r0 * 16u;
        const uint32_t b_lane = dig_u32 + (uint32_t)(tq * (kDigits * 16) + gq * 16);
        const uint32_t s_lane = gsum_u32 + (uint32_t)(2 * tq) * 4u;
        // groups of 32 or 64: lane tq's codes of a 128-input block are group lsub of it; its B column gq is
        // non-zero only for that group's inputs (group gq / 2 or gq / 4 of the block), so the MMA's column sums
        // stay per group, and its accumulator columns 2 tq, 2 tq + 1 are digits of its own group
        const int lsub = SUB == 4 ? tq : SUB == 2 ? (tq >> 1) : 0;
        const bool bown = SUB == 4 ? (gq >> 1) == tq : SUB == 2 ? (gq >> 2) == (tq >> 1) : false;
        const uint32_t b_lane_g = dig_u32 + (uint32_t)(tq * (kDigits * 16) + (SUB == 4 ? (gq & 1) : (gq & 3)) * 16);
        float accg[2] = {0.0f, 0.0f};  // groups of 32 or 64: [row r0, r0 + 8], digit weights applied
        // A wait that runs out sets the abort flag and every later wait returns at once: the loop then runs
        // to its end on garbage, with the same control flow in every warp, so the barriers below still meet.
        for (int i = 0; i < n; ++i) {
            // ---- s/z window ----
            if (i == 0 || (p & (UPW - 1)) == 0) {
                if (win >= 0) {  // the previous window is consumed
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&szempty[win & 1]);
                }
                ++win;
                mbar_wait(&szfull[win & 1], (uint32_t)(win >> 1) & 1u, status, flags);
            }
            mbar_wait(&full[s], ph, status, flags);
            // ---- loads from the stage: rows r0, r0 + 8 of both groups; their s, z ----
            const uint32_t wsrc = w_lane + w_off;
            uint4 wv[2][2];  // [group h][row r0, row r0 + 8]
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int a = 0; a < 2; ++a) wv[h][a] = lds128(wsrc + (uint32_t)h * (kTile * 64u) + (uint32_t)a * 8u * 64u);
            float sv[2][2], zv[2][2];  // [block h][row r0, r0 + 8]: the (lane's) group's s and z
            if constexpr (SUB == 1) {
                const int kg = 2 * p;
                const uint32_t szsrc = sz_lane + (uint32_t)(win & 1) * 2u * kSzBytes + (uint32_t)(kg & 7) * 2u;
                // s and z of groups kg, kg + 1 are adjacent in the window box (kg is even): one 32-bit load per
                // row and array
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                    const uint32_t o = szsrc + (uint32_t)a * 8u * 16u;
                    const uint32_t s2 = lds_u32(o), z2 = lds_u32(o + kSzBytes);
                    sv[0][a] = __uint_as_float(s2 << 16);
                    sv[1][a] = __uint_as_float(s2 & 0xffff0000u);
                    zv[0][a] = __uint_as_float(z2 << 16);
                    zv[1][a] = __uint_as_float(z2 & 0xffff0000u);
                }
            } else {
                const int g0 = 2 * SUB * p;  // the unit's first group
                const uint32_t szw = sz_lane + (uint32_t)(win & 1) * 2u * kSzBytes;
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int a = 0; a < 2; ++a) {
                        const uint32_t o = szw + (uint32_t)a * 8u * 16u + (uint32_t)((g0 + h * SUB + lsub) & 7) * 2u;
                        sv[h][a] = __uint_as_float((uint32_t)lds_u16(o) << 16);
                        zv[h][a] = __uint_as_float((uint32_t)lds_u16(o + kSzBytes) << 16);
                    }
            }
            // the stage's weight bytes are in registers: hand the slot back to the producer
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            if (++s == STAGES) { s = 0; ph ^= 1u; w_off = 0; } else { w_off += kStageBytes; }
            const uint32_t bsrc = b_lane + (uint32_t)di * kDigitPairBytes;
            if constexpr (SUB == 1) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                // digit column gq of this lane's 8 inputs of each k32 step: steps 0, 1 then 2, 3
                uint4 Bv[2];
#pragma unroll
                for (int hf = 0; hf < 2; ++hf)
                    Bv[hf] = bcol ? lds128(bsrc + (uint32_t)((h * 2 + hf) * 4) * (kDigits * 16)) : make_uint4(0u, 0u, 0u, 0u);
                uint32_t C[4];
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const uint32_t va = word_of(wv[h][0], w), vb = word_of(wv[h][1], w);
                    const uint32_t b0 = word_of(Bv[w >> 1], (w & 1) * 2), b1 = word_of(Bv[w >> 1], (w & 1) * 2 + 1);
                    mma_u8s8(C, w == 0 ? cmag : C, va & 0x0F0F0F0Fu, vb & 0x0F0F0F0Fu, (va >> 4) & 0x0F0F0F0Fu,
                             (vb >> 4) & 0x0F0F0F0Fu, b0, b1);
                }
                // C: (row r0, column 2 tq), (r0, 2 tq + 1), (r0 + 8, 2 tq), (r0 + 8, 2 tq + 1), each 1.5 2^23 + D_c
                const float2 S = ccol ? lds_f2(s_lane + (uint32_t)(di * 2 + h) * (kDigits * 4)) : make_float2(0.0f, 0.0f);
                const float F = lds_f32(gfac_u32 + (uint32_t)(di * 2 + h) * 4u);
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                    const float sF = sv[h][a] * F;
                    const float d0 = fmaf(-zv[h][a], S.x, __uint_as_float(C[2 * a]) - kMagic);
                    const float d1 = fmaf(-zv[h][a], S.y, __uint_as_float(C[2 * a + 1]) - kMagic);
                    acc[a][0] = fmaf(sF, d0, acc[a][0]);
                    acc[a][1] = fmaf(sF, d1, acc[a][1]);
                }
            }
            } else {
            const uint32_t bsrc_g = b_lane_g + (uint32_t)di * kDigitPairBytes;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float F = lds_f32(gfac_u32 + (uint32_t)(di * 2 + h) * 4u);
                // groups of 32: two passes, digits 0, 1 then 2, 3 of each group; groups of 64: one pass, digits
                // 2 (tq % 2), + 1 of the lane's group in its accumulator columns
#pragma unroll
                for (int pass = 0; pass < (SUB == 4 ? 2 : 1); ++pass) {
                    uint4 Bv[2];
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf)
                        Bv[hf] = bown ? lds128(bsrc_g + (uint32_t)((h * 2 + hf) * 4) * (kDigits * 16) + (uint32_t)pass * 32u)
                                      : make_uint4(0u, 0u, 0u, 0u);
                    uint32_t C[4];
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const uint32_t va = word_of(wv[h][0], w), vb = word_of(wv[h][1], w);
                        const uint32_t b0 = word_of(Bv[w >> 1], (w & 1) * 2), b1 = word_of(Bv[w >> 1], (w & 1) * 2 + 1);
                        mma_u8s8(C, w == 0 ? cmag : C, va & 0x0F0F0F0Fu, vb & 0x0F0F0F0Fu, (va >> 4) & 0x0F0F0F0Fu,
                                 (vb >> 4) & 0x0F0F0F0Fu, b0, b1);
                    }
                    const int d0i = SUB == 4 ? 2 * pass : 2 * (tq & 1);  // the digits in columns 2 tq, 2 tq + 1
                    const float2 S = lds_f2(gsum_u32 + (uint32_t)(((di * 2 + h) * SUB + lsub) * kDigits + d0i) * 4u);
                    const float w0 = exp2i(-7 * d0i), w1 = exp2i(-7 * d0i - 7);
#pragma unroll
                    for (int a = 0; a < 2; ++a) {
                        const float d0 = fmaf(-zv[h][a], S.x, __uint_as_float(C[2 * a]) - kMagic);
                        const float d1 = fmaf(-zv[h][a], S.y, __uint_as_float(C[2 * a + 1]) - kMagic);
                        accg[a] = fmaf(sv[h][a] * F, fmaf(d1, w1, d0 * w0), accg[a]);
                    }
                }
            }
            }
            if (++di == P) di = 0;
            // ---- end of a segment: the tile's last pair, or the end of this CTA's range ----
            const bool tile_done = (p + 1 == P);
            if (tile_done || i + 1 == n) {
                // the row sums: columns weighted by 128^-c, then summed over the four tq lanes
                float rs[2];
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                    float v = SUB == 1 ? fmaf(acc[a][1], cw1, acc[a][0] * cw0) : accg[a];
                    accg[a] = 0.0f;
                    v += __shfl_xor_sync(0xffffffffu, v, 1);
                    v += __shfl_xor_sync(0xffffffffu, v, 2);
                    rs[a] = v;
                    acc[a][0] = acc[a][1] = 0.0f;
                }
                const int row0 = t * kTile + r0;
                if (seg_first == 0 && tile_done) {
                    if (tq == 0) {
                        if (row0 < N) y[row0] = f32_to_bf16(rs[0]);
                        if (row0 + 8 < N) y[row0 + 8] = f32_to_bf16(rs[1]);
                    }
                } else {
                    // partial: this warp's 16 row sums go to the shared tile of this segment; the combiner
                    // warp takes it from there (tiles alternate between two buffers)
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
            if (++p == P) { p = 0; ++t; seg_first = 0; }
        }
    }
    __syncthreads();
}

// Shape-dependent launch parameters, cached per (device, N, K): grid (one CTA per SM, fewer when there is
// less work), the digit slots a CTA needs, and the stage count that fits shared memory.
struct M1Config {
    int grid, npairs, stages;
    size_t smem;
};

M1Config m1_config(int64_t N, int64_t K, int g)
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
            int v = 148, o = 0;
            cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
            cudaDeviceGetAttribute(&o, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
#define WQ_M1_ATTR(G_, S_) cudaFuncSetAttribute(gemv_w4a16_m1_kernel<G_, S_>, cudaFuncAttributeMaxDynamicSharedMemorySize, o)
            WQ_M1_ATTR(128, 3); WQ_M1_ATTR(128, 2); WQ_M1_ATTR(64, 3); WQ_M1_ATTR(64, 2); WQ_M1_ATTR(32, 3); WQ_M1_ATTR(32, 2);
#undef WQ_M1_ATTR
            it = dev_of.emplace(dev, std::make_pair(v, o)).first;
        }
        sms = it->second.first;
        optin = it->second.second;
    }
    const int64_t P = K / 256;
    const int64_t units = ((N + kTile - 1) / kTile) * P;
    M1Config c;
    c.grid = (int)std::max<int64_t>(1, std::min<int64_t>(units, sms));
    const int64_t per = (units + c.grid - 1) / c.grid;  // most units any CTA takes
    c.npairs = (int)std::min<int64_t>(per, P);
    const int sub = 128 / g;
    c.stages = M1Layout(3, c.npairs, sub).total <= (size_t)optin ? 3 : 2;
    c.smem = M1Layout(c.stages, c.npairs, sub).total;
    return c;
}

// Most segments (CTAs) any tile is split into, for this grid.
int m1_max_segments(int64_t N, int64_t K, int grid)
{
    const int64_t P = K / 256;
    const int64_t units = ((N + kTile - 1) / kTile) * P;
    const int64_t per = units / std::min<int64_t>(grid, units);  // >= 1 unit per CTA
    return (int)std::min<int64_t>((P + per - 1) / per + 1, P);
}

size_t m1_slots_bytes(int64_t N, int64_t K, int grid)
{
    const int64_t ntiles = (N + kTile - 1) / kTile;
    return ((size_t)ntiles * m1_max_segments(N, K, grid) * kTile * 4 + 255) / 256 * 256;
}

}  // namespace

bool gemv_m1_eligible(int64_t M, int64_t N, int64_t K, int g)
{
    // groups of 32, 64 or 128; K % 1024: the s/z row stride (K / g bf16) must be a multiple of 16 bytes for
    // their tensor maps; two stages and the digit planes and sums of every group pair of a tile must fit in the
    // 227 KB of shared memory a block can have (K <= 32768 for groups of 64 and 128, K <= 31744 for 32)
    if (M != 1 || !(g == 128 || g == 64 || g == 32) || K < 1024 || K % 1024 != 0 || K > 32768 || N < 1 ||
        N > 0x7fffffffLL)
        return false;
    return M1Layout(2, (int)(K / 256), 128 / g).total <= (size_t)232448;
}

size_t gemv_m1_workspace_bytes(int64_t M, int64_t N, int64_t K, int g)
{
    if (!gemv_m1_eligible(M, N, K, g)) return 0;
    const int64_t ntiles = (N + kTile - 1) / kTile;
    return counter_region_bytes(ntiles) + m1_slots_bytes(N, K, m1_config(N, K, g).grid);
}

int launch_gemv_w4a16_m1(const uint16_t *x, int64_t N, int64_t K, const uint8_t *q, const uint16_t *s,
                         const uint16_t *z, int g, uint16_t *y, void *workspace, int *status, cudaStream_t st,
                         const float *col_scale)
{
    // packed codes seen as (64-byte group slice, row, group): strides K/2 bytes (row) and 64 bytes (group)
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
    const uint64_t Gs = (uint64_t)K / (uint64_t)g;  // s and z: one per group of g
    if (!encode_tmap_2d(&smap, CU_TENSOR_MAP_DATA_TYPE_UINT16, s, Gs, (uint64_t)N, Gs * 2, 8, kTile,
                        CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_tmap_2d(&zmap, CU_TENSOR_MAP_DATA_TYPE_UINT16, z, Gs, (uint64_t)N, Gs * 2, 8, kTile,
                        CU_TENSOR_MAP_SWIZZLE_NONE))
        return -1;
    const M1Config c = m1_config(N, K, g);
    const int grid = c.grid;
    const int max_segs = m1_max_segments(N, K, grid);
    const int64_t ntiles = (N + kTile - 1) / kTile;
    uint8_t *w8 = static_cast<uint8_t *>(workspace);
    int *cnt = reinterpret_cast<int *>(w8);
    float *ws = reinterpret_cast<float *>(w8 + counter_region_bytes(ntiles));
    if (clear_extra_counters(workspace, ntiles, st) != cudaSuccess) return -2;
    // programmatic dependent launch: this grid may start while the previous kernel in the stream finishes;
    // the kernel reads nothing that kernel may write, and writes nothing, before griddepcontrol.wait
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kT);
    cfg.dynamicSmemBytes = c.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // three stages in flight measured the same as four on the 70B-shaped linears
    cudaError_t e = cudaErrorInvalidValue;
#define WQ_M1_LAUNCH(G_)                                                                                           \
    e = c.stages == 3 ? cudaLaunchKernelEx(&cfg, gemv_w4a16_m1_kernel<G_, 3>, wmap, smap, zmap, x, (int)N, (int)K, y, \
                                           ws, cnt, max_segs, status, c.npairs, col_scale)                            \
                      : cudaLaunchKernelEx(&cfg, gemv_w4a16_m1_kernel<G_, 2>, wmap, smap, zmap, x, (int)N, (int)K, y, \
                                           ws, cnt, max_segs, status, c.npairs, col_scale)
    if (g == 128) WQ_M1_LAUNCH(128);
    else if (g == 64) WQ_M1_LAUNCH(64);
    else WQ_M1_LAUNCH(32);
#undef WQ_M1_LAUNCH
    if (e != cudaSuccess) return -2;
    return 0;
}

}  // namespace wq

// wq_quant.cu -- group-wise INT4 (asymmetric) and INT8 (symmetric absmax)
// quantisation kernels.
//
// Asymmetric INT4 follows "Quantization for LLM inference: FP8, INT4 (GPTQ,
// AWQ) and GGUF", section "The minimum maths: scale and zero-point":
// s = (max - min) / 15, z = round(-min / s), q = clip(round(w / s + z), 0, 15).
// Symmetric INT8 follows "Quantization Methods Compared: INT8, GPTQ, AWQ, FP8,
// FP4 and KV-Cache Quantization", section "What quantisation does":
// s = max|w| / 127, q = round(w / s).  Symmetric INT4 (levels -7..7,
// s = max|w| / 7) is described at quant_int4_sym_kernel.
//
// Both are HBM streams (read 2 or 4 B per weight, write 0.5 or 1 B plus the
// per-group parameters).  Layout of the work: a warp takes 256 consecutive
// weights of one row, 8 per lane (one 16-byte load for bf16), so a group of
// g weights spans g/8 adjacent lanes and its min/max (or absmax) is a
// log2(g/8)-step xor-shuffle reduction (for bf16 weights, min and -max
// travel as one bf16 pair).  Every lane then derives the same (s, z) and
// encodes its 8 weights into one 32-bit word of nibbles (INT4) or one 64-bit
// word of bytes (INT8); stores are 128 contiguous bytes per warp.
//
// Arithmetic matches the library contract bit for bit: binary32 with
// explicit round-to-nearest-even intrinsics (no contraction is possible),
// round half to even, bf16 rounding to nearest even.  Three equivalences
// save instructions without changing a bit:
//  * every quotient (w / s, -min / s, range / 15, absmax / 127) is RN of the
//    exact quotient, formed from a reciprocal and one correction
//    (quotient_rn), with the IEEE division outside the proven range;
//  * clipping to the code range before rounding gives the same integer as
//    rounding first, and adding 1.5 * 2^23 does the rounding (rint_bits);
//  * the eight rounded patterns, shifted into place and summed, minus their
//    summed offsets, are the packed nibbles.
#include <map>
#include <mutex>
#include <type_traits>
#include <utility>

#include "wq_common.cuh"
#include "wq_internal.h"

namespace wq {

namespace {

constexpr int kQuantThreads = 256;
constexpr int kQuantUnroll = 4;  // row chunks in flight per warp

// Position (row n, 256-weight chunk c) of a warp's task t = n * chunks + c, advanced by the grid's warp
// count without a 64-bit division per task.
struct TaskWalk {
    int64_t n, c, dn, dc, chunks;
    __device__ __forceinline__ TaskWalk(int64_t t, int64_t stride, int64_t chunks_) : chunks(chunks_)
    {
        n = t / chunks;
        c = t - n * chunks;
        dn = stride / chunks;
        dc = stride - dn * chunks;
    }
    __device__ __forceinline__ void step()
    {
        n += dn;
        c += dc;
        if (c >= chunks) { c -= chunks; ++n; }
    }
};

template <typename T>
__device__ __forceinline__ void load8(const T *p, float v[8]);

template <>
__device__ __forceinline__ void load8<float>(const float *p, float v[8])
{
    const uint4 a = ld_stream_v4(p), b = ld_stream_v4(p + 4);
    v[0] = __uint_as_float(a.x); v[1] = __uint_as_float(a.y);
    v[2] = __uint_as_float(a.z); v[3] = __uint_as_float(a.w);
    v[4] = __uint_as_float(b.x); v[5] = __uint_as_float(b.y);
    v[6] = __uint_as_float(b.z); v[7] = __uint_as_float(b.w);
}

template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16 *p, float v[8])
{
    const uint4 a = ld_stream_v4(p);
    const uint32_t u[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(u[i] << 16);
        v[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
    }
}

// Correctly rounded quotients w / s for the codes, without a division per weight.  Markstein's final
// correction step (P. Markstein, "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990): with r = RN(1/s) and q0 = RN(w * r), the residual
// e = w - q0 * s is exact (one fused multiply-add), and RN(q0 + e * r) = RN(w / s) provided the reciprocal
// and the quotient stay in the normal range.  The scales here are bf16 values; for every bf16 significand
// of s and every binary32 significand of w this identity was checked exhaustively (the check is part of
// the test suite).  A group whose scale or largest quotient could leave the normal range uses the IEEE
// division instead; quotients too small to be normal never change a code (t = RN(q + z) rounds to z, or
// to 0 when z = 0).
__device__ __forceinline__ bool quotients_by_reciprocal(float s, float maxabs)
{
    return s >= 0x1p-100f && s <= 0x1p100f && maxabs <= s * 0x1p100f;
}

__device__ __forceinline__ float quotient_rn(float w, float s, float r)
{
    const float q0 = __fmul_rn(w, r);
    const float e = __fmaf_rn(-q0, s, w);
    return __fmaf_rn(e, r, q0);
}

// RN(d / c) for a bf16-representable constant c (15 or 127) with rc = RN(1 / c): the same identity, with
// the IEEE division where d could leave its proven range (d non-finite, above 2^100, or tiny but not 0).
__device__ __forceinline__ float div_by_const_rn(float d, float c, float rc)
{
    const float ad = fabsf(d);
    return (ad <= 0x1p100f && (ad >= 0x1p-90f || ad == 0.0f)) ? quotient_rn(d, c, rc) : __fdiv_rn(d, c);
}
constexpr float kRcp15 = 0x1.111112p-4f;   // RN(1 / 15)
constexpr float kRcp7 = 0x1.24924ap-3f;    // RN(1 / 7)
constexpr float kRcp127 = 0x1.020408p-7f;  // RN(1 / 127)

// Round an integer-bound value t, already clipped to [-127, 127], to the nearest integer with ties to
// even, and return the binary32 bit pattern of 1.5 * 2^23 + round(t): the integer sits in the low bits
// (two's complement in the low byte for negative t).  Adding 1.5 * 2^23 leaves a unit in the last place
// of 1, so the addition itself is the rounding.
__device__ __forceinline__ uint32_t rint_bits(float t) { return __float_as_uint(__fadd_rn(t, 0x1.8p23f)); }
constexpr uint32_t kRintBase = 0x4B400000u;  // bits of 1.5 * 2^23

// Packed binary32 pairs (sm_100 f32x2 arithmetic; round to nearest, no fused contraction across the pair):
// the low 32 bits hold the first value.
__device__ __forceinline__ uint64_t f32x2_bits(float lo, float hi)
{
    return ((uint64_t)__float_as_uint(hi) << 32) | (uint64_t)__float_as_uint(lo);
}
__device__ __forceinline__ uint64_t f32x2_mul(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f32x2_add(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f32x2_fma(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint32_t word_of(const uint4 &v, int i)
{
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// s of one INT4 group from its min and max (the library contract): RN((max - min) / 15) rounded to bf16;
// a zero range falls back to max(|min|, |max|), then to 1.
__device__ __forceinline__ float int4_scale(float mn, float mx)
{
    float s = round_bf16(div_by_const_rn(__fsub_rn(mx, mn), 15.0f, kRcp15));
    if (s == 0.0f) {
        s = round_bf16(fmaxf(fabsf(mn), fabsf(mx)));
        if (s == 0.0f) s = 1.0f;
    }
    return s;
}

// bf16x2 minimum (each half; a NaN half yields the other operand's half, as fminf does)
__device__ __forceinline__ uint32_t bf16x2_min(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("min.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t bf16x2_max(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// SCALED: quantise w[n][k] * col_scale[k] (each product rounded to binary32), the weights an
// activation-aware per-input-channel scaling hands the quantiser ("Quantization Methods Compared",
// section "The methods compared": AWQ scales the salient channels up before quantising).
//
// A lane takes kWordsPerLane x 8 = 32 consecutive weights of a row (two 32-byte loads for bf16), so a group
// of G weights spans G / 32 lanes (1, 2 or 4) and a warp task is 1,024 weights.  The group's parameters
// (min, max, s, 1/s, z) are formed once per 32 weights instead of once per 8, which is where the
// instructions of an issue-bound quantiser went.
constexpr int kWordsPerLane = 4;                        // 8-weight words per lane
constexpr int kLaneWeights = 8 * kWordsPerLane;         // 32
constexpr int kWarpWeights = 32 * kLaneWeights;         // 1,024 weights per warp task
constexpr int kInt4Unroll = 2;                          // tasks in flight per warp

// Weight i of 32 held either as widened binary32 values (v) or as the loaded bf16 words (raw).
template <bool BF16>
__device__ __forceinline__ float lane_weight(const float *v, const uint4 *raw, int i)
{
    if (BF16) {
        const uint4 &r = raw[i >> 3];
        const int w = (i >> 1) & 3;
        const uint32_t word = w == 0 ? r.x : w == 1 ? r.y : w == 2 ? r.z : r.w;
        return __uint_as_float((i & 1) ? (word & 0xffff0000u) : (word << 16));
    }
    return v[i];
}

template <typename T, int G, bool SCALED>
__global__ void __launch_bounds__(kQuantThreads)
quant_int4_kernel(const T *__restrict__ w, int64_t N, int64_t K, int64_t ldw,
                  uint8_t *__restrict__ qweight, uint16_t *__restrict__ scales,
                  uint16_t *__restrict__ zeros, const float *__restrict__ col_scale)
{
    constexpr int LPG = G / kLaneWeights;  // lanes per group
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t chunks = (K + kWarpWeights - 1) / kWarpWeights;
    const int64_t tasks = N * chunks;
    const int64_t Gn = K / G;

    // packed bf16 min/max only for unscaled bf16 weights (scaled products are binary32 values)
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value && !SCALED;
    TaskWalk walk(warp0, n_warps, chunks);
    for (int64_t t0 = warp0; t0 < tasks; t0 += n_warps * kInt4Unroll) {
        float v[kInt4Unroll][kBf16 ? 1 : kLaneWeights];  // binary32 input or scaled products
        uint4 raw[kInt4Unroll][kWordsPerLane];             // bf16 input: the weights as loaded
        int64_t n[kInt4Unroll], k0[kInt4Unroll];
        bool active[kInt4Unroll];
#pragma unroll
        for (int u = 0; u < kInt4Unroll; ++u) {
            n[u] = walk.n;
            k0[u] = walk.c * kWarpWeights + lane * kLaneWeights;
            active[u] = (walk.n < N) && (k0[u] < K);
            if (kBf16) {
#pragma unroll
                for (int j = 0; j < kWordsPerLane; ++j) raw[u][j] = make_uint4(0u, 0u, 0u, 0u);
                if (active[u]) {
#pragma unroll
                    for (int j = 0; j < kWordsPerLane; ++j) raw[u][j] = ld_stream_v4(w + n[u] * ldw + k0[u] + 8 * j);
                }
            } else if (active[u]) {
#pragma unroll
                for (int j = 0; j < kWordsPerLane; ++j) {
                    load8<T>(w + n[u] * ldw + k0[u] + 8 * j, v[u] + 8 * j);
                    if (SCALED) {
                        float c[8];
                        load8<float>(col_scale + k0[u] + 8 * j, c);
#pragma unroll
                        for (int i = 0; i < 8; ++i) v[u][8 * j + i] = __fmul_rn(v[u][8 * j + i], c[i]);
                    }
                }
            }
            walk.step();
        }
#pragma unroll
        for (int u = 0; u < kInt4Unroll; ++u) {
            if (t0 + u * n_warps >= tasks) break;  // warp-uniform
            float mn, mx;
            if (kBf16) {
                // bf16 weights are exact in bf16: reduce (min, -max) as one packed pair (a group's lanes are
                // all active or all inactive; inactive ones contribute +inf to both minima)
                uint32_t lo = bf16x2_min(raw[u][0].x, raw[u][0].y), hi = bf16x2_max(raw[u][0].x, raw[u][0].y);
                lo = bf16x2_min(lo, bf16x2_min(raw[u][0].z, raw[u][0].w));
                hi = bf16x2_max(hi, bf16x2_max(raw[u][0].z, raw[u][0].w));
#pragma unroll
                for (int j = 1; j < kWordsPerLane; ++j) {
                    lo = bf16x2_min(lo, bf16x2_min(bf16x2_min(raw[u][j].x, raw[u][j].y), bf16x2_min(raw[u][j].z, raw[u][j].w)));
                    hi = bf16x2_max(hi, bf16x2_max(bf16x2_max(raw[u][j].x, raw[u][j].y), bf16x2_max(raw[u][j].z, raw[u][j].w)));
                }
                hi ^= 0x80008000u;
                uint32_t pk = active[u] ? bf16x2_min(__byte_perm(lo, hi, 0x5410), __byte_perm(lo, hi, 0x7632)) : 0x7F807F80u;
#pragma unroll
                for (int o = 1; o < LPG; o <<= 1) pk = bf16x2_min(pk, __shfl_xor_sync(0xffffffffu, pk, o));
                mn = __uint_as_float(pk << 16);
                mx = __uint_as_float((pk & 0xffff0000u) ^ 0x80000000u);
            } else {
                mn = INFINITY;
                mx = -INFINITY;
                if (active[u]) {
#pragma unroll
                    for (int i = 0; i < kLaneWeights; ++i) { mn = fminf(mn, v[u][i]); mx = fmaxf(mx, v[u][i]); }
                }
#pragma unroll
                for (int o = 1; o < LPG; o <<= 1) {
                    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                }
            }
            if (!active[u]) continue;
            const float s = int4_scale(mn, mx);
            float z;  // round_bf16(rint(RN(-min / s)) + 0)
            uint32_t packed[kWordsPerLane];
            // q = clip(rint(RN(w / s) + z), 0, 15): clipping before the rounding gives the same integer, and
            // rint_bits leaves it in the low bits; the eight patterns shifted into place and summed, minus
            // the summed offsets, are the eight nibbles of a word
            const float maxabs = fmaxf(fabsf(mn), fabsf(mx));
            if (quotients_by_reciprocal(s, maxabs)) {
                const float r = __frcp_rn(s);
                z = round_bf16(__fadd_rn(rintf(quotient_rn(-mn, s, r)), 0.0f));
                if (kBf16 && maxabs <= s * 8192.0f && fabsf(z) <= 8192.0f) {
                    // two weights per instruction: the same correctly rounded quotients (packed binary32
                    // multiply and fused multiply-adds), + z, and the rounding by 1.5 * 2^23; |t| < 2^14 here,
                    // so each rounded t is the low half-word of its bit pattern, and the pair is clipped to
                    // [0, 15] as two 16-bit integers
                    const uint64_t r2 = f32x2_bits(r, r), ns2 = f32x2_bits(-s, -s), z2 = f32x2_bits(z, z);
                    const uint64_t m2 = f32x2_bits(0x1.8p23f, 0x1.8p23f);
#pragma unroll
                    for (int j = 0; j < kWordsPerLane; ++j) {
                        uint32_t b[4];
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            const uint32_t wd = word_of(raw[u][j], h);
                            const uint64_t w2 = ((uint64_t)(wd & 0xffff0000u) << 32) | (uint64_t)(wd << 16);
                            const uint64_t q0 = f32x2_mul(w2, r2);
                            const uint64_t q = f32x2_fma(f32x2_fma(q0, ns2, w2), r2, q0);
                            const uint64_t t = f32x2_add(f32x2_add(q, z2), m2);
                            uint32_t p2 = __byte_perm((uint32_t)t, (uint32_t)(t >> 32), 0x5410);
                            p2 = __vmins2(__vmaxs2(p2, 0u), 0x000F000Fu);
                            b[h] = p2 | (p2 >> 12);  // byte 0: q of the pair's first weight | second << 4
                        }
                        packed[j] = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040),
                                                0x5410);
                    }
                } else {
#pragma unroll
                for (int j = 0; j < kWordsPerLane; ++j) {
                    uint32_t pw = 0u - kRintBase * 0x11111111u;
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        pw += rint_bits(fminf(fmaxf(__fadd_rn(quotient_rn(lane_weight<kBf16>(v[u], raw[u], 8 * j + i), s, r),
                                                              z), 0.0f), 15.0f))
                              << (4 * i);
                    packed[j] = pw;
                }
                }
            } else {
                z = round_bf16(__fadd_rn(rintf(__fdiv_rn(-mn, s)), 0.0f));
#pragma unroll
                for (int j = 0; j < kWordsPerLane; ++j) {
                    uint32_t pw = 0u - kRintBase * 0x11111111u;
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        pw += rint_bits(fminf(fmaxf(__fadd_rn(__fdiv_rn(lane_weight<kBf16>(v[u], raw[u], 8 * j + i), s), z),
                                                    0.0f), 15.0f)) << (4 * i);
                    packed[j] = pw;
                }
            }
            *reinterpret_cast<uint4 *>(qweight + n[u] * (K >> 1) + (k0[u] >> 1)) =
                make_uint4(packed[0], packed[1], packed[2], packed[3]);
            if ((lane & (LPG - 1)) == 0) {
                const int64_t gi = n[u] * Gn + k0[u] / G;
                scales[gi] = f32_to_bf16(s);
                zeros[gi] = f32_to_bf16(z);
            }
        }
    }
}

__device__ __forceinline__ float int8_scale(float amax)
{
    float s = round_bf16(div_by_const_rn(amax, 127.0f, kRcp127));
    return s == 0.0f ? 1.0f : s;
}

__device__ __forceinline__ uint2 int8_encode8(const float v[8], float s)
{
    float qd[8];  // RN(w / s); |w / s| <= 127.5, so only the scale's range decides the method
    if (quotients_by_reciprocal(s, 0.0f)) {
        const float r = __frcp_rn(s);
#pragma unroll
        for (int i = 0; i < 8; ++i) qd[i] = quotient_rn(v[i], s, r);
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) qd[i] = __fdiv_rn(v[i], s);
    }
    // q = clip(rint(RN(w / s)), -127, 127): clip, then rint_bits leaves the code in the low byte
    uint32_t b[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) b[i] = rint_bits(fminf(fmaxf(qd[i], -127.0f), 127.0f));
    const uint32_t lo = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
    const uint32_t hi = __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410);
    return make_uint2(lo, hi);
}

template <typename T, int LPG>
__global__ void __launch_bounds__(kQuantThreads)
quant_int8_group_kernel(const T *__restrict__ w, int64_t N, int64_t K, int64_t ldw,
                        int8_t *__restrict__ qweight, uint16_t *__restrict__ scales)
{
    constexpr int g = LPG * 8;
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t chunks = (K + 255) >> 8;
    const int64_t tasks = N * chunks;
    const int64_t G = K / g;

    TaskWalk walk(warp0, n_warps, chunks);
    for (int64_t t0 = warp0; t0 < tasks; t0 += n_warps * kQuantUnroll) {
        float v[kQuantUnroll][8];
        int64_t n[kQuantUnroll], k0[kQuantUnroll];
        bool active[kQuantUnroll];
#pragma unroll
        for (int u = 0; u < kQuantUnroll; ++u) {
            n[u] = walk.n;
            k0[u] = walk.c * 256 + lane * 8;
            active[u] = (walk.n < N) && (k0[u] < K);
            if (active[u]) load8<T>(w + n[u] * ldw + k0[u], v[u]);
            walk.step();
        }
#pragma unroll
        for (int u = 0; u < kQuantUnroll; ++u) {
            if (t0 + u * n_warps >= tasks) break;
            float amax = 0.0f;
            if (active[u]) {
#pragma unroll
                for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[u][i]));
            }
#pragma unroll
            for (int o = 1; o < LPG; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            if (!active[u]) continue;
            const float s = int8_scale(amax);
            *reinterpret_cast<uint2 *>(qweight + n[u] * K + k0[u]) = int8_encode8(v[u], s);
            if ((lane & (LPG - 1)) == 0) scales[n[u] * G + k0[u] / g] = f32_to_bf16(s);
        }
    }
}

// One scale per output channel: one CTA per row, absmax over the row, then a
// second pass over the same row (an L2 hit) to encode.
template <typename T>
__global__ void __launch_bounds__(kQuantThreads)
quant_int8_row_kernel(const T *__restrict__ w, int64_t N, int64_t K, int64_t ldw,
                      int8_t *__restrict__ qweight, uint16_t *__restrict__ scales)
{
    __shared__ float warp_max[kQuantThreads / 32];
    const int64_t n = blockIdx.x;
    const T *row = w + n * ldw;
    float amax = 0.0f;
    for (int64_t k = (int64_t)threadIdx.x * 8; k < K; k += kQuantThreads * 8) {
        float v[8];
        load8<T>(row + k, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = warp_max[0];
#pragma unroll
    for (int i = 1; i < kQuantThreads / 32; ++i) amax = fmaxf(amax, warp_max[i]);
    const float s = int8_scale(amax);
    if (threadIdx.x == 0) scales[n] = f32_to_bf16(s);
    for (int64_t k = (int64_t)threadIdx.x * 8; k < K; k += kQuantThreads * 8) {
        float v[8];
        const uint4 *src = reinterpret_cast<const uint4 *>(row + k);
        if (sizeof(T) == 2) {
            const uint4 a = ld_nc_v4(src);  // second read of the row: keep it cacheable
            const uint32_t u[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                v[2 * i] = __uint_as_float(u[i] << 16);
                v[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
            }
        } else {
            const uint4 a = ld_nc_v4(src), b = ld_nc_v4(src + 1);
            v[0] = __uint_as_float(a.x); v[1] = __uint_as_float(a.y);
            v[2] = __uint_as_float(a.z); v[3] = __uint_as_float(a.w);
            v[4] = __uint_as_float(b.x); v[5] = __uint_as_float(b.y);
            v[6] = __uint_as_float(b.z); v[7] = __uint_as_float(b.w);
        }
        *reinterpret_cast<uint2 *>(qweight + n * K + k) = int8_encode8(v, s);
    }
}

// The same for rows that fit in registers: each thread keeps its CH chunks of 8 weights (chunk i at
// k = 8 (256 i + thread)) as loaded, so the row crosses HBM once and the absmax and the encode read registers.
template <typename T, int CH>
__global__ void __launch_bounds__(kQuantThreads)
quant_int8_row_reg_kernel(const T *__restrict__ w, int64_t N, int64_t K, int64_t ldw,
                          int8_t *__restrict__ qweight, uint16_t *__restrict__ scales)
{
    constexpr int W = sizeof(T) == 2 ? 1 : 2;  // 16-byte words per chunk of 8 weights
    __shared__ float warp_max[kQuantThreads / 32];
    const int64_t n = blockIdx.x;
    const T *row = w + n * ldw;
    uint4 r[CH][W];
#pragma unroll
    for (int i = 0; i < CH; ++i) {
        const int64_t k = ((int64_t)i * kQuantThreads + threadIdx.x) * 8;
#pragma unroll
        for (int j = 0; j < W; ++j)
            r[i][j] = k < K ? ld_stream_v4(row + k + 4 * j) : make_uint4(0u, 0u, 0u, 0u);
    }
    auto unpack = [&](int i, float v[8]) {
        if (sizeof(T) == 2) {
            const uint32_t u[4] = {r[i][0].x, r[i][0].y, r[i][0].z, r[i][0].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                v[2 * e] = __uint_as_float(u[e] << 16);
                v[2 * e + 1] = __uint_as_float(u[e] & 0xffff0000u);
            }
        } else {
            const uint4 a = r[i][0], b = r[i][W - 1];
            v[0] = __uint_as_float(a.x); v[1] = __uint_as_float(a.y);
            v[2] = __uint_as_float(a.z); v[3] = __uint_as_float(a.w);
            v[4] = __uint_as_float(b.x); v[5] = __uint_as_float(b.y);
            v[6] = __uint_as_float(b.z); v[7] = __uint_as_float(b.w);
        }
    };
    float amax = 0.0f;  // chunks past K hold zeros
#pragma unroll
    for (int i = 0; i < CH; ++i) {
        float v[8];
        unpack(i, v);
#pragma unroll
        for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[e]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = warp_max[0];
#pragma unroll
    for (int i = 1; i < kQuantThreads / 32; ++i) amax = fmaxf(amax, warp_max[i]);
    const float s = int8_scale(amax);
    if (threadIdx.x == 0) scales[n] = f32_to_bf16(s);
#pragma unroll
    for (int i = 0; i < CH; ++i) {
        const int64_t k = ((int64_t)i * kQuantThreads + threadIdx.x) * 8;
        if (k < K) {
            float v[8];
            unpack(i, v);
            *reinterpret_cast<uint2 *>(qweight + n * K + k) = int8_encode8(v, s);
        }
    }
}

// Symmetric INT4 ("Test-time quantization: quantising on the fly with no calibration dataset", section
// "The error of quantising an outlier with the wrong scale": s = M / (2^(b-1) - 1) = max|w| / 7 at 4
// bits; the comparison page's AWQ example: codes -7 to 7).  q = clip(rint(RN(w / s)), -7, 7), stored as
// the nibble q + 8 with a zero-point of 8, so the asymmetric decode s (code - z) reads it as s q.
__device__ __forceinline__ float int4_sym_scale(float amax)
{
    float s = round_bf16(div_by_const_rn(amax, 7.0f, kRcp7));
    return s == 0.0f ? 1.0f : s;
}

// The layout of quant_int4_kernel: a lane takes 32 consecutive weights of a row, a group of G spans G / 32
// lanes, the scale is formed once per 32 weights; for bf16 weights the absolute maximum is reduced as a
// packed bf16 pair and, on the reciprocal path, two quotients are formed per instruction.
template <typename T, int G>
__global__ void __launch_bounds__(kQuantThreads)
quant_int4_sym_kernel(const T *__restrict__ w, int64_t N, int64_t K, int64_t ldw, uint8_t *__restrict__ qweight,
                      uint16_t *__restrict__ scales, uint16_t *__restrict__ zeros)
{
    constexpr int LPG = G / kLaneWeights;  // lanes per group
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t chunks = (K + kWarpWeights - 1) / kWarpWeights;
    const int64_t tasks = N * chunks;
    const int64_t Gn = K / G;

    TaskWalk walk(warp0, n_warps, chunks);
    for (int64_t t0 = warp0; t0 < tasks; t0 += n_warps * kInt4Unroll) {
        float v[kInt4Unroll][kBf16 ? 1 : kLaneWeights];  // binary32 input
        uint4 raw[kInt4Unroll][kWordsPerLane];             // bf16 input: the weights as loaded
        int64_t n[kInt4Unroll], k0[kInt4Unroll];
        bool active[kInt4Unroll];
#pragma unroll
        for (int u = 0; u < kInt4Unroll; ++u) {
            n[u] = walk.n;
            k0[u] = walk.c * kWarpWeights + lane * kLaneWeights;
            active[u] = (walk.n < N) && (k0[u] < K);
            if (kBf16) {
#pragma unroll
                for (int j = 0; j < kWordsPerLane; ++j) raw[u][j] = make_uint4(0u, 0u, 0u, 0u);
                if (active[u]) {
#pragma unroll
                    for (int j = 0; j < kWordsPerLane; ++j) raw[u][j] = ld_stream_v4(w + n[u] * ldw + k0[u] + 8 * j);
                }
            } else if (active[u]) {
#pragma unroll
                for (int j = 0; j < kWordsPerLane; ++j) load8<T>(w + n[u] * ldw + k0[u] + 8 * j, v[u] + 8 * j);
            }
            walk.step();
        }
#pragma unroll
        for (int u = 0; u < kInt4Unroll; ++u) {
            if (t0 + u * n_warps >= tasks) break;  // warp-uniform
            float amax;
            if (kBf16) {
                // |w| of both halves (sign bits cleared), the packed maximum over the lane's 32 weights and then
                // over the group's lanes (inactive lanes hold zeros)
                uint32_t m2 = 0u;
#pragma unroll
                for (int j = 0; j < kWordsPerLane; ++j)
                    m2 = bf16x2_max(m2, bf16x2_max(bf16x2_max(raw[u][j].x & 0x7FFF7FFFu, raw[u][j].y & 0x7FFF7FFFu),
                                                   bf16x2_max(raw[u][j].z & 0x7FFF7FFFu, raw[u][j].w & 0x7FFF7FFFu)));
#pragma unroll
                for (int o = 1; o < LPG; o <<= 1) m2 = bf16x2_max(m2, __shfl_xor_sync(0xffffffffu, m2, o));
                amax = fmaxf(__uint_as_float(m2 << 16), __uint_as_float(m2 & 0xffff0000u));
            } else {
                amax = 0.0f;
                if (active[u]) {
#pragma unroll
                    for (int i = 0; i < kLaneWeights; ++i) amax = fmaxf(amax, fabsf(v[u][i]));
                }
#pragma unroll
                for (int o = 1; o < LPG; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            }
            if (!active[u]) continue;
            const float s = int4_sym_scale(amax);
            uint32_t packed[kWordsPerLane];
            if (quotients_by_reciprocal(s, amax)) {
                const float r = __frcp_rn(s);
                if (kBf16) {
                    // two weights per instruction: the correctly rounded quotients (packed binary32 multiply and
                    // fused multiply-adds), then + 8 + 1.5 * 2^23 in one addition, which rounds (rint(q + 8) =
                    // rint(q) + 8: 8 is even); |w / s| < 8 here, so each rounded q + 8 is the low half-word of
                    // its bit pattern, clipped to [1, 15] (q to [-7, 7]) as two 16-bit integers
                    const uint64_t r2 = f32x2_bits(r, r), ns2 = f32x2_bits(-s, -s);
                    const uint64_t m2 = f32x2_bits(0x1.8p23f + 8.0f, 0x1.8p23f + 8.0f);
#pragma unroll
                    for (int j = 0; j < kWordsPerLane; ++j) {
                        uint32_t b[4];
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            const uint32_t wd = word_of(raw[u][j], h);
                            const uint64_t w2 = ((uint64_t)(wd & 0xffff0000u) << 32) | (uint64_t)(wd << 16);
                            const uint64_t q0 = f32x2_mul(w2, r2);
                            const uint64_t q = f32x2_fma(f32x2_fma(q0, ns2, w2), r2, q0);
                            const uint64_t t = f32x2_add(q, m2);
                            uint32_t p2 = __byte_perm((uint32_t)t, (uint32_t)(t >> 32), 0x5410);
                            p2 = __vmins2(__vmaxs2(p2, 0x00010001u), 0x000F000Fu);
                            b[h] = p2 | (p2 >> 12);  // byte 0: q + 8 of the pair's first weight | second << 4
                        }
                        packed[j] = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040),
                                                0x5410);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < kWordsPerLane; ++j) {
                        // rint_bits leaves q (two's complement) in the low bits: the shifted patterns summed, minus
                        // their offsets, plus 8 in every nibble, are the eight nibbles q + 8 (1..15, no carries)
                        uint32_t pw = 0x88888888u - kRintBase * 0x11111111u;
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            pw += rint_bits(fminf(fmaxf(quotient_rn(v[u][8 * j + i], s, r), -7.0f), 7.0f)) << (4 * i);
                        packed[j] = pw;
                    }
                }
            } else {
#pragma unroll
                for (int j = 0; j < kWordsPerLane; ++j) {
                    uint32_t pw = 0x88888888u - kRintBase * 0x11111111u;
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        pw += rint_bits(fminf(fmaxf(__fdiv_rn(lane_weight<kBf16>(v[u], raw[u], 8 * j + i), s), -7.0f),
                                              7.0f))
                              << (4 * i);
                    packed[j] = pw;
                }
            }
            *reinterpret_cast<uint4 *>(qweight + n[u] * (K >> 1) + (k0[u] >> 1)) =
                make_uint4(packed[0], packed[1], packed[2], packed[3]);
            if ((lane & (LPG - 1)) == 0) {
                const int64_t gi = n[u] * Gn + k0[u] / G;
                scales[gi] = f32_to_bf16(s);
                zeros[gi] = 0x4100u;  // 8.0 in bf16
            }
        }
    }
}

// Grid of a persistent quantiser: enough CTAs for the work, at most the resident capacity of the device
// (SMs x resident CTAs of this kernel), which is looked up once per kernel and device.
template <typename KernelT>
int persistent_grid(KernelT kernel, int64_t tasks_in_warps)
{
    static std::mutex mu;
    static std::map<std::pair<int, const void *>, int64_t> cap_of;  // (device, kernel) -> capacity
    int dev = 0;
    cudaGetDevice(&dev);
    const std::pair<int, const void *> key(dev, reinterpret_cast<const void *>(kernel));
    int64_t cap;
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = cap_of.find(key);
        if (it == cap_of.end()) {
            int sms = 148, per_sm = 1;
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kQuantThreads, 0);
            it = cap_of.emplace(key, (int64_t)sms * (per_sm < 1 ? 1 : per_sm)).first;
        }
        cap = it->second;
    }
    const int64_t want = (tasks_in_warps + (kQuantThreads / 32) - 1) / (kQuantThreads / 32);
    return (int)(want < cap ? (want > 0 ? want : 1) : cap);
}

template <typename T, int G, bool SCALED>
void launch_int4(const void *w, int64_t N, int64_t K, int64_t ldw, uint8_t *q, uint16_t *s, uint16_t *z,
                 const float *cs, cudaStream_t st)
{
    auto k = quant_int4_kernel<T, G, SCALED>;
    const int64_t tasks = N * ((K + kWarpWeights - 1) / kWarpWeights);
    const int grid = persistent_grid(k, tasks);
    k<<<grid, kQuantThreads, 0, st>>>(static_cast<const T *>(w), N, K, ldw, q, s, z, cs);
}

template <typename T, int LPG>
void launch_int8(const void *w, int64_t N, int64_t K, int64_t ldw, int8_t *q, uint16_t *s, cudaStream_t st)
{
    auto k = quant_int8_group_kernel<T, LPG>;
    const int64_t tasks = N * ((K + 255) / 256);
    const int grid = persistent_grid(k, tasks);
    k<<<grid, kQuantThreads, 0, st>>>(static_cast<const T *>(w), N, K, ldw, q, s);
}

template <typename T, bool SCALED>
void dispatch_int4(const void *w, int64_t N, int64_t K, int64_t ldw, int g, uint8_t *q, uint16_t *s,
                   uint16_t *z, const float *cs, cudaStream_t st)
{
    switch (g) {
    case 32: launch_int4<T, 32, SCALED>(w, N, K, ldw, q, s, z, cs, st); break;
    case 64: launch_int4<T, 64, SCALED>(w, N, K, ldw, q, s, z, cs, st); break;
    default: launch_int4<T, 128, SCALED>(w, N, K, ldw, q, s, z, cs, st); break;
    }
}

template <typename T, int G>
void launch_int4_sym(const void *w, int64_t N, int64_t K, int64_t ldw, uint8_t *q, uint16_t *s, uint16_t *z,
                     cudaStream_t st)
{
    auto k = quant_int4_sym_kernel<T, G>;
    const int64_t tasks = N * ((K + kWarpWeights - 1) / kWarpWeights);
    const int grid = persistent_grid(k, tasks);
    k<<<grid, kQuantThreads, 0, st>>>(static_cast<const T *>(w), N, K, ldw, q, s, z);
}

template <typename T>
void dispatch_int4_sym(const void *w, int64_t N, int64_t K, int64_t ldw, int g, uint8_t *q, uint16_t *s,
                       uint16_t *z, cudaStream_t st)
{
    switch (g) {
    case 32: launch_int4_sym<T, 32>(w, N, K, ldw, q, s, z, st); break;
    case 64: launch_int4_sym<T, 64>(w, N, K, ldw, q, s, z, st); break;
    default: launch_int4_sym<T, 128>(w, N, K, ldw, q, s, z, st); break;
    }
}

template <typename T>
void dispatch_int8(const void *w, int64_t N, int64_t K, int64_t ldw, int g, int8_t *q, uint16_t *s,
                   cudaStream_t st)
{
    if (g == K) {
        // one read of the row when it fits in registers (up to 8 chunks of 8 per thread: K <= 16384; 16 chunks
        // were slower than two passes at K = 28672, B200)
        const int64_t per = (K / 8 + kQuantThreads - 1) / kQuantThreads;
        const T *wt = static_cast<const T *>(w);
        if (per <= 4) quant_int8_row_reg_kernel<T, 4><<<(unsigned)N, kQuantThreads, 0, st>>>(wt, N, K, ldw, q, s);
        else if (per <= 8) quant_int8_row_reg_kernel<T, 8><<<(unsigned)N, kQuantThreads, 0, st>>>(wt, N, K, ldw, q, s);
        else quant_int8_row_kernel<T><<<(unsigned)N, kQuantThreads, 0, st>>>(wt, N, K, ldw, q, s);
        return;
    }
    switch (g) {
    case 32: launch_int8<T, 4>(w, N, K, ldw, q, s, st); break;
    case 64: launch_int8<T, 8>(w, N, K, ldw, q, s, st); break;
    default: launch_int8<T, 16>(w, N, K, ldw, q, s, st); break;
    }
}

}  // namespace

void launch_quantize_int4(const void *w, int wtype, int64_t N, int64_t K, int64_t ldw, int g, uint8_t *q,
                          uint16_t *s, uint16_t *z, cudaStream_t st)
{
    if (wtype == WQ_F32) dispatch_int4<float, false>(w, N, K, ldw, g, q, s, z, nullptr, st);
    else dispatch_int4<__nv_bfloat16, false>(w, N, K, ldw, g, q, s, z, nullptr, st);
}

void launch_quantize_int4_scaled(const void *w, int wtype, int64_t N, int64_t K, int64_t ldw, int g,
                                 const float *col_scale, uint8_t *q, uint16_t *s, uint16_t *z, cudaStream_t st)
{
    if (wtype == WQ_F32) dispatch_int4<float, true>(w, N, K, ldw, g, q, s, z, col_scale, st);
    else dispatch_int4<__nv_bfloat16, true>(w, N, K, ldw, g, q, s, z, col_scale, st);
}

void launch_quantize_int4_sym(const void *w, int wtype, int64_t N, int64_t K, int64_t ldw, int g, uint8_t *q,
                              uint16_t *s, uint16_t *z, cudaStream_t st)
{
    if (wtype == WQ_F32) dispatch_int4_sym<float>(w, N, K, ldw, g, q, s, z, st);
    else dispatch_int4_sym<__nv_bfloat16>(w, N, K, ldw, g, q, s, z, st);
}

void launch_quantize_int8(const void *w, int wtype, int64_t N, int64_t K, int64_t ldw, int g, int8_t *q,
                          uint16_t *s, cudaStream_t st)
{
    if (wtype == WQ_F32) dispatch_int8<float>(w, N, K, ldw, g, q, s, st);
    else dispatch_int8<__nv_bfloat16>(w, N, K, ldw, g, q, s, st);
}

}  // namespace wq

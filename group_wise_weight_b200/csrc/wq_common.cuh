// wq_common.cuh -- device helpers shared by the libwq kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/wq.h"

namespace wq {

constexpr int kWarp = 32;

// ---------------------------------------------------------------------------
// Status word for bounded waits (see wq_device_status).  Kernels that wait
// on barriers receive its device address as an argument.
// ---------------------------------------------------------------------------
enum DeviceStatus : int { kStatusOk = 0, kStatusTimeout = 1 };

__device__ __forceinline__ void record_timeout(int *status) { atomicExch(status, kStatusTimeout); }

// ---------------------------------------------------------------------------
// Loads.  Packed weights are read once per call: stream them past L1.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 ld_stream_v4(const void *p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ uint4 ld_nc_v4(const void *p)
{
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ uint32_t ld_nc_u32(const uint32_t *p)
{
    uint32_t r;
    asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(r) : "l"(p));
    return r;
}

__device__ __forceinline__ uint16_t ld_nc_u16(const uint16_t *p)
{
    uint16_t r;
    asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(r) : "l"(p));
    return r;
}

// ---------------------------------------------------------------------------
// bf16 <-> binary32, both round-to-nearest-even.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16_to_f32(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }

__device__ __forceinline__ uint16_t f32_to_bf16(float f)
{
    __nv_bfloat16 b = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t *>(&b);
}

// Round a binary32 to its bf16 value and widen back.
__device__ __forceinline__ float round_bf16(float f) { return bf16_to_f32(f32_to_bf16(f)); }

// Pack two binary32 into a bf16x2 word (lo = a, hi = b), each rounded to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b)
{
    return (uint32_t)f32_to_bf16(a) | ((uint32_t)f32_to_bf16(b) << 16);
}

// (128 + q) - (128 + z) on a bf16 pair: exact for the integers of a code and a zero-point (any integer of
// magnitude <= 256 is a bf16 value), so a matmul operand built this way holds q - z itself.
__device__ __forceinline__ uint32_t sub_bf16x2(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Zero-points outside [0, 15].  z = round(-min / s) is not clamped, so a group that lies on one side of
// zero, far from it compared with its width, has |z| up to thousands, and neither 128 + z nor q - z need
// fit bf16's 8 significant bits.  The kernels then split z = z_hi + z_lo with z_lo in [0, 16) and z_hi a
// multiple of 16: (128 + q) - (128 + z_lo) = q - z_lo is exact, and -z_hi times the group's activation sum
// is added in binary32 (whose rounding is tiny next to s |q - z| sum |x|, since |q - z| >= |z_hi| - 15).
// Returns z_lo; z is an integer.
__device__ __forceinline__ float zp_split(float z, float &z_hi)
{
    z_hi = floorf(z * 0.0625f) * 16.0f;
    return z - z_hi;
}

// bf16 pair (128 + v, 128 + v) for an integer v in [0, 16): exact.
__device__ __forceinline__ uint32_t bf16_pair_128_plus(float v)
{
    return (__float_as_uint(128.0f + v) >> 16) * 0x10001u;
}

// Both halves of a bf16 pair (128 + z0, 128 + z1), formed by one bf16 addition, hold 128 .. 143,
// i.e. z0 and z1 are integers in [0, 15] and the pair is exact.
__device__ __forceinline__ bool zz_pair_in_range(uint32_t zz)
{
    return ((zz ^ 0x43004300u) & 0xFFF0FFF0u) == 0u;
}

// Sum of the 8 bf16 values of a uint4, in binary32, in a fixed order.
__device__ __forceinline__ float sum_bf16x8(const uint4 &v)
{
    float t = __uint_as_float(v.x << 16) + __uint_as_float(v.x & 0xffff0000u);
    t += __uint_as_float(v.y << 16);
    t += __uint_as_float(v.y & 0xffff0000u);
    t += __uint_as_float(v.z << 16);
    t += __uint_as_float(v.z & 0xffff0000u);
    t += __uint_as_float(v.w << 16);
    t += __uint_as_float(v.w & 0xffff0000u);
    return t;
}

// ---------------------------------------------------------------------------
// Mixed-precision FMA: d = a * b + c with bf16 a, b and binary32 c, d
// (the product of two bf16 is exact in binary32; one rounding).
// ---------------------------------------------------------------------------
__device__ __forceinline__ float fma_bf16_lo(uint32_t a2, uint32_t b2, float c)
{
    float d;
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
        "mov.b32 {al, ah}, %1;\n\t"
        "mov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, al, bl, %3;\n\t}"
        : "=f"(d)
        : "r"(a2), "r"(b2), "f"(c));
    return d;
}

__device__ __forceinline__ float fma_bf16_hi(uint32_t a2, uint32_t b2, float c)
{
    float d;
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
        "mov.b32 {al, ah}, %1;\n\t"
        "mov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, ah, bh, %3;\n\t}"
        : "=f"(d)
        : "r"(a2), "r"(b2), "f"(c));
    return d;
}

// Dot-accumulate both halves: c + a.lo * b.lo + a.hi * b.hi.
__device__ __forceinline__ float fma_bf16x2(uint32_t a2, uint32_t b2, float c)
{
    return fma_bf16_hi(a2, b2, fma_bf16_lo(a2, b2, c));
}

// Packed binary32 pair arithmetic (two lanes per instruction on sm_100).
struct f32x2 {
    float x, y;
};

__device__ __forceinline__ f32x2 fma2(f32x2 a, f32x2 b, f32x2 c)
{
    uint64_t r;
    uint64_t ua = ((uint64_t)__float_as_uint(a.y) << 32) | __float_as_uint(a.x);
    uint64_t ub = ((uint64_t)__float_as_uint(b.y) << 32) | __float_as_uint(b.x);
    uint64_t uc = ((uint64_t)__float_as_uint(c.y) << 32) | __float_as_uint(c.x);
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(ua), "l"(ub), "l"(uc));
    return f32x2{__uint_as_float((uint32_t)r), __uint_as_float((uint32_t)(r >> 32))};
}

// The same product-sum with the pairs joined and split inside the asm, so the compiler can keep each
// pair in an aligned register pair (cheaper where the operands come from loads and stay in pairs, as in
// the tensor-core kernel's promotion).
__device__ __forceinline__ f32x2 fma2_pairs(f32x2 a, f32x2 b, f32x2 c)
{
    f32x2 r;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\t"
        "mov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\t"
        "mov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return r;
}

__device__ __forceinline__ f32x2 add2(f32x2 a, f32x2 b)
{
    uint64_t r;
    uint64_t ua = ((uint64_t)__float_as_uint(a.y) << 32) | __float_as_uint(a.x);
    uint64_t ub = ((uint64_t)__float_as_uint(b.y) << 32) | __float_as_uint(b.x);
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(ua), "l"(ub));
    return f32x2{__uint_as_float((uint32_t)r), __uint_as_float((uint32_t)(r >> 32))};
}

// ---------------------------------------------------------------------------
// 4-bit code extraction.  (v >> sh) & 0x000F000F | 0x43004300 places the
// nibbles at bit sh and sh+16 into the mantissas of two bf16 values equal to
// 128 + code (exact: bf16 has an ulp of 1 on [128, 256)).  For a word holding
// codes c0..c7 (c_i in bits 4i..4i+3) the four shifts 0, 4, 8, 12 give the
// pairs (c0, c4), (c1, c5), (c2, c6), (c3, c7).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t nib_pair_bf16(uint32_t v, int sh)
{
    return ((v >> sh) & 0x000F000Fu) | 0x43004300u;  // one LOP3 after the shift
}

// Warp-wide sum.
__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

}  // namespace wq

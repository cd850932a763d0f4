// wq_quant.cu -- group-wise INT4 (asymmetric) and INT8 (symmetric absmax)
// quantisation kernels.
//
// Asymmetric INT4 follows "Quantization for LLM inference: FP8, INT4 (GPTQ,
// AWQ) and GGUF", section "The minimum maths: scale and zero-point":
// s = (max - min) / 15, z = round(-min / s), q = clip(round(w / s + z), 0, 15).
// Symmetric INT8 follows "Quantization Methods Compared: INT8, GPTQ, AWQ, FP8,
// FP4 and KV-Cache Quantization", section "What quantisation does":
// s = max|w| / 127, q = round(w / s).
//
// Both are HBM streams (read 2 or 4 B per weight, write 0.5 or 1 B plus the
// per-group parameters).  Layout of the work: a warp takes 256 consecutive
// weights of one row, 8 per lane (one 16-byte load for bf16), so a group of
// g weights spans g/8 adjacent lanes and its min/max (or absmax) is a
// log2(g/8)-step xor-shuffle reduction.  Every lane then derives the same
// (s, z) and encodes its 8 weights into one 32-bit word of nibbles (INT4) or
// one 64-bit word of bytes (INT8); stores are 128 contiguous bytes per warp.
//
// Arithmetic matches the library contract bit for bit: binary32 with
// explicit round-to-nearest-even intrinsics (no contraction is possible),
// rintf (round half to even), bf16 rounding to nearest even.
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

// s, z of one INT4 group from its min and max (the library contract).
__device__ __forceinline__ void int4_params(float mn, float mx, float &s, float &z)
{
    s = round_bf16(__fdiv_rn(__fsub_rn(mx, mn), 15.0f));
    if (s == 0.0f) {
        s = round_bf16(fmaxf(fabsf(mn), fabsf(mx)));
        if (s == 0.0f) s = 1.0f;
    }
    z = round_bf16(__fadd_rn(rintf(__fdiv_rn(-mn, s)), 0.0f));
}

template <typename T, int LPG>
__global__ void __launch_bounds__(kQuantThreads)
quant_int4_kernel(const T *__restrict__ w, int64_t N, int64_t K, int64_t ldw,
                  uint8_t *__restrict__ qweight, uint16_t *__restrict__ scales,
                  uint16_t *__restrict__ zeros)
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
            if (t0 + u * n_warps >= tasks) break;  // warp-uniform
            float mn = INFINITY, mx = -INFINITY;
            if (active[u]) {
#pragma unroll
                for (int i = 0; i < 8; ++i) { mn = fminf(mn, v[u][i]); mx = fmaxf(mx, v[u][i]); }
            }
#pragma unroll
            for (int o = 1; o < LPG; o <<= 1) {
                mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            }
            if (!active[u]) continue;
            float s, z;
            int4_params(mn, mx, s, z);
            float qd[8];  // RN(w / s)
            if (quotients_by_reciprocal(s, fmaxf(fabsf(mn), fabsf(mx)))) {
                const float r = __frcp_rn(s);
#pragma unroll
                for (int i = 0; i < 8; ++i) qd[i] = quotient_rn(v[u][i], s, r);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) qd[i] = __fdiv_rn(v[u][i], s);
            }
            uint32_t packed = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float q = rintf(__fadd_rn(qd[i], z));
                q = fminf(fmaxf(q, 0.0f), 15.0f);
                packed |= (uint32_t)q << (4 * i);
            }
            *reinterpret_cast<uint32_t *>(qweight + n[u] * (K >> 1) + (k0[u] >> 1)) = packed;
            if ((lane & (LPG - 1)) == 0) {
                const int64_t gi = n[u] * G + k0[u] / g;
                scales[gi] = f32_to_bf16(s);
                zeros[gi] = f32_to_bf16(z);
            }
        }
    }
}

__device__ __forceinline__ float int8_scale(float amax)
{
    float s = round_bf16(__fdiv_rn(amax, 127.0f));
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
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float q = rintf(qd[i]);
        q = fminf(fmaxf(q, -127.0f), 127.0f);
        const uint32_t b = (uint32_t)(int)q & 0xffu;
        if (i < 4) lo |= b << (8 * i); else hi |= b << (8 * (i - 4));
    }
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

template <typename KernelT>
int persistent_grid(KernelT kernel, int64_t tasks_in_warps)
{
    int dev = 0, sms = 148, per_sm = 1;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kQuantThreads, 0);
    if (per_sm < 1) per_sm = 1;
    const int64_t want = (tasks_in_warps + (kQuantThreads / 32) - 1) / (kQuantThreads / 32);
    const int64_t cap = (int64_t)sms * per_sm;
    return (int)(want < cap ? (want > 0 ? want : 1) : cap);
}

template <typename T, int LPG>
void launch_int4(const void *w, int64_t N, int64_t K, int64_t ldw, uint8_t *q, uint16_t *s, uint16_t *z,
                 cudaStream_t st)
{
    auto k = quant_int4_kernel<T, LPG>;
    const int64_t tasks = N * ((K + 255) / 256);
    const int grid = persistent_grid(k, tasks);
    k<<<grid, kQuantThreads, 0, st>>>(static_cast<const T *>(w), N, K, ldw, q, s, z);
}

template <typename T, int LPG>
void launch_int8(const void *w, int64_t N, int64_t K, int64_t ldw, int8_t *q, uint16_t *s, cudaStream_t st)
{
    auto k = quant_int8_group_kernel<T, LPG>;
    const int64_t tasks = N * ((K + 255) / 256);
    const int grid = persistent_grid(k, tasks);
    k<<<grid, kQuantThreads, 0, st>>>(static_cast<const T *>(w), N, K, ldw, q, s);
}

template <typename T>
void dispatch_int4(const void *w, int64_t N, int64_t K, int64_t ldw, int g, uint8_t *q, uint16_t *s,
                   uint16_t *z, cudaStream_t st)
{
    switch (g) {
    case 32: launch_int4<T, 4>(w, N, K, ldw, q, s, z, st); break;
    case 64: launch_int4<T, 8>(w, N, K, ldw, q, s, z, st); break;
    default: launch_int4<T, 16>(w, N, K, ldw, q, s, z, st); break;
    }
}

template <typename T>
void dispatch_int8(const void *w, int64_t N, int64_t K, int64_t ldw, int g, int8_t *q, uint16_t *s,
                   cudaStream_t st)
{
    if (g == K) {
        quant_int8_row_kernel<T><<<(unsigned)N, kQuantThreads, 0, st>>>(static_cast<const T *>(w), N, K, ldw, q, s);
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
    if (wtype == WQ_F32) dispatch_int4<float>(w, N, K, ldw, g, q, s, z, st);
    else dispatch_int4<__nv_bfloat16>(w, N, K, ldw, g, q, s, z, st);
}

void launch_quantize_int8(const void *w, int wtype, int64_t N, int64_t K, int64_t ldw, int g, int8_t *q,
                          uint16_t *s, cudaStream_t st)
{
    if (wtype == WQ_F32) dispatch_int8<float>(w, N, K, ldw, g, q, s, st);
    else dispatch_int8<__nv_bfloat16>(w, N, K, ldw, g, q, s, st);
}

}  // namespace wq

// wq_lowp.cuh -- helpers shared by the FP8 and NVFP4 quantisers: loads of
// eight inputs widened to binary32, a block-wide maximum, and the grid-wide
// largest magnitude of a tensor.
#pragma once

#include "wq_common.cuh"

namespace wq {
namespace lowp {

constexpr int kThreads = 256;

// Eight consecutive inputs widened to binary32 (exact for bf16).
template <typename T>
__device__ __forceinline__ void ld8(const T *p, float v[8]);

template <>
__device__ __forceinline__ void ld8<float>(const float *p, float v[8])
{
    const float4 a = *reinterpret_cast<const float4 *>(p);
    const float4 b = *reinterpret_cast<const float4 *>(p + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

template <>
__device__ __forceinline__ void ld8<uint16_t>(const uint16_t *p, float v[8])
{
    const uint4 a = *reinterpret_cast<const uint4 *>(p);
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

__device__ __forceinline__ float block_max(float v, float *red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[wid] = v;
    __syncthreads();
    if (wid == 0) {
        v = lane < (int)(blockDim.x >> 5) ? red[lane] : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0) red[0] = v;
    }
    __syncthreads();
    v = red[0];
    __syncthreads();
    return v;
}

// Grid-wide largest magnitude of a dense tensor of `count` values (count % 8 == 0) into *amax_bits,
// which must hold 0 (the bit pattern of +0) before the launch.
template <typename T>
__global__ void __launch_bounds__(kThreads)
tensor_amax_kernel(const T *__restrict__ x, int64_t count, unsigned int *__restrict__ amax_bits)
{
    __shared__ float red[32];
    float amax = 0.0f;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x * 8;
    for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 8; i < count; i += stride) {
        float v[8];
        ld8<T>(x + i, v);
#pragma unroll
        for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(v[j]));
    }
    amax = block_max(amax, red);
    if (threadIdx.x == 0) atomicMax(amax_bits, __float_as_uint(amax));
}

}  // namespace lowp
}  // namespace wq

// wq_quant_nvfp4.cu -- NVFP4 quantisation: E2M1 values, one E4M3 scale per
// block of 16 consecutive values of a row, one binary32 scale per tensor.
//
// "Quantization Methods Compared: INT8, GPTQ, AWQ, FP8, FP4 and KV-Cache
// Quantization", section "Hardware, formats and the roofline": NVFP4 is the
// Blackwell-native 4-bit format, 4-bit values with an 8-bit E4M3 scale per
// 16 values and an fp32 tensor scale (4.5 bits per value); "Quantization for
// LLM inference: FP8, INT4 (GPTQ, AWQ) and GGUF", section "Microscaling:
// NVFP4 and MXFP4".  The pages define neither the 4-bit values nor how the
// scales are chosen; the reading used here, in binary32:
//   st   = max|w over the tensor| / (6 * 448)        (1 when that is 0)
//   sb   = E4M3 code of ((max|w over the block| / 6) / st)
//   S    = e4m3(sb) * st
//   code = nearest E2M1 value (0, 0.5, 1, 1.5, 2, 3, 4, 6 and negatives) to
//          w / S, ties to the even code, saturated at +-6; 0 when S == 0.
// Every division is IEEE; the conversions are the hardware's
// cvt.rn.satfinite (round to nearest even, saturate finite values).
//
// Storage (what the NVFP4 tensor-core matmul reads):
//  * codes [N][K/2] bytes, element 2j of a row in the low nibble of byte j;
//  * block scales in the layout tcgen05.mma's block-scaled kinds take from
//    tensor memory after a 32x128b.warpx4 copy: 512-byte atoms of 128 rows x
//    4 blocks (64 values of K), the scale of (row r, block b) at byte
//    16 (r % 32) + 4 ((r % 128) / 32) + (b % 4) of atom
//    (r / 128) * (K / 64) + b / 4; rows are padded to a multiple of 128
//    (padding scales 0);
//  * the tensor scale, one binary32 value on the device.
// A thread takes one block of 16 values (two 16-byte loads for bf16 input),
// so the pass is an HBM stream; the tensor maximum is a separate pass.
#include "wq_internal.h"
#include "wq_lowp.cuh"

namespace wq {

namespace {

constexpr int kThreads = lowp::kThreads;

// E4M3 code (saturated, round to nearest even) of a non-negative v, in the low byte.
__device__ __forceinline__ uint32_t e4m3_code(float v)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
    return r & 0xffu;
}

// Value of a non-negative E4M3 code (exact): subnormals m * 2^-9, normals (1 + m/8) 2^(e-7).
__device__ __forceinline__ float e4m3_value(uint32_t c)
{
    const uint32_t e = (c >> 3) & 15u, m = c & 7u;
    return e == 0 ? (float)m * 0x1p-9f : __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Two E2M1 codes (round to nearest even, saturate at +-6): lo in bits 0-3, hi in bits 4-7.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi)
{
    uint16_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tmov.b16 %0, {t, 0};\n\t}"
        : "=h"(r)
        : "f"(hi), "f"(lo));
    return r & 0xffu;
}

__device__ __forceinline__ float tensor_scale_of(float amax)
{
    const float st = __fdiv_rn(amax, 6.0f * 448.0f);
    return st == 0.0f ? 1.0f : st;
}

// Byte offset of the scale of (row r, block b) in the tensor-core layout (K/64 atoms per 128-row tile).
__host__ __device__ __forceinline__ int64_t sf_offset(int64_t r, int64_t b, int64_t K)
{
    return ((r >> 7) * (K >> 6) + (b >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (b & 3);
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
nvfp4_encode_kernel(const T *__restrict__ w, int64_t N, int64_t K, int64_t ldw, const float *__restrict__ amax,
                    uint8_t *__restrict__ codes, uint8_t *__restrict__ sf)
{
    const float st = tensor_scale_of(*amax);
    const int64_t nb = K >> 4;  // blocks per row
    const int64_t blocks = N * nb;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < blocks; i += stride) {
        const int64_t n = i / nb, b = i - n * nb;
        float v[16];
        lowp::ld8<T>(w + n * ldw + b * 16, v);
        lowp::ld8<T>(w + n * ldw + b * 16 + 8, v + 8);
        float bmax = 0.0f;
#pragma unroll
        for (int j = 0; j < 16; ++j) bmax = fmaxf(bmax, fabsf(v[j]));
        const uint32_t sc = e4m3_code(__fdiv_rn(__fdiv_rn(bmax, 6.0f), st));
        const float S = e4m3_value(sc) * st;
        uint32_t word[2] = {0u, 0u};
        if (S != 0.0f) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
                word[j >> 2] |= e2m1x2(__fdiv_rn(v[2 * j], S), __fdiv_rn(v[2 * j + 1], S)) << (8 * (j & 3));
        }
        *reinterpret_cast<uint2 *>(codes + n * (K >> 1) + b * 8) = make_uint2(word[0], word[1]);
        sf[sf_offset(n, b, K)] = (uint8_t)sc;
    }
}

// Largest magnitude of the first K values of N rows of stride ldw into *amax_bits (which must hold 0).
template <typename T>
__global__ void __launch_bounds__(kThreads)
rows_amax_kernel(const T *__restrict__ w, int64_t N, int64_t K, int64_t ldw, unsigned int *__restrict__ amax_bits)
{
    __shared__ float red[32];
    const int64_t per_row = K >> 3, chunks = N * per_row;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    float amax = 0.0f;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < chunks; i += stride) {
        const int64_t n = i / per_row, c = i - n * per_row;
        float v[8];
        lowp::ld8<T>(w + n * ldw + c * 8, v);
#pragma unroll
        for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(v[j]));
    }
    amax = lowp::block_max(amax, red);
    if (threadIdx.x == 0) atomicMax(amax_bits, __float_as_uint(amax));
}

__global__ void nvfp4_tensor_scale_kernel(float *scale)
{
    if (threadIdx.x == 0 && blockIdx.x == 0) *scale = tensor_scale_of(*scale);
}

int sm_count()
{
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

template <typename T>
int run(const void *w, int64_t N, int64_t K, int64_t ldw, uint8_t *codes, uint8_t *sf, float *tscale,
        cudaStream_t st)
{
    if (cudaMemsetAsync(tscale, 0, sizeof(float), st) != cudaSuccess) return -1;
    if (cudaMemsetAsync(sf, 0, nvfp4_scale_bytes(N, K), st) != cudaSuccess) return -1;
    const T *wt = static_cast<const T *>(w);
    const int sms = sm_count();
    const int64_t chunks = N * (K / 8);
    const int64_t agrid = std::max<int64_t>(1, std::min<int64_t>((chunks + kThreads - 1) / kThreads, (int64_t)sms * 8));
    rows_amax_kernel<T><<<(unsigned)agrid, kThreads, 0, st>>>(wt, N, K, ldw, reinterpret_cast<unsigned *>(tscale));
    const int64_t blocks = N * (K / 16);
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>((blocks + kThreads - 1) / kThreads, (int64_t)sms * 8));
    nvfp4_encode_kernel<T><<<(unsigned)grid, kThreads, 0, st>>>(wt, N, K, ldw, tscale, codes, sf);
    nvfp4_tensor_scale_kernel<<<1, 32, 0, st>>>(tscale);
    return 0;
}

}  // namespace

size_t nvfp4_scale_bytes(int64_t N, int64_t K) { return (size_t)((N + 127) / 128) * 128 * (size_t)(K / 16); }

int launch_quantize_nvfp4(const void *w, int wtype, int64_t N, int64_t K, int64_t ldw, uint8_t *codes, uint8_t *sf,
                          float *tscale, cudaStream_t st)
{
    return wtype == WQ_F32 ? run<float>(w, N, K, ldw, codes, sf, tscale, st)
                           : run<uint16_t>(w, N, K, ldw, codes, sf, tscale, st);
}

}  // namespace wq

// wq_quant_fp8.cu -- FP8 quantisation: per output channel (weights) and per
// tensor (activations, the dynamic scaling of a W8A8 matmul).
//
// "Quantization for LLM inference: FP8, INT4 (GPTQ, AWQ) and GGUF", section
// "FP8: the Hopper/Blackwell datacenter format": E4M3 (4 exponent bits, 3
// mantissa bits, range +-448) and E5M2 (5 and 2, range +-57,344); the scale
// maps a channel's (or the tensor's) largest magnitude onto the format's
// largest value.  Arithmetic, binary32 throughout:
//   s    = max|w| / max_fmt   (one IEEE division; 1 when max|w| == 0)
//   code = the FP8 value nearest to w / s (IEEE division), ties to the even
//          code, finite values beyond the range saturated to +-max_fmt.
// The conversion is the hardware's cvt.rn.satfinite, which rounds to nearest
// even and saturates exactly as stated; subnormal FP8 values are kept.
//
// Both forms are HBM streams of two passes over the data (the second mostly
// from L2): the largest magnitude, then the encode.  Per channel, one CTA
// takes one row; per tensor, a grid-wide maximum (atomicMax on the binary32
// bit pattern, which orders non-negative values), then the encode, then a
// one-thread kernel that turns the maximum into the scale in place.
#include "wq_internal.h"
#include "wq_lowp.cuh"

namespace wq {

namespace {

constexpr int kRowThreads = lowp::kThreads;
using lowp::block_max;
using lowp::ld8;

__host__ __device__ constexpr float fp8_max(int fmt) { return fmt == 0 ? 448.0f : 57344.0f; }

// Two FP8 codes of (lo, hi), lo in the low byte: round to nearest even, saturate finite values.
template <int FMT>
__device__ __forceinline__ uint32_t cvt_fp8x2(float lo, float hi)
{
    uint16_t r;
    if (FMT == 0)
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    else
        asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Codes of v[0..7] / s (IEEE quotients), packed little-endian into 8 bytes.
template <int FMT>
__device__ __forceinline__ uint2 encode8(const float v[8], float s)
{
    uint32_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) c[i] = cvt_fp8x2<FMT>(__fdiv_rn(v[2 * i], s), __fdiv_rn(v[2 * i + 1], s));
    return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

// s = max|w| / max_fmt, 1 for an all-zero input.
template <int FMT>
__device__ __forceinline__ float fp8_scale(float amax)
{
    const float s = __fdiv_rn(amax, fp8_max(FMT));
    return s == 0.0f ? 1.0f : s;
}

// One CTA per row: the row's largest magnitude, then its codes.
template <typename T, int FMT>
__global__ void __launch_bounds__(kRowThreads)
quant_fp8_rows_kernel(const T *__restrict__ w, int64_t N, int64_t K, int64_t ldw, uint8_t *__restrict__ q,
                      float *__restrict__ scales)
{
    __shared__ float red[32];
    for (int64_t n = blockIdx.x; n < N; n += gridDim.x) {
        const T *row = w + n * ldw;
        float amax = 0.0f;
        for (int64_t k = (int64_t)threadIdx.x * 8; k < K; k += (int64_t)blockDim.x * 8) {
            float v[8];
            ld8<T>(row + k, v);
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
        }
        amax = block_max(amax, red);
        const float s = fp8_scale<FMT>(amax);
        for (int64_t k = (int64_t)threadIdx.x * 8; k < K; k += (int64_t)blockDim.x * 8) {
            float v[8];
            ld8<T>(row + k, v);
            *reinterpret_cast<uint2 *>(q + n * K + k) = encode8<FMT>(v, s);
        }
        if (threadIdx.x == 0) scales[n] = s;
    }
}

// Codes of the whole tensor against the scale derived from the maximum in *amax.
template <typename T, int FMT>
__global__ void __launch_bounds__(kRowThreads)
tensor_encode_kernel(const T *__restrict__ x, int64_t count, const float *__restrict__ amax, uint8_t *__restrict__ q)
{
    const float s = fp8_scale<FMT>(*amax);
    const int64_t stride = (int64_t)gridDim.x * blockDim.x * 8;
    for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 8; i < count; i += stride) {
        float v[8];
        ld8<T>(x + i, v);
        *reinterpret_cast<uint2 *>(q + i) = encode8<FMT>(v, s);
    }
}

// *scale holds the tensor's largest magnitude; replace it with the scale.
template <int FMT>
__global__ void tensor_scale_kernel(float *scale)
{
    if (threadIdx.x == 0 && blockIdx.x == 0) *scale = fp8_scale<FMT>(*scale);
}

int sm_count()
{
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

template <typename T, int FMT>
void rows(const void *w, int64_t N, int64_t K, int64_t ldw, uint8_t *q, float *s, cudaStream_t st)
{
    const int64_t grid = std::min<int64_t>(N, (int64_t)sm_count() * 8);
    quant_fp8_rows_kernel<T, FMT><<<(unsigned)grid, kRowThreads, 0, st>>>(static_cast<const T *>(w), N, K, ldw, q, s);
}

template <typename T, int FMT>
int tensor(const void *x, int64_t count, uint8_t *q, float *scale, cudaStream_t st)
{
    if (cudaMemsetAsync(scale, 0, sizeof(float), st) != cudaSuccess) return -1;
    const int64_t chunks = count / 8;
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>((chunks + kRowThreads - 1) / kRowThreads,
                                                                (int64_t)sm_count() * 8));
    const T *xt = static_cast<const T *>(x);
    lowp::tensor_amax_kernel<T><<<(unsigned)grid, kRowThreads, 0, st>>>(xt, count, reinterpret_cast<unsigned int *>(scale));
    tensor_encode_kernel<T, FMT><<<(unsigned)grid, kRowThreads, 0, st>>>(xt, count, scale, q);
    tensor_scale_kernel<FMT><<<1, 32, 0, st>>>(scale);
    return 0;
}

}  // namespace

void launch_quantize_fp8_rows(const void *w, int wtype, int64_t N, int64_t K, int64_t ldw, int fmt, uint8_t *q,
                              float *s, cudaStream_t st)
{
    if (wtype == WQ_F32) {
        if (fmt == WQ_FP8_E4M3) rows<float, 0>(w, N, K, ldw, q, s, st);
        else rows<float, 1>(w, N, K, ldw, q, s, st);
    } else {
        if (fmt == WQ_FP8_E4M3) rows<uint16_t, 0>(w, N, K, ldw, q, s, st);
        else rows<uint16_t, 1>(w, N, K, ldw, q, s, st);
    }
}

int launch_quantize_fp8_tensor(const void *x, int xtype, int64_t count, int fmt, uint8_t *q, float *scale,
                               cudaStream_t st)
{
    if (xtype == WQ_F32)
        return fmt == WQ_FP8_E4M3 ? tensor<float, 0>(x, count, q, scale, st) : tensor<float, 1>(x, count, q, scale, st);
    return fmt == WQ_FP8_E4M3 ? tensor<uint16_t, 0>(x, count, q, scale, st)
                              : tensor<uint16_t, 1>(x, count, q, scale, st);
}

}  // namespace wq

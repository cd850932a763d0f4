// wq_colscale.cu -- the activation side of per-input-channel (AWQ-style)
// scaling: the channel statistics and scales of the offline search, and
// x / s for the matmul.
//
// "Quantization Methods Compared: INT8, GPTQ, AWQ, FP8, FP4 and KV-Cache
// Quantization", section "The methods compared": AWQ finds the salient input
// channels from activation magnitudes and scales them up before quantising;
// "Test-time quantization: quantising on the fly with no calibration
// dataset", section "The idea": the activations are divided by the same
// scales, so the product is unchanged up to the quantisation.  The pages give
// no formula for the scale; the reading used (also in the search that drives
// these kernels): s_c = m_c^alpha with m_c the mean |x[m][c]| over the
// calibration rows, normalised so that max(s) * min(s) = 1, a channel with
// m_c = 0 taking the smallest positive magnitude.  The statistics run in
// binary64 (rows summed in order), the scales are rounded to binary32 once.
//
// The matmul's activation side, bf16(x / s) with an IEEE binary32 quotient,
// is applied inside the M = 1 decode kernel while it stages x; for other
// shapes launch_colscale_x writes the scaled activations once (M x K bf16,
// a small fraction of the weight bytes at any M the matmul serves).
#include "wq_common.cuh"
#include "wq_internal.h"

namespace wq {

namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
colscale_x_kernel(const uint16_t *__restrict__ x, int64_t M, int64_t K, const float *__restrict__ s,
                  uint16_t *__restrict__ out)
{
    const int64_t chunks = M * (K / 8);
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < chunks; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t m = i / (K / 8), c = i - m * (K / 8);
        const uint4 v = *reinterpret_cast<const uint4 *>(x + m * K + 8 * c);
        const float4 s0 = __ldg(reinterpret_cast<const float4 *>(s + 8 * c));
        const float4 s1 = __ldg(reinterpret_cast<const float4 *>(s + 8 * c) + 1);
        const float sc[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
            w[j] = pack_bf16x2(__fdiv_rn(__uint_as_float(w[j] << 16), sc[2 * j]),
                               __fdiv_rn(__uint_as_float(w[j] & 0xffff0000u), sc[2 * j + 1]));
        *reinterpret_cast<uint4 *>(out + m * K + 8 * c) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// mag[k] = (sum over rows, in row order, of |x[m][k]|) / M in binary64, rounded to binary32 only for output.
__global__ void __launch_bounds__(kThreads)
channel_absmean_kernel(const uint16_t *__restrict__ x, int64_t M, int64_t K, double *__restrict__ mag64,
                       float *__restrict__ mag)
{
    const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= K) return;
    double acc = 0.0;
    for (int64_t m = 0; m < M; ++m) acc += fabs((double)bf16_to_f32(x[m * K + k]));
    const double v = acc / (double)M;
    mag64[k] = v;
    if (mag) mag[k] = (float)v;
}

// One CTA: s[k] = m'^alpha normalised so that max * min = 1 (binary64, rounded once to binary32).
__global__ void __launch_bounds__(1024)
channel_scales_kernel(const double *__restrict__ mag64, int64_t K, double alpha, float *__restrict__ s)
{
    __shared__ double red[32];
    __shared__ double bcast;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5, nw = blockDim.x >> 5;
    // smallest positive magnitude (1 if none)
    double mn = INFINITY;
    for (int64_t k = tid; k < K; k += blockDim.x)
        if (mag64[k] > 0.0) mn = fmin(mn, mag64[k]);
    for (int o = 16; o > 0; o >>= 1) mn = fmin(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    if (lane == 0) red[wid] = mn;
    __syncthreads();
    if (tid == 0) {
        double v = red[0];
        for (int w = 1; w < nw; ++w) v = fmin(v, red[w]);
        bcast = v == INFINITY ? 1.0 : v;
    }
    __syncthreads();
    const double floor_m = bcast;
    __syncthreads();
    // largest and smallest m'^alpha
    double hi = 0.0, lo = INFINITY;
    for (int64_t k = tid; k < K; k += blockDim.x) {
        const double v = pow(mag64[k] > 0.0 ? mag64[k] : floor_m, alpha);
        hi = fmax(hi, v);
        lo = fmin(lo, v);
    }
    for (int o = 16; o > 0; o >>= 1) {
        hi = fmax(hi, __shfl_xor_sync(0xffffffffu, hi, o));
        lo = fmin(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    }
    __shared__ double red2[32];
    if (lane == 0) {
        red[wid] = hi;
        red2[wid] = lo;
    }
    __syncthreads();
    if (tid == 0) {
        double h = red[0], l = red2[0];
        for (int w = 1; w < nw; ++w) {
            h = fmax(h, red[w]);
            l = fmin(l, red2[w]);
        }
        bcast = sqrt(h * l);
    }
    __syncthreads();
    const double norm = bcast;
    for (int64_t k = tid; k < K; k += blockDim.x)
        s[k] = (float)(pow(mag64[k] > 0.0 ? mag64[k] : floor_m, alpha) / norm);
}

}  // namespace

void launch_colscale_x(const uint16_t *x, int64_t M, int64_t K, const float *col_scale, uint16_t *x_out,
                       cudaStream_t st)
{
    const int64_t chunks = M * (K / 8);
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>((chunks + kThreads - 1) / kThreads, 148 * 8));
    colscale_x_kernel<<<(unsigned)grid, kThreads, 0, st>>>(x, M, K, col_scale, x_out);
}

void launch_channel_magnitudes(const uint16_t *x, int64_t M, int64_t K, double *mag64, float *mag, cudaStream_t st)
{
    channel_absmean_kernel<<<(unsigned)((K + kThreads - 1) / kThreads), kThreads, 0, st>>>(x, M, K, mag64, mag);
}

void launch_channel_scales(const double *mag64, int64_t K, double alpha, float *s, cudaStream_t st)
{
    channel_scales_kernel<<<1, 1024, 0, st>>>(mag64, K, alpha, s);
}

}  // namespace wq

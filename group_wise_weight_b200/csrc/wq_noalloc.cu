// wq_noalloc.cu -- wq_gemm_w4a16_noalloc: the decode-regime W4A16 matmul for
// callers that cannot allocate device memory.
//
// The regular entry point, wq_gemm_w4a16, takes a caller-provided workspace
// for the binary32 partial sums and tile counters of its split-K kernel.
// Some callers have no way to provide one: code that must not call
// cudaMalloc in the middle of a step (it synchronises the whole device),
// inference runtimes and plug-in hosts that own every byte of device memory
// and hand a kernel only its inputs and outputs, and fixed-budget embedded
// or real-time deployments that forbid allocation after start-up.  This
// entry point runs the same kernel with its scratch in a fixed array that is
// part of the library's device image instead.
//
// The array (kScratchBytes, 2 MiB) is a file-scope __device__ variable: every
// GPU that loads the library holds it until the process exits.  Host code
// cannot pass the array's name to a kernel (on the host it is only a
// stand-in symbol), so its device address is looked up with
// cudaGetSymbolAddress once per device, on the first call made with that
// device current; make that first call before any stream capture.
// All calls share the one array: the part a call uses is cleared on the
// call's stream before the kernel runs, and calls whose executions overlap on
// the GPU (different streams, or the same array from several host threads at
// once) race on it.  The cached address belongs to the CUDA context current
// at the first call: the library must not be used across a cudaDeviceReset
// (nor is the device status word's address, cached the same way in
// wq_api.cu, looked up again after one).
#include <cstdio>
#include <mutex>

#include "wq_common.cuh"
#include "wq_internal.h"

namespace {

constexpr size_t kScratchBytes = 2u << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// Device address of g_noalloc_scratch on the current device, looked up once per device.
int scratch_address(void **out)
{
    static std::mutex mu;
    static void *addr[128] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return -1;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return -1;
        addr[dev] = p;
    }
    *out = addr[dev];
    return 0;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int wq_gemm_w4a16_noalloc(const uint16_t *x, int64_t M, int64_t N, int64_t K, const uint8_t *qweight,
                                     const uint16_t *scales, const uint16_t *zeros, int g, uint16_t *y, void *stream)
{
    wq::clear_error();
    if (!x || !qweight || !scales || !zeros || !y)
        return wq::record_error(WQ_ERR_ARG, "wq_gemm_w4a16_noalloc: null pointer");
    if (M <= 0 || N <= 0 || K <= 0)
        return wq::record_error(WQ_ERR_ARG, "wq_gemm_w4a16_noalloc: M, N and K must be positive");
    if (!wq::gemv_tma_eligible(M, N, K, g) || K % 128 != 0)
        return wq::record_error(WQ_ERR_UNSUPPORTED,
                                "wq_gemm_w4a16_noalloc: needs g = 128, 2 <= M <= 16, N >= 128, K >= 256 and "
                                "K % 128 == 0 (other shapes: wq_gemm_w4a16)");
    if (!aligned16(x) || !aligned16(qweight) || !aligned16(scales) || !aligned16(zeros) || !aligned16(y))
        return wq::record_error(WQ_ERR_ALIGN, "wq_gemm_w4a16_noalloc: pointers must be 16-byte aligned");
    if (wq::output_overlaps_inputs(x, M, N, K, qweight, scales, zeros, g, y, false))
        return wq::record_error(WQ_ERR_ARG, "wq_gemm_w4a16_noalloc: y overlaps x, the codes, the scales or the zero-points");
    const size_t need = wq::gemv_tma_compact_bytes(M, N, K, g);
    if (need > kScratchBytes) {
        char msg[256];
        snprintf(msg, sizeof msg,
                 "wq_gemm_w4a16_noalloc: this shape needs %zu bytes of scratch, the fixed array holds %zu "
                 "(M * N * 4 bytes plus counters; use wq_gemm_w4a16 with a workspace)", need, kScratchBytes);
        return wq::record_error(WQ_ERR_WORKSPACE, msg);
    }
    void *scratch = nullptr;
    if (scratch_address(&scratch) != 0)
        return wq::record_error(WQ_ERR_CUDA, "wq_gemm_w4a16_noalloc: cudaGetSymbolAddress failed");
    int *status = wq::device_status_word();
    if (!status) return wq::record_error(WQ_ERR_CUDA, "wq_gemm_w4a16_noalloc: no device status word");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // partial sums and tile counters must start at zero
    if (cudaMemsetAsync(scratch, 0, need, st) != cudaSuccess)
        return wq::record_error(WQ_ERR_CUDA, "wq_gemm_w4a16_noalloc: clearing the scratch array failed");
    if (wq::launch_gemv_w4a16_tma(x, M, N, K, qweight, scales, zeros, y, scratch, status, st, true) != 0)
        return wq::record_error(WQ_ERR_CUDA, "wq_gemm_w4a16_noalloc: tensor map encoding failed");
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof msg, "wq_gemm_w4a16_noalloc: launch failed: %s", cudaGetErrorString(e));
        return wq::record_error(WQ_ERR_CUDA, msg);
    }
    return WQ_OK;
}

// wq_api.cu -- the C ABI of libwq (declared in include/wq.h): argument
// checks, kernel choice and launch.  Kernel choice is a pure function of
// (M, N, K, g); nothing is cached between calls except the per-device status
// word used by bounded waits.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <string>

#include "wq_common.cuh"
#include "wq_internal.h"

namespace {

thread_local std::string g_last_error;

int fail(int status, const char *fmt, ...) __attribute__((format(printf, 2, 3)));

int fail(int status, const char *fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return status;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// a * b * c bytes, saturating (the ranges compared below never wrap)
uint64_t span(int64_t a, int64_t b, int64_t c)
{
    const unsigned __int128 v = (unsigned __int128)(uint64_t)a * (uint64_t)b * (uint64_t)c;
    return v > (unsigned __int128)UINT64_MAX ? UINT64_MAX : (uint64_t)v;
}

// [a, a + an) and [b, b + bn) share a byte
bool overlap(const void *a, uint64_t an, const void *b, uint64_t bn)
{
    if (!a || !b || an == 0 || bn == 0) return false;
    const unsigned __int128 a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + bn && b0 < a0 + an;
}

int check_launch(const char *what)
{
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(WQ_ERR_CUDA, "%s: launch failed: %s", what, cudaGetErrorString(e));
    return WQ_OK;
}

// Shared checks of the quantisers.
int check_quantize(const char *what, const void *w, int wtype, int64_t N, int64_t K, int64_t ldw, int g,
                   const void *q, const void *s, const void *z, bool int8)
{
    if (!w || !q || !s || (!int8 && !z)) return fail(WQ_ERR_ARG, "%s: null pointer", what);
    if (N <= 0 || K <= 0 || ldw <= 0) return fail(WQ_ERR_ARG, "%s: N, K and ldw must be positive", what);
    if (wtype != WQ_F32 && wtype != WQ_BF16) return fail(WQ_ERR_UNSUPPORTED, "%s: wtype %d", what, wtype);
    const bool g_ok = g == 32 || g == 64 || g == 128 || (int8 && (int64_t)g == K);
    if (!g_ok) return fail(WQ_ERR_UNSUPPORTED, "%s: group size %d", what, g);
    if (K % 32 != 0 || K % g != 0 || ldw < K)
        return fail(WQ_ERR_SHAPE, "%s: need K %% 32 == 0, K %% g == 0, ldw >= K (K=%lld g=%d ldw=%lld)", what,
                    (long long)K, g, (long long)ldw);
    if (N > 0x7fffffffLL) return fail(WQ_ERR_SHAPE, "%s: N too large", what);
    if (ldw % 8 != 0 || !aligned16(w) || !aligned16(q) || !aligned16(s) || (z && !aligned16(z)))
        return fail(WQ_ERR_ALIGN, "%s: pointers must be 16-byte aligned and ldw a multiple of 8", what);
    // the outputs must not overlap the weights or one another
    const uint64_t wb = span(N - 1, ldw, wtype == WQ_F32 ? 4 : 2) + span(1, K, wtype == WQ_F32 ? 4 : 2);
    const uint64_t qb = span(N, K, 1) / (int8 ? 1 : 2), pb = span(N, K / g, 2);
    if (overlap(q, qb, w, wb) || overlap(s, pb, w, wb) || overlap(z, pb, w, wb) || overlap(q, qb, s, pb) ||
        overlap(q, qb, z, pb) || overlap(s, pb, z, pb))
        return fail(WQ_ERR_ARG, "%s: output buffers overlap the weights or each other", what);
    return WQ_OK;
}

int check_gemm(const char *what, const void *x, int64_t M, int64_t N, int64_t K, const void *q, const void *s,
               const void *z, int g, const void *y, bool int8)
{
    if (!x || !q || !s || (!int8 && !z) || !y) return fail(WQ_ERR_ARG, "%s: null pointer", what);
    if (M <= 0 || N <= 0 || K <= 0) return fail(WQ_ERR_ARG, "%s: M, N and K must be positive", what);
    const bool g_ok = g == 32 || g == 64 || g == 128 || (int8 && (int64_t)g == K);
    if (!g_ok) return fail(WQ_ERR_UNSUPPORTED, "%s: group size %d", what, g);
    if (K % 32 != 0 || K % g != 0)
        return fail(WQ_ERR_SHAPE, "%s: need K %% 32 == 0 and K %% g == 0 (K=%lld g=%d)", what, (long long)K, g);
    if (N > 0x7fffffffLL * 8 || M > 0x7fffffffLL) return fail(WQ_ERR_SHAPE, "%s: M or N too large", what);
    if (!aligned16(x) || !aligned16(q) || !aligned16(s) || (z && !aligned16(z)) || !aligned16(y))
        return fail(WQ_ERR_ALIGN, "%s: pointers must be 16-byte aligned", what);
    if (wq::output_overlaps_inputs(x, M, N, K, q, s, z, g, y, int8))
        return fail(WQ_ERR_ARG, "%s: y overlaps x, the codes, the scales or the zero-points", what);
    return WQ_OK;
}

}  // namespace

// Per-device status word written by kernels whose waits ran out.
__device__ int g_wq_device_status = 0;

namespace {

// Device address of the status word on the current device (looked up once per device).
int *status_word()
{
    // the device address of the status word, looked up once per device (host threads may race to fill
    // an entry; they store the same address)
    static std::atomic<int *> addr[128] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return nullptr;
    int *a = addr[dev].load(std::memory_order_acquire);
    if (!a) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_wq_device_status) != cudaSuccess) return nullptr;
        a = static_cast<int *>(p);
        addr[dev].store(a, std::memory_order_release);
    }
    return a;
}

}  // namespace

namespace wq {

bool output_overlaps_inputs(const void *x, int64_t M, int64_t N, int64_t K, const void *q, const void *s,
                            const void *z, int g, const void *y, bool int8)
{
    const uint64_t yb = span(M, N, 2), xb = span(M, K, 2);
    const uint64_t qb = span(N, K, 1) / (int8 ? 1 : 2), pb = span(N, K / g, 2);
    return overlap(y, yb, x, xb) || overlap(y, yb, q, qb) || overlap(y, yb, s, pb) || overlap(y, yb, z, pb);
}

// Record `msg` as this thread's last error and return `status` (for entry points in other files).
int record_error(int status, const char *msg)
{
    g_last_error = msg;
    return status;
}

void clear_error() { g_last_error.clear(); }

// Device address of the per-device status word on the current device (nullptr on failure).
int *device_status_word() { return status_word(); }

}  // namespace wq

namespace {

// The W4A16 dispatch after the argument checks.  col_scale, when given, is applied by the M = 1 kernel while
// it stages x; callers pass it only when gemv_m1_eligible holds.
int run_w4a16(const char *what, const uint16_t *x, int64_t M, int64_t N, int64_t K, const uint8_t *qweight,
              const uint16_t *scales, const uint16_t *zeros, int g, uint16_t *y, void *workspace, cudaStream_t st,
              const float *col_scale)
{
    if (wq::gemm_tc_eligible(M, N, K, g)) {
        int *status = status_word();
        if (!status) return fail(WQ_ERR_CUDA, "%s: no device status word", what);
        if (wq::launch_gemm_w4a16_tc(x, M, N, K, qweight, scales, zeros, g, y, workspace, status, st) == -1)
            return fail(WQ_ERR_CUDA, "%s: tensor map encoding failed", what);
        return check_launch(what);
    }
    if (wq::gemv_m1_eligible(M, N, K, g)) {
        int *status = status_word();
        if (!status) return fail(WQ_ERR_CUDA, "%s: no device status word", what);
        const int rc = wq::launch_gemv_w4a16_m1(x, N, K, qweight, scales, zeros, g, y, workspace, status, st, col_scale);
        if (rc == -1) return fail(WQ_ERR_CUDA, "%s: tensor map encoding failed", what);
        return check_launch(what);
    }
    if (wq::gemv_i4mt_eligible(M, N, K, g)) {
        int *status = status_word();
        if (!status) return fail(WQ_ERR_CUDA, "%s: no device status word", what);
        const int rc = wq::launch_gemv_w4a16_i4mt(x, M, N, K, qweight, scales, zeros, y, workspace, status, st);
        if (rc == -1) return fail(WQ_ERR_CUDA, "%s: tensor map encoding failed", what);
        return check_launch(what);
    }
    if (wq::gemv_mt_eligible(M, N, K, g)) {
        int *status = status_word();
        if (!status) return fail(WQ_ERR_CUDA, "%s: no device status word", what);
        const int rc = wq::launch_gemv_w4a16_mt(x, M, N, K, qweight, scales, zeros, y, workspace, status, st);
        if (rc == -1) return fail(WQ_ERR_CUDA, "%s: tensor map encoding failed", what);
        return check_launch(what);
    }
    if (wq::gemv_tma_eligible(M, N, K, g)) {
        int *status = status_word();
        if (!status) return fail(WQ_ERR_CUDA, "%s: no device status word", what);
        if (wq::launch_gemv_w4a16_tma(x, M, N, K, qweight, scales, zeros, y, workspace, status, st) != 0)
            return fail(WQ_ERR_CUDA, "%s: tensor map encoding failed", what);
        return check_launch(what);
    }
    wq::launch_gemv_w4a16(x, M, N, K, qweight, scales, zeros, g, y, st);
    return check_launch(what);
}

// Bytes of the bf16(x / s) staging area of wq_gemm_w4a16_colscaled (none when the M = 1 kernel applies the
// scales itself), rounded up to 256.
size_t colscaled_x_bytes(int64_t M, int64_t N, int64_t K, int g)
{
    return wq::gemv_m1_eligible(M, N, K, g) ? 0 : (span(M, K, 2) + 255) / 256 * 256;
}

}  // namespace

extern "C" {

const char *wq_status_str(int status)
{
    switch (status) {
    case WQ_OK: return "WQ_OK";
    case WQ_ERR_ARG: return "WQ_ERR_ARG: null pointer, non-positive size or overlapping buffers";
    case WQ_ERR_SHAPE: return "WQ_ERR_SHAPE: K, g or ldw do not fit the layout";
    case WQ_ERR_ALIGN: return "WQ_ERR_ALIGN: pointer or leading dimension misaligned";
    case WQ_ERR_UNSUPPORTED: return "WQ_ERR_UNSUPPORTED: group size or dtype not supported";
    case WQ_ERR_CUDA: return "WQ_ERR_CUDA: CUDA error";
    case WQ_ERR_WORKSPACE: return "WQ_ERR_WORKSPACE: workspace missing or too small";
    case WQ_ERR_DEVICE_TIMEOUT: return "WQ_ERR_DEVICE_TIMEOUT: a kernel gave up on a bounded wait";
    default: return "unknown status";
    }
}

const char *wq_last_error(void) { return g_last_error.c_str(); }

int wq_version(void) { return 100; }

int wq_quantize_int4(const void *w, int wtype, int64_t N, int64_t K, int64_t ldw, int g, uint8_t *qweight,
                     uint16_t *scales, uint16_t *zeros, void *stream)
{
    g_last_error.clear();
    int rc = check_quantize("wq_quantize_int4", w, wtype, N, K, ldw, g, qweight, scales, zeros, false);
    if (rc != WQ_OK) return rc;
    wq::launch_quantize_int4(w, wtype, N, K, ldw, g, qweight, scales, zeros, static_cast<cudaStream_t>(stream));
    return check_launch("wq_quantize_int4");
}

int wq_quantize_int4_scaled(const void *w, int wtype, int64_t N, int64_t K, int64_t ldw, int g,
                            const float *col_scale, uint8_t *qweight, uint16_t *scales, uint16_t *zeros,
                            void *stream)
{
    g_last_error.clear();
    int rc = check_quantize("wq_quantize_int4_scaled", w, wtype, N, K, ldw, g, qweight, scales, zeros, false);
    if (rc != WQ_OK) return rc;
    if (!col_scale) return fail(WQ_ERR_ARG, "wq_quantize_int4_scaled: null col_scale");
    if (!aligned16(col_scale)) return fail(WQ_ERR_ALIGN, "wq_quantize_int4_scaled: col_scale must be 16-byte aligned");
    wq::launch_quantize_int4_scaled(w, wtype, N, K, ldw, g, col_scale, qweight, scales, zeros,
                                    static_cast<cudaStream_t>(stream));
    return check_launch("wq_quantize_int4_scaled");
}

int wq_quantize_int4_sym(const void *w, int wtype, int64_t N, int64_t K, int64_t ldw, int g, uint8_t *qweight,
                         uint16_t *scales, uint16_t *zeros, void *stream)
{
    g_last_error.clear();
    int rc = check_quantize("wq_quantize_int4_sym", w, wtype, N, K, ldw, g, qweight, scales, zeros, false);
    if (rc != WQ_OK) return rc;
    wq::launch_quantize_int4_sym(w, wtype, N, K, ldw, g, qweight, scales, zeros, static_cast<cudaStream_t>(stream));
    return check_launch("wq_quantize_int4_sym");
}

int wq_quantize_int8(const void *w, int wtype, int64_t N, int64_t K, int64_t ldw, int g, int8_t *qweight,
                     uint16_t *scales, void *stream)
{
    g_last_error.clear();
    int rc = check_quantize("wq_quantize_int8", w, wtype, N, K, ldw, g, qweight, scales, nullptr, true);
    if (rc != WQ_OK) return rc;
    wq::launch_quantize_int8(w, wtype, N, K, ldw, g, qweight, scales, static_cast<cudaStream_t>(stream));
    return check_launch("wq_quantize_int8");
}

size_t wq_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int g, int wbits)
{
    if (M <= 0 || N <= 0 || K <= 0) return 0;
    if (wbits == 4) {
        if (wq::gemm_tc_eligible(M, N, K, g)) return wq::gemm_tc_workspace_bytes(M, N, K, g);
        if (wq::gemv_m1_eligible(M, N, K, g)) return wq::gemv_m1_workspace_bytes(M, N, K, g);
        if (wq::gemv_i4mt_eligible(M, N, K, g)) return wq::gemv_i4mt_workspace_bytes(M, N, K, g);
        if (wq::gemv_mt_eligible(M, N, K, g)) return wq::gemv_mt_workspace_bytes(M, N, K, g);
        return wq::gemv_tma_workspace_bytes(M, N, K, g);
    }
    if (wbits == 8) {
        if (wq::gemv_w8int_eligible(M, N, K, g)) return wq::gemv_w8int_workspace_bytes(M, N, K, g);
        return wq::gemm_tc_w8_workspace_bytes(M, N, K, g);
    }
    return 0;
}

int wq_gemm_w4a16(const uint16_t *x, int64_t M, int64_t N, int64_t K, const uint8_t *qweight,
                  const uint16_t *scales, const uint16_t *zeros, int g, uint16_t *y, void *workspace,
                  size_t ws_bytes, void *stream)
{
    g_last_error.clear();
    int rc = check_gemm("wq_gemm_w4a16", x, M, N, K, qweight, scales, zeros, g, y, false);
    if (rc != WQ_OK) return rc;
    const size_t need = wq_gemm_workspace_bytes(M, N, K, g, 4);
    if (need > 0 && (!workspace || ws_bytes < need || !aligned16(workspace)))
        return fail(WQ_ERR_WORKSPACE, "wq_gemm_w4a16: need %zu workspace bytes", need);
    return run_w4a16("wq_gemm_w4a16", x, M, N, K, qweight, scales, zeros, g, y, workspace,
                     static_cast<cudaStream_t>(stream), nullptr);
}

int wq_gemm_w8a16(const uint16_t *x, int64_t M, int64_t N, int64_t K, const int8_t *qweight,
                  const uint16_t *scales, int g, uint16_t *y, void *workspace, size_t ws_bytes, void *stream)
{
    g_last_error.clear();
    int rc = check_gemm("wq_gemm_w8a16", x, M, N, K, qweight, scales, nullptr, g, y, true);
    if (rc != WQ_OK) return rc;
    const size_t need = wq_gemm_workspace_bytes(M, N, K, g, 8);
    if (need > 0 && (!workspace || ws_bytes < need || !aligned16(workspace)))
        return fail(WQ_ERR_WORKSPACE, "wq_gemm_w8a16: need %zu workspace bytes", need);
    if (wq::gemv_w8int_eligible(M, N, K, g)) {
        int *status = status_word();
        if (!status) return fail(WQ_ERR_CUDA, "wq_gemm_w8a16: no device status word");
        const int rc = wq::launch_gemv_w8a16_int(x, M, N, K, qweight, scales, y, workspace, status,
                                                 static_cast<cudaStream_t>(stream));
        if (rc == -1) return fail(WQ_ERR_CUDA, "wq_gemm_w8a16: tensor map encoding failed");
        return check_launch("wq_gemm_w8a16");
    }
    if (wq::gemm_tc_w8_eligible(M, N, K, g)) {
        int *status = status_word();
        if (!status) return fail(WQ_ERR_CUDA, "wq_gemm_w8a16: no device status word");
        if (wq::launch_gemm_w8a16_tc(x, M, N, K, qweight, scales, g, y, workspace, status,
                                     static_cast<cudaStream_t>(stream)) != 0)
            return fail(WQ_ERR_CUDA, "wq_gemm_w8a16: tensor map encoding failed");
        return check_launch("wq_gemm_w8a16");
    }
    wq::launch_gemv_w8a16(x, M, N, K, qweight, scales, g, y, static_cast<cudaStream_t>(stream));
    return check_launch("wq_gemm_w8a16");
}

int wq_quantize_fp8(const void *w, int wtype, int64_t N, int64_t K, int64_t ldw, int fmt, uint8_t *qweight,
                    float *scales, void *stream)
{
    g_last_error.clear();
    const char *what = "wq_quantize_fp8";
    if (!w || !qweight || !scales) return fail(WQ_ERR_ARG, "%s: null pointer", what);
    if (N <= 0 || K <= 0 || ldw <= 0) return fail(WQ_ERR_ARG, "%s: N, K and ldw must be positive", what);
    if (wtype != WQ_F32 && wtype != WQ_BF16) return fail(WQ_ERR_UNSUPPORTED, "%s: wtype %d", what, wtype);
    if (fmt != WQ_FP8_E4M3 && fmt != WQ_FP8_E5M2) return fail(WQ_ERR_UNSUPPORTED, "%s: fmt %d", what, fmt);
    if (K % 32 != 0 || ldw < K)
        return fail(WQ_ERR_SHAPE, "%s: need K %% 32 == 0 and ldw >= K (K=%lld ldw=%lld)", what, (long long)K,
                    (long long)ldw);
    if (ldw % 8 != 0 || !aligned16(w) || !aligned16(qweight) || !aligned16(scales))
        return fail(WQ_ERR_ALIGN, "%s: pointers must be 16-byte aligned and ldw a multiple of 8", what);
    const uint64_t wb = span(N - 1, ldw, wtype == WQ_F32 ? 4 : 2) + span(1, K, wtype == WQ_F32 ? 4 : 2);
    const uint64_t qb = span(N, K, 1), sb = span(N, 1, 4);
    if (overlap(qweight, qb, w, wb) || overlap(scales, sb, w, wb) || overlap(qweight, qb, scales, sb))
        return fail(WQ_ERR_ARG, "%s: output buffers overlap the weights or each other", what);
    wq::launch_quantize_fp8_rows(w, wtype, N, K, ldw, fmt, qweight, scales, static_cast<cudaStream_t>(stream));
    return check_launch(what);
}

int wq_quantize_fp8_tensor(const void *x, int xtype, int64_t M, int64_t K, int fmt, uint8_t *q, float *scale,
                           void *stream)
{
    g_last_error.clear();
    const char *what = "wq_quantize_fp8_tensor";
    if (!x || !q || !scale) return fail(WQ_ERR_ARG, "%s: null pointer", what);
    if (M <= 0 || K <= 0) return fail(WQ_ERR_ARG, "%s: M and K must be positive", what);
    if (xtype != WQ_F32 && xtype != WQ_BF16) return fail(WQ_ERR_UNSUPPORTED, "%s: xtype %d", what, xtype);
    if (fmt != WQ_FP8_E4M3 && fmt != WQ_FP8_E5M2) return fail(WQ_ERR_UNSUPPORTED, "%s: fmt %d", what, fmt);
    if (K % 32 != 0) return fail(WQ_ERR_SHAPE, "%s: need K %% 32 == 0 (K=%lld)", what, (long long)K);
    if (!aligned16(x) || !aligned16(q) || (reinterpret_cast<uintptr_t>(scale) & 3u) != 0)
        return fail(WQ_ERR_ALIGN, "%s: x and q must be 16-byte aligned, scale 4-byte aligned", what);
    const uint64_t xb = span(M, K, xtype == WQ_F32 ? 4 : 2), qb = span(M, K, 1);
    if (overlap(q, qb, x, xb) || overlap(scale, 4, x, xb) || overlap(scale, 4, q, qb))
        return fail(WQ_ERR_ARG, "%s: q or scale overlaps x, or each other", what);
    if (wq::launch_quantize_fp8_tensor(x, xtype, M * K, fmt, q, scale, static_cast<cudaStream_t>(stream)) != 0)
        return fail(WQ_ERR_CUDA, "%s: clearing the scale failed: %s", what, cudaGetErrorString(cudaGetLastError()));
    return check_launch(what);
}

size_t wq_gemm_w8a8_fp8_workspace_bytes(int64_t M, int64_t N, int64_t K)
{
    return wq::gemm_fp8_workspace_bytes(M, N, K);
}

int wq_gemm_w8a8_fp8(const uint8_t *xq, const float *xscale, int64_t M, int64_t N, int64_t K, const uint8_t *wq_,
                     const float *wscales, uint16_t *y, void *workspace, size_t ws_bytes, void *stream)
{
    g_last_error.clear();
    const char *what = "wq_gemm_w8a8_fp8";
    if (!xq || !xscale || !wq_ || !wscales || !y) return fail(WQ_ERR_ARG, "%s: null pointer", what);
    if (M <= 0 || N <= 0 || K <= 0) return fail(WQ_ERR_ARG, "%s: M, N and K must be positive", what);
    if (K % 128 != 0) return fail(WQ_ERR_SHAPE, "%s: need K %% 128 == 0 (K=%lld)", what, (long long)K);
    if (M > 0x7fffffffLL || N > 0x7fffffffLL) return fail(WQ_ERR_SHAPE, "%s: M or N too large", what);
    if (!aligned16(xq) || !aligned16(wq_) || !aligned16(wscales) || !aligned16(y) ||
        (reinterpret_cast<uintptr_t>(xscale) & 3u) != 0)
        return fail(WQ_ERR_ALIGN, "%s: pointers must be 16-byte aligned (xscale 4-byte)", what);
    const uint64_t yb = span(M, N, 2);
    if (overlap(y, yb, xq, span(M, K, 1)) || overlap(y, yb, wq_, span(N, K, 1)) || overlap(y, yb, wscales, span(N, 1, 4)) ||
        overlap(y, yb, xscale, 4))
        return fail(WQ_ERR_ARG, "%s: y overlaps an input", what);
    const size_t need = wq::gemm_fp8_workspace_bytes(M, N, K);
    if (need > 0 && (!workspace || ws_bytes < need || !aligned16(workspace)))
        return fail(WQ_ERR_WORKSPACE, "%s: need %zu workspace bytes", what, need);
    int *status = status_word();
    if (!status) return fail(WQ_ERR_CUDA, "%s: no device status word", what);
    if (wq::launch_gemm_w8a8_fp8(xq, xscale, M, N, K, wq_, wscales, y, workspace, status,
                                 static_cast<cudaStream_t>(stream)) != 0)
        return fail(WQ_ERR_CUDA, "%s: tensor map encoding failed", what);
    return check_launch(what);
}

size_t wq_nvfp4_scale_bytes(int64_t N, int64_t K)
{
    if (N <= 0 || K <= 0 || K % 64 != 0) return 0;
    return wq::nvfp4_scale_bytes(N, K);
}

int wq_quantize_nvfp4(const void *w, int wtype, int64_t N, int64_t K, int64_t ldw, uint8_t *codes,
                      uint8_t *block_scales, float *tensor_scale, void *stream)
{
    g_last_error.clear();
    const char *what = "wq_quantize_nvfp4";
    if (!w || !codes || !block_scales || !tensor_scale) return fail(WQ_ERR_ARG, "%s: null pointer", what);
    if (N <= 0 || K <= 0 || ldw <= 0) return fail(WQ_ERR_ARG, "%s: N, K and ldw must be positive", what);
    if (wtype != WQ_F32 && wtype != WQ_BF16) return fail(WQ_ERR_UNSUPPORTED, "%s: wtype %d", what, wtype);
    if (K % 64 != 0 || ldw < K)
        return fail(WQ_ERR_SHAPE, "%s: need K %% 64 == 0 and ldw >= K (K=%lld ldw=%lld)", what, (long long)K,
                    (long long)ldw);
    if (N > 0x7fffffffLL) return fail(WQ_ERR_SHAPE, "%s: N too large", what);
    if (ldw % 8 != 0 || !aligned16(w) || !aligned16(codes) || !aligned16(block_scales) ||
        (reinterpret_cast<uintptr_t>(tensor_scale) & 3u) != 0)
        return fail(WQ_ERR_ALIGN, "%s: pointers must be 16-byte aligned (tensor_scale 4-byte), ldw %% 8 == 0", what);
    const uint64_t wb = span(N - 1, ldw, wtype == WQ_F32 ? 4 : 2) + span(1, K, wtype == WQ_F32 ? 4 : 2);
    const uint64_t cb = span(N, K, 1) / 2, sb = wq::nvfp4_scale_bytes(N, K);
    if (overlap(codes, cb, w, wb) || overlap(block_scales, sb, w, wb) || overlap(tensor_scale, 4, w, wb) ||
        overlap(codes, cb, block_scales, sb) || overlap(codes, cb, tensor_scale, 4) ||
        overlap(block_scales, sb, tensor_scale, 4))
        return fail(WQ_ERR_ARG, "%s: output buffers overlap the input or each other", what);
    if (wq::launch_quantize_nvfp4(w, wtype, N, K, ldw, codes, block_scales, tensor_scale,
                                  static_cast<cudaStream_t>(stream)) != 0)
        return fail(WQ_ERR_CUDA, "%s: clearing the outputs failed: %s", what, cudaGetErrorString(cudaGetLastError()));
    return check_launch(what);
}

size_t wq_gemm_nvfp4_workspace_bytes(int64_t M, int64_t N, int64_t K)
{
    return wq::gemm_nvfp4_workspace_bytes(M, N, K);
}

int wq_gemm_nvfp4(const uint8_t *xc, const uint8_t *xsf, const float *xts, int64_t M, int64_t N, int64_t K,
                  const uint8_t *wc, const uint8_t *wsf, const float *wts, uint16_t *y, void *workspace,
                  size_t ws_bytes, void *stream)
{
    g_last_error.clear();
    const char *what = "wq_gemm_nvfp4";
    if (!xc || !xsf || !xts || !wc || !wsf || !wts || !y) return fail(WQ_ERR_ARG, "%s: null pointer", what);
    if (M <= 0 || N <= 0 || K <= 0) return fail(WQ_ERR_ARG, "%s: M, N and K must be positive", what);
    if (K % 256 != 0) return fail(WQ_ERR_SHAPE, "%s: need K %% 256 == 0 (K=%lld)", what, (long long)K);
    if (M > 0x7fffffffLL || N > 0x7fffffffLL) return fail(WQ_ERR_SHAPE, "%s: M or N too large", what);
    if (!aligned16(xc) || !aligned16(xsf) || !aligned16(wc) || !aligned16(wsf) || !aligned16(y) ||
        (reinterpret_cast<uintptr_t>(xts) & 3u) != 0 || (reinterpret_cast<uintptr_t>(wts) & 3u) != 0)
        return fail(WQ_ERR_ALIGN, "%s: pointers must be 16-byte aligned (tensor scales 4-byte)", what);
    const uint64_t yb = span(M, N, 2);
    if (overlap(y, yb, xc, span(M, K, 1) / 2) || overlap(y, yb, wc, span(N, K, 1) / 2) ||
        overlap(y, yb, xsf, wq::nvfp4_scale_bytes(M, K)) || overlap(y, yb, wsf, wq::nvfp4_scale_bytes(N, K)) ||
        overlap(y, yb, xts, 4) || overlap(y, yb, wts, 4))
        return fail(WQ_ERR_ARG, "%s: y overlaps an input", what);
    const size_t need = wq::gemm_nvfp4_workspace_bytes(M, N, K);
    if (need > 0 && (!workspace || ws_bytes < need || !aligned16(workspace)))
        return fail(WQ_ERR_WORKSPACE, "%s: need %zu workspace bytes", what, need);
    int *status = status_word();
    if (!status) return fail(WQ_ERR_CUDA, "%s: no device status word", what);
    if (wq::launch_gemm_nvfp4(xc, xsf, xts, M, N, K, wc, wsf, wts, y, workspace, status,
                              static_cast<cudaStream_t>(stream)) != 0)
        return fail(WQ_ERR_CUDA, "%s: tensor map encoding failed", what);
    return check_launch(what);
}

size_t wq_decode_attention_workspace_bytes(int64_t B, int64_t T, int64_t H)
{
    if (B <= 0 || T <= 0 || H <= 0) return 0;
    return wq::kv_attn_workspace_bytes(B, T, H);
}

namespace {

int check_attention(const char *what, bool fp8, const void *q, const void *kc, const void *ks, const void *kz,
                    const void *vc, const void *vs, const void *vz, const void *lengths, int64_t B, int64_t T,
                    int64_t H, int64_t Hq, int64_t D, const void *o, const void *ws, size_t ws_bytes)
{
    if (!q || !kc || !ks || !vc || !vs || !lengths || !o || (!fp8 && (!kz || !vz)))
        return fail(WQ_ERR_ARG, "%s: null pointer", what);
    if (B <= 0 || T <= 0 || H <= 0 || Hq <= 0 || D <= 0)
        return fail(WQ_ERR_ARG, "%s: B, T, H, Hq and D must be positive", what);
    if (D != 128 || Hq % H != 0 || Hq / H > 8)
        return fail(WQ_ERR_UNSUPPORTED, "%s: needs D == 128 and Hq a multiple of H with Hq / H <= 8 (D=%lld H=%lld Hq=%lld)",
                    what, (long long)D, (long long)H, (long long)Hq);
    if (B > 65535 || T > 0x7fffffffLL / 2 || H > 65535 || B * T * H > 0x7fffffffffffLL)
        return fail(WQ_ERR_SHAPE, "%s: B, T or H too large", what);
    const bool al = aligned16(q) && aligned16(kc) && aligned16(vc) && aligned16(lengths) && aligned16(o) &&
                    (fp8 ? ((reinterpret_cast<uintptr_t>(ks) & 3u) == 0 && (reinterpret_cast<uintptr_t>(vs) & 3u) == 0)
                         : (aligned16(ks) && aligned16(kz) && aligned16(vs) && aligned16(vz)));
    if (!al) return fail(WQ_ERR_ALIGN, "%s: pointers must be 16-byte aligned (fp8 scales 4-byte)", what);
    const uint64_t ob = span(B, Hq, D * 4), cb = span(B * T, H, fp8 ? D : D / 2), pb = fp8 ? 4 : span(B * T, H, 2);
    if (overlap(o, ob, q, span(B, Hq, D * 2)) || overlap(o, ob, kc, cb) || overlap(o, ob, vc, cb) ||
        overlap(o, ob, ks, pb) || overlap(o, ob, vs, pb) || overlap(o, ob, kz, fp8 ? 0 : pb) ||
        overlap(o, ob, vz, fp8 ? 0 : pb) || overlap(o, ob, lengths, span(B, 4, 1)))
        return fail(WQ_ERR_ARG, "%s: o overlaps an input", what);
    const size_t need = wq::kv_attn_workspace_bytes(B, T, H);
    if (!ws || ws_bytes < need || !aligned16(ws)) return fail(WQ_ERR_WORKSPACE, "%s: need %zu workspace bytes", what, need);
    if (overlap(ws, need, o, ob)) return fail(WQ_ERR_ARG, "%s: the workspace overlaps o", what);
    return WQ_OK;
}

}  // namespace

int wq_decode_attention_int4(const uint16_t *q, const uint8_t *kc, const uint16_t *ks, const uint16_t *kz,
                             const uint8_t *vc, const uint16_t *vs, const uint16_t *vz, const int32_t *lengths,
                             int64_t B, int64_t T, int64_t H, int64_t Hq, int64_t D, float *o, void *workspace,
                             size_t ws_bytes, void *stream)
{
    g_last_error.clear();
    const char *what = "wq_decode_attention_int4";
    const int rc = check_attention(what, false, q, kc, ks, kz, vc, vs, vz, lengths, B, T, H, Hq, D, o, workspace, ws_bytes);
    if (rc != WQ_OK) return rc;
    wq::launch_kv_attn(false, q, kc, ks, kz, nullptr, vc, vs, vz, nullptr, lengths, B, T, H, Hq, o, workspace,
                       static_cast<cudaStream_t>(stream));
    return check_launch(what);
}

int wq_decode_attention_fp8(const uint16_t *q, const uint8_t *kc, const float *ks, const uint8_t *vc, const float *vs,
                            const int32_t *lengths, int64_t B, int64_t T, int64_t H, int64_t Hq, int64_t D, float *o,
                            void *workspace, size_t ws_bytes, void *stream)
{
    g_last_error.clear();
    const char *what = "wq_decode_attention_fp8";
    const int rc = check_attention(what, true, q, kc, ks, nullptr, vc, vs, nullptr, lengths, B, T, H, Hq, D, o,
                                   workspace, ws_bytes);
    if (rc != WQ_OK) return rc;
    wq::launch_kv_attn(true, q, kc, nullptr, nullptr, ks, vc, nullptr, nullptr, vs, lengths, B, T, H, Hq, o,
                       workspace, static_cast<cudaStream_t>(stream));
    return check_launch(what);
}

size_t wq_gemm_w4a16_colscaled_workspace_bytes(int64_t M, int64_t N, int64_t K, int g)
{
    if (M <= 0 || N <= 0 || K <= 0) return 0;
    return colscaled_x_bytes(M, N, K, g) + wq_gemm_workspace_bytes(M, N, K, g, 4);
}

int wq_gemm_w4a16_colscaled(const uint16_t *x, const float *col_scale, int64_t M, int64_t N, int64_t K,
                            const uint8_t *qweight, const uint16_t *scales, const uint16_t *zeros, int g, uint16_t *y,
                            void *workspace, size_t ws_bytes, void *stream)
{
    g_last_error.clear();
    const char *what = "wq_gemm_w4a16_colscaled";
    int rc = check_gemm(what, x, M, N, K, qweight, scales, zeros, g, y, false);
    if (rc != WQ_OK) return rc;
    if (!col_scale) return fail(WQ_ERR_ARG, "%s: null col_scale", what);
    if (!aligned16(col_scale)) return fail(WQ_ERR_ALIGN, "%s: col_scale must be 16-byte aligned", what);
    if (overlap(y, span(M, N, 2), col_scale, span(K, 4, 1)))
        return fail(WQ_ERR_ARG, "%s: y overlaps col_scale", what);
    const size_t xb = colscaled_x_bytes(M, N, K, g), need = xb + wq_gemm_workspace_bytes(M, N, K, g, 4);
    if (need > 0 && (!workspace || ws_bytes < need || !aligned16(workspace)))
        return fail(WQ_ERR_WORKSPACE, "%s: need %zu workspace bytes", what, need);
    if (need > 0 && (overlap(workspace, need, x, span(M, K, 2)) || overlap(workspace, need, y, span(M, N, 2))))
        return fail(WQ_ERR_ARG, "%s: the workspace overlaps x or y", what);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (xb == 0)  // the M = 1 kernel divides x by the scales while it stages x
        return run_w4a16(what, x, M, N, K, qweight, scales, zeros, g, y, workspace, st, col_scale);
    // the matmul's workspace first (its counters at the front, as in every call), the scaled activations after it
    uint16_t *xs = reinterpret_cast<uint16_t *>(static_cast<uint8_t *>(workspace) + (need - xb));
    wq::launch_colscale_x(x, M, K, col_scale, xs, st);
    rc = check_launch(what);
    if (rc != WQ_OK) return rc;
    return run_w4a16(what, xs, M, N, K, qweight, scales, zeros, g, y, workspace, st, nullptr);
}

int wq_awq_channel_magnitudes(const uint16_t *x, int64_t M, int64_t K, double *magnitudes, void *stream)
{
    g_last_error.clear();
    const char *what = "wq_awq_channel_magnitudes";
    if (!x || !magnitudes) return fail(WQ_ERR_ARG, "%s: null pointer", what);
    if (M <= 0 || K <= 0) return fail(WQ_ERR_ARG, "%s: M and K must be positive", what);
    if (!aligned16(x) || !aligned16(magnitudes)) return fail(WQ_ERR_ALIGN, "%s: pointers must be 16-byte aligned", what);
    if (overlap(magnitudes, span(K, 8, 1), x, span(M, K, 2))) return fail(WQ_ERR_ARG, "%s: output overlaps x", what);
    wq::launch_channel_magnitudes(x, M, K, magnitudes, nullptr, static_cast<cudaStream_t>(stream));
    return check_launch(what);
}

int wq_awq_channel_scales(const double *magnitudes, int64_t K, double alpha, float *col_scale, void *stream)
{
    g_last_error.clear();
    const char *what = "wq_awq_channel_scales";
    if (!magnitudes || !col_scale) return fail(WQ_ERR_ARG, "%s: null pointer", what);
    if (K <= 0) return fail(WQ_ERR_ARG, "%s: K must be positive", what);
    if (!(alpha >= 0.0 && alpha <= 1.0)) return fail(WQ_ERR_ARG, "%s: alpha must lie in [0, 1]", what);
    if (!aligned16(magnitudes) || !aligned16(col_scale))
        return fail(WQ_ERR_ALIGN, "%s: pointers must be 16-byte aligned", what);
    if (overlap(col_scale, span(K, 4, 1), magnitudes, span(K, 8, 1)))
        return fail(WQ_ERR_ARG, "%s: output overlaps the magnitudes", what);
    wq::launch_channel_scales(magnitudes, K, alpha, col_scale, static_cast<cudaStream_t>(stream));
    return check_launch(what);
}

int wq_device_status(void *stream)
{
    g_last_error.clear();
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int host = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&host, g_wq_device_status, sizeof(int), 0,
                                              cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return fail(WQ_ERR_CUDA, "wq_device_status: %s", cudaGetErrorString(e));
    if (host != 0) {
        const int zero = 0;
        e = cudaMemcpyToSymbolAsync(g_wq_device_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) return fail(WQ_ERR_CUDA, "wq_device_status: %s", cudaGetErrorString(e));
        return fail(WQ_ERR_DEVICE_TIMEOUT, "a kernel recorded a bounded-wait timeout (code %d)", host);
    }
    return WQ_OK;
}

}  // extern "C"

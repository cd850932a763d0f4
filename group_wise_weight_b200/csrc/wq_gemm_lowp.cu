// wq_gemm_lowp.cu -- weight-and-activation quantised matmuls on the
// 5th-generation tensor cores (sm_100a): FP8 W8A8 (tcgen05.mma
// kind::f8f6f4) and NVFP4 W4A4 (kind::mxf4nvf4 with block scales).
//
// FP8: "Quantization for LLM inference: FP8, INT4 (GPTQ, AWQ) and GGUF",
// section "FP8: the Hopper/Blackwell datacenter format": weights and
// activations both in FP8, multiplied by the tensor cores directly, weights
// with one scale per output channel, activations with one dynamic scale per
// tensor:
//   y[m][n] = bf16( (sum_k e4m3(xq[m][k]) e4m3(wq[n][k])) * sx * sw[n] ).
// NVFP4: "Quantization Methods Compared: INT8, GPTQ, AWQ, FP8, FP4 and
// KV-Cache Quantization", section "Hardware, formats and the roofline": E2M1
// values with an E4M3 scale per 16 values and a binary32 tensor scale, the
// Blackwell tensor cores applying the block scales inside the MMA:
//   y[m][n] = bf16( (sum_b bx[m][b] bw[n][b] sum_{k in b} e2m1(x) e2m1(w)) * tx * tw ).
// Products of the narrow values, and their products with the block scales,
// are exact in binary32; the tensor core accumulates in binary32 and the
// per-tensor / per-channel scales are applied once per output.
//
// Formulation: D[n][m] = sum_k w[n][k] x[m][k], a 128 x BN tile per CTA at a
// time (MMA M = 128 weight rows, N = BN activation rows).  Both operands are
// K-major in shared memory, loaded by TMA with the 128-byte swizzle; a stage
// is 128 bytes of K of every row (128 FP8 values or 256 E2M1 values), four
// MMAs of 32 bytes of K each.  For NVFP4 each stage also brings the 2 KB of
// block scales of the weight tile and of the activation tile (four 512-byte
// atoms each, stored by the quantiser in the layout the copy to tensor
// memory takes), and the MMA lane copies them into tensor memory with
// tcgen05.cp.32x128b.warpx4 right before the MMAs that read them (copies and
// MMAs issued by one thread execute in order).  D lives in tensor memory,
// double buffered, so the epilogue of one tile overlaps the MMAs of the next.
//
// At M = 128 the weights are one byte (FP8) or 0.56 byte (NVFP4) each, below
// the ridge point of these formats: the kernel streams weights and its job is
// to keep HBM busy.  Warp roles (192 threads): warp 0 issues the copies into
// a ring of stages, warp 1 allocates tensor memory and one lane issues the
// MMAs, warps 2..5 read D back (one 32-lane quarter of tensor memory each),
// scale it and write y.  Stream-K over (tile, stage) units gives every SM the
// same number of stages; a tile split between CTAs leaves one binary32
// partial per segment in the workspace, and the CTA of the tile's first
// segment waits (bounded) for the others, sums the segments in segment order
// (so results do not depend on timing) and writes y.  Every barrier wait is
// bounded.
#include <algorithm>
#include <map>
#include <mutex>

#include "wq_internal.h"
#include "wq_sm100.cuh"

namespace wq {

namespace {

// Device-scope add with release semantics (no value returned): the writes that happen before it (this
// thread's, and through the preceding CTA barrier and fences the other threads') are visible before the add.
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

constexpr int kTileN = 128;     // weight rows per tile (MMA M)
constexpr int kRowBytes = 128;  // bytes of K per row and stage (one 128-byte swizzle row)
constexpr int kThreads = 192;   // warp 0: copies, warp 1: MMA, warps 2..5: epilogue
constexpr int kEpiWarp0 = 2;
constexpr int kSfAtom = 512;    // block scales of 128 rows x 64 values of K

enum Kind { kFp8 = 0, kNvfp4 = 1 };

template <int BN, int KIND>
struct Cfg {
    static constexpr int kABytes = kTileN * kRowBytes;  // 16 KB of weights
    static constexpr int kBBytes = BN * kRowBytes;
    static constexpr int kSfBytes = KIND == kNvfp4 ? 4 * kSfAtom : 0;  // per operand and stage
    static constexpr int kStageBytes = kABytes + kBBytes + 2 * kSfBytes;
    static constexpr int kStages = KIND == kNvfp4 ? 5 : (BN <= 128 ? 6 : 4);
    static constexpr size_t kBarOff = (size_t)kStages * kStageBytes;
    // full[S], empty[S], d_full[2], d_empty[2], done
    static constexpr size_t kFlagOff = kBarOff + (2 * kStages + 5) * 8;
    static constexpr size_t kBytes = kFlagOff + 64;
    // two accumulators of BN columns, then (NVFP4) 16 columns of weight block scales and 16 of activation
    static constexpr uint32_t kSfaCol = 2 * BN, kSfbCol = 2 * BN + 16;
    static constexpr uint32_t kTmemCols = KIND == kNvfp4 ? 512 : 2 * BN;
    static_assert(KIND == kFp8 || BN == 128, "NVFP4 tiles are 128 x 128");
    static_assert((kStageBytes & 1023) == 0, "stages stay 1024-byte aligned (128-byte swizzle atoms)");
};

struct Sched {
    int64_t n_tiles, tiles, spt, total, per, extra;
    __host__ __device__ int64_t cta_of(int64_t u) const
    {
        const int64_t big = extra * (per + 1);
        return u < big ? u / (per + 1) : extra + (u - big) / per;
    }
    __host__ __device__ int64_t begin_of(int64_t b) const { return b * per + (b < extra ? b : extra); }
};

struct Ring {
    uint32_t slot = 0, phase = 0;
    __device__ __forceinline__ void next(uint32_t n)
    {
        if (++slot == n) { slot = 0; phase ^= 1u; }
    }
};

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f8f6f4 (formats from the instruction descriptor, f32 accumulate).
__device__ __forceinline__ void mma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
                 "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
                 : "memory");
}

// D[tmem] (+)= (A * SFA) (B * SFB)^T, kind::mxf4nvf4 with one E4M3 scale per 16 values of K.
__device__ __forceinline__ void mma_nvf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
                 ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
                 : "memory");
}

// Copy one 512-byte atom of block scales (32 rows of 16 bytes) into 4 columns of every 32-lane quarter of
// tensor memory.
__device__ __forceinline__ void sf_copy(uint32_t taddr, uint64_t s_desc)
{
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(s_desc) : "memory");
}

// Instruction descriptor, kind::f8f6f4: E4M3 A and B (format code 0), both K-major, f32 D, M x N.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int m, int n)
{
    return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

// Block-scaled instruction descriptor, kind::mxf4nvf4: E2M1 A and B (format code 1), both K-major, E4M3
// scales (bit 23 clear), scale-factor ids 0, K = 64 per instruction (bit 31 clear), M x N.
__host__ __device__ constexpr uint32_t idesc_nvf4(int m, int n)
{
    return (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void wait_drain(uint64_t *bar, uint32_t parity, int *status)
{
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_ns() - t0 > kWaitLimitNs) { record_timeout(status); return; }
}

// Operands of one call.  For FP8: xs = per-tensor activation scale, ws = per-row weight scales (stride 1).
// For NVFP4: xs, ws = the two tensor scales (ws stride 0); sfw, sfx = block scales in the atom layout.
struct Args {
    int64_t M, N, K;
    const float *xs, *ws;
    int ws_stride;
    const uint8_t *sfw, *sfx;
    uint16_t *y;
    float *part;
    int *counters;
    int max_segs;
    int *status;
};

template <int BN, int KIND>
__global__ void __launch_bounds__(kThreads, 1)
gemm_lowp_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap xmap, const Args p)
{
    using C = Cfg<BN, KIND>;
    constexpr uint32_t S = (uint32_t)C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
    uint64_t *empty = full + S;
    uint64_t *d_full = empty + S;
    uint64_t *d_empty = d_full + 2;
    uint64_t *done = d_empty + 2;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kFlagOff);
    volatile int *last_flag = abort_flag + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kFlagOff + 16);
    int *status = p.status;
    const int64_t M = p.M, N = p.N;

    const int tid = threadIdx.x, wid = tid >> 5, lane = tid & 31;
    Sched sc;
    sc.n_tiles = (N + kTileN - 1) / kTileN;
    sc.tiles = sc.n_tiles * ((M + BN - 1) / BN);
    sc.spt = (KIND == kNvfp4 ? p.K / 2 : p.K) / kRowBytes;
    sc.total = sc.tiles * sc.spt;
    sc.per = sc.total / gridDim.x;
    sc.extra = sc.total % gridDim.x;
    const int64_t beg = sc.begin_of(blockIdx.x);
    const int64_t end = beg + sc.per + ((int64_t)blockIdx.x < sc.extra ? 1 : 0);
    const int spt = (int)sc.spt;

    if (tid == 0) {
        for (uint32_t i = 0; i < S; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&d_full[i], 1);
            mbar_init(&d_empty[i], 4);
        }
        mbar_init(done, 1);
        *abort_flag = 0;
        *last_flag = 0;
        fence_mbar_init();
    }
    if (wid == 1) tmem_alloc(tmem_slot, C::kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (wid == 0) {
        // ------------------------------ producer ------------------------------
        if (lane == 0 && beg < end) {
            Ring rg;
            uint32_t issued = 0;
            int64_t tile = beg / spt;
            int ks = (int)(beg - tile * spt);
            const int64_t atoms_per_tile = p.K / 64;  // NVFP4: scale atoms per 128-row tile
            for (int64_t u = beg; u < end; ++u) {
                if (issued >= S && !mbar_wait_fast(&empty[rg.slot], rg.phase ^ 1u, status, abort_flag)) break;
                const int nt = (int)(tile % sc.n_tiles), mt = (int)(tile / sc.n_tiles);
                uint8_t *st = smem + (size_t)rg.slot * C::kStageBytes;
                mbar_arrive_expect_tx(&full[rg.slot], C::kStageBytes);
                tma_load_2d(st, &wmap, &full[rg.slot], ks * kRowBytes, nt * kTileN);
                tma_load_2d(st + C::kABytes, &xmap, &full[rg.slot], ks * kRowBytes, mt * BN);
                if (KIND == kNvfp4) {
                    // a stage covers 256 values of K = 4 scale atoms of the tile's 128 rows
                    bulk_g2s(st + C::kABytes + C::kBBytes, p.sfw + ((int64_t)nt * atoms_per_tile + 4 * ks) * kSfAtom,
                             C::kSfBytes, &full[rg.slot]);
                    bulk_g2s(st + C::kABytes + C::kBBytes + C::kSfBytes,
                             p.sfx + ((int64_t)mt * atoms_per_tile + 4 * ks) * kSfAtom, C::kSfBytes, &full[rg.slot]);
                }
                ++issued;
                rg.next(S);
                if (++ks == spt) { ks = 0; ++tile; }
            }
            // every issued copy must land before the CTA may exit (bounded, ignoring abort)
            for (uint32_t j = issued > S ? issued - S : 0; j < issued; ++j) wait_drain(&full[j % S], (j / S) & 1u, status);
        }
    } else if (wid == 1) {
        // ------------------------------ MMA issuer (one lane) ------------------------------
        if (lane == 0) {
            constexpr uint32_t idesc = KIND == kNvfp4 ? idesc_nvf4(kTileN, BN) : idesc_e4m3_f32(kTileN, BN);
            Ring fr, dr;
            int seg = 0;
            const uint32_t base = smem_u32(smem);
            for (int64_t u = beg; u < end;) {
                const int64_t tile = u / spt;
                const int ks0 = (int)(u - tile * spt);
                const int ks1 = (int)std::min<int64_t>(spt, ks0 + (end - u));
                if (seg >= 2) mbar_wait_fast(&d_empty[dr.slot], dr.phase ^ 1u, status, abort_flag);
                tc_fence_after();
                const uint32_t d_col = tmem + dr.slot * (uint32_t)BN;
                for (int ks = ks0; ks < ks1; ++ks) {
                    mbar_wait_fast(&full[fr.slot], fr.phase, status, abort_flag);
                    tc_fence_after();
                    const uint32_t a = base + fr.slot * (uint32_t)C::kStageBytes;
                    const uint32_t b = a + (uint32_t)C::kABytes;
                    if (KIND == kNvfp4) {
                        const uint32_t sfa = b + (uint32_t)C::kBBytes, sfb = sfa + (uint32_t)C::kSfBytes;
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            // 32 rows x 16 bytes, core matrices of 8 rows 128 bytes apart, no swizzle
                            sf_copy(tmem + C::kSfaCol + 4u * j, smem_desc(sfa + (uint32_t)(j * kSfAtom), 128, 128, 0));
                            sf_copy(tmem + C::kSfbCol + 4u * j, smem_desc(sfb + (uint32_t)(j * kSfAtom), 128, 128, 0));
                        }
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            mma_nvf4(d_col, smem_desc(a + 32u * j, 16, 1024, 2), smem_desc(b + 32u * j, 16, 1024, 2),
                                     idesc, tmem + C::kSfaCol + 4u * j, tmem + C::kSfbCol + 4u * j,
                                     (ks > ks0 || j > 0) ? 1u : 0u);
                    } else {
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            mma_f8(d_col, smem_desc(a + 32u * j, 16, 1024, 2), smem_desc(b + 32u * j, 16, 1024, 2),
                                   idesc, (ks > ks0 || j > 0) ? 1u : 0u);
                    }
                    tc_commit(&empty[fr.slot]);
                    fr.next(S);
                }
                tc_commit(&d_full[dr.slot]);
                dr.next(2);
                ++seg;
                u += ks1 - ks0;
            }
            tc_commit(done);
            wait_drain(done, 0, status);  // every MMA must complete before tensor memory is released
        }
    } else {
        // ------------------------------ epilogue ------------------------------
        const int quarter = wid & 3;
        const int r = quarter * 32 + lane;  // row of the tile = tensor-memory lane
        const uint32_t lane_bits = (uint32_t)(quarter * 32) << 16;
        const float xs = *p.xs;
        Ring dr;
        for (int64_t u = beg; u < end;) {
            const int64_t tile = u / spt;
            const int ks0 = (int)(u - tile * spt);
            const int ks1 = (int)std::min<int64_t>(spt, ks0 + (end - u));
            const int64_t nt = tile % sc.n_tiles, mt = tile / sc.n_tiles;
            const int64_t n = nt * kTileN + r;
            const int64_t m0 = mt * BN;
            mbar_wait_fast(&d_full[dr.slot], dr.phase, status, abort_flag);
            tc_fence_after();
            const float scale = n < N ? xs * p.ws[n * p.ws_stride] : 0.0f;
            const uint32_t d_addr = tmem + lane_bits + dr.slot * (uint32_t)BN;
            if (ks0 == 0 && ks1 == spt) {
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 32) {
                    uint32_t v[32];
                    tmem_ld32(d_addr + (uint32_t)c0, v);
                    tmem_wait_ld();
                    if (n < N) {
#pragma unroll
                        for (int c = 0; c < 32; ++c)
                            if (m0 + c0 + c < M) p.y[(m0 + c0 + c) * N + n] = f32_to_bf16(__uint_as_float(v[c]) * scale);
                    }
                }
            } else {
                const int64_t cta_first = sc.cta_of(tile * spt);
                const int64_t my_seg = (int64_t)blockIdx.x - cta_first;
                const int64_t nseg = sc.cta_of(tile * spt + spt - 1) - cta_first + 1;
                // The CTA of the tile's first segment combines it: that segment ends its range, while the tile's
                // last segment starts the next CTA's, so it is usually among the last to finish.  The others
                // write their slots and add their stage counts with release semantics (no round trip); the
                // first keeps its sums in tensor memory and waits (bounded) until the counter shows every other
                // stage.
                if (my_seg != 0) {
                    float *slot = p.part + ((tile * p.max_segs + my_seg) * BN) * kTileN;
#pragma unroll 1
                    for (int c0 = 0; c0 < BN; c0 += 32) {
                        uint32_t v[32];
                        tmem_ld32(d_addr + (uint32_t)c0, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int c = 0; c < 32; ++c) slot[(int64_t)(c0 + c) * kTileN + r] = __uint_as_float(v[c]);
                    }
                    __threadfence();
                    named_bar_sync(1, 128);
                    if (tid == kEpiWarp0 * 32) red_add_release(p.counters + tile, ks1 - ks0);
                } else {
                if (tid == kEpiWarp0 * 32) {
                    const int others = spt - (ks1 - ks0);
                    int arrived = 1;
                    const uint64_t t0 = global_ns();
                    while (ld_acquire(p.counters + tile) != others) {
                        if (*abort_flag) { arrived = 0; break; }
                        if (global_ns() - t0 > kWaitLimitNs) {
                            record_timeout(status);
                            *abort_flag = 1;
                            arrived = 0;
                            break;
                        }
                    }
                    *last_flag = arrived;
                }
                named_bar_sync(1, 128);
                if (*last_flag) {
                    // sum the segments in segment order (this CTA's own first, from tensor memory)
                    __threadfence();
#pragma unroll 1
                    for (int c0 = 0; c0 < BN; c0 += 32) {
                        uint32_t v[32];
                        tmem_ld32(d_addr + (uint32_t)c0, v);
                        tmem_wait_ld();
                        float tot[32];
#pragma unroll
                        for (int c = 0; c < 32; ++c) tot[c] = 0.0f;
                        for (int64_t o = 0; o < nseg; ++o) {
                            const float *other = p.part + ((tile * p.max_segs + o) * BN) * kTileN;
#pragma unroll
                            for (int c = 0; c < 32; ++c)
                                tot[c] += (o == my_seg) ? __uint_as_float(v[c])
                                                        : __ldcg(other + (int64_t)(c0 + c) * kTileN + r);
                        }
                        if (n < N) {
#pragma unroll
                            for (int c = 0; c < 32; ++c)
                                if (m0 + c0 + c < M) p.y[(m0 + c0 + c) * N + n] = f32_to_bf16(tot[c] * scale);
                        }
                    }
                    named_bar_sync(1, 128);
                    if (tid == kEpiWarp0 * 32) atomicExch(p.counters + tile, 0);
                }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&d_empty[dr.slot]);
            dr.next(2);
            u += ks1 - ks0;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (wid == 1) tmem_dealloc(tmem, C::kTmemCols);
}

int fp8_bn(int64_t M) { return M <= 32 ? 32 : M <= 64 ? 64 : M <= 128 ? 128 : 256; }

int sms_of_device()
{
    static std::mutex mu;
    static std::map<int, int> sms_of;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(mu);
    auto it = sms_of.find(dev);
    if (it == sms_of.end()) {
        int v = 148, optin = 0;
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        cudaFuncSetAttribute(gemm_lowp_kernel<32, kFp8>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
        cudaFuncSetAttribute(gemm_lowp_kernel<64, kFp8>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
        cudaFuncSetAttribute(gemm_lowp_kernel<128, kFp8>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
        cudaFuncSetAttribute(gemm_lowp_kernel<256, kFp8>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
        cudaFuncSetAttribute(gemm_lowp_kernel<128, kNvfp4>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
        it = sms_of.emplace(dev, v).first;
    }
    return it->second;
}

struct Plan {
    int64_t tiles, spt, total, grid, max_segs;
};

// kbytes: bytes of K per row (K for FP8, K / 2 for NVFP4).
Plan plan(int64_t M, int64_t N, int64_t kbytes, int bn, int sms)
{
    Plan p;
    p.tiles = ((N + kTileN - 1) / kTileN) * ((M + bn - 1) / bn);
    p.spt = kbytes / kRowBytes;
    p.total = p.tiles * p.spt;
    p.grid = std::max<int64_t>(1, std::min<int64_t>(p.total, sms));
    const int64_t per = p.total / p.grid;  // >= 1
    p.max_segs = (p.spt + per - 1) / per + 1;
    return p;
}

size_t partials_bytes(const Plan &p, int bn)
{
    return ((size_t)p.tiles * (size_t)p.max_segs * (size_t)bn * kTileN * sizeof(float) + 255) / 256 * 256;
}

size_t workspace_bytes(int64_t M, int64_t N, int64_t kbytes, int bn)
{
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const Plan p = plan(M, N, kbytes, bn, sms);
    return counter_region_bytes(p.tiles) + partials_bytes(p, bn);
}

template <int BN, int KIND>
int run(const uint8_t *x, const uint8_t *w, Args a, void *workspace, cudaStream_t st)
{
    const int64_t kbytes = KIND == kNvfp4 ? a.K / 2 : a.K;
    CUtensorMap wmap, xmap;
    if (!encode_tmap_2d(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, w, (uint64_t)kbytes, (uint64_t)a.N, (uint64_t)kbytes,
                        kRowBytes, kTileN, CU_TENSOR_MAP_SWIZZLE_128B))
        return -1;
    if (!encode_tmap_2d(&xmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, x, (uint64_t)kbytes, (uint64_t)a.M, (uint64_t)kbytes,
                        kRowBytes, BN, CU_TENSOR_MAP_SWIZZLE_128B))
        return -1;
    const int sms = sms_of_device();
    const Plan pl = plan(a.M, a.N, kbytes, BN, sms);
    uint8_t *w8 = static_cast<uint8_t *>(workspace);
    a.counters = reinterpret_cast<int *>(w8);
    a.part = reinterpret_cast<float *>(w8 + counter_region_bytes(pl.tiles));
    if (clear_extra_counters(workspace, pl.tiles, st) != cudaSuccess) return -2;
    a.max_segs = (int)pl.max_segs;
    // at least 120 KB so that one CTA owns each SM (and its tensor memory)
    const size_t smem = std::max<size_t>(Cfg<BN, KIND>::kBytes + 1024, 120 * 1024);
    gemm_lowp_kernel<BN, KIND><<<(unsigned)pl.grid, kThreads, smem, st>>>(wmap, xmap, a);
    return 0;
}

}  // namespace

size_t gemm_fp8_workspace_bytes(int64_t M, int64_t N, int64_t K)
{
    if (M <= 0 || N <= 0 || K <= 0 || K % kRowBytes != 0) return 0;
    return workspace_bytes(M, N, K, fp8_bn(M));
}

int launch_gemm_w8a8_fp8(const uint8_t *xq, const float *xscale, int64_t M, int64_t N, int64_t K, const uint8_t *wq,
                         const float *wscale, uint16_t *y, void *workspace, int *status, cudaStream_t st)
{
    Args a{};
    a.M = M; a.N = N; a.K = K;
    a.xs = xscale; a.ws = wscale; a.ws_stride = 1;
    a.y = y; a.status = status;
    switch (fp8_bn(M)) {
    case 32: return run<32, kFp8>(xq, wq, a, workspace, st);
    case 64: return run<64, kFp8>(xq, wq, a, workspace, st);
    case 128: return run<128, kFp8>(xq, wq, a, workspace, st);
    default: return run<256, kFp8>(xq, wq, a, workspace, st);
    }
}

size_t gemm_nvfp4_workspace_bytes(int64_t M, int64_t N, int64_t K)
{
    if (M <= 0 || N <= 0 || K <= 0 || K % (2 * kRowBytes) != 0) return 0;
    return workspace_bytes(M, N, K / 2, 128);
}

int launch_gemm_nvfp4(const uint8_t *xc, const uint8_t *xsf, const float *xts, int64_t M, int64_t N, int64_t K,
                      const uint8_t *wc, const uint8_t *wsf, const float *wts, uint16_t *y, void *workspace,
                      int *status, cudaStream_t st)
{
    Args a{};
    a.M = M; a.N = N; a.K = K;
    a.xs = xts; a.ws = wts; a.ws_stride = 0;
    a.sfw = wsf; a.sfx = xsf;
    a.y = y; a.status = status;
    return run<128, kNvfp4>(xc, wc, a, workspace, st);
}

}  // namespace wq

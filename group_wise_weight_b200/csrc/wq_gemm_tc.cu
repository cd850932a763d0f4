// wq_gemm_tc.cu -- W4A16 matmul for batches of activations (M > 16) on the
// 5th-generation tensor cores (tcgen05, sm_100a).
//
// At batch sizes like 128 the matmul is a dense contraction and the pages'
// roofline argument ("Quantization Methods Compared: INT8, GPTQ, AWQ, FP8,
// FP4 and KV-Cache Quantization", section "Hardware, formats and the
// roofline") puts it near or past the ridge point, so the tensor cores do
// the work.  The 4-bit weights are dequantised inside the kernel, as that
// section describes for practical 4-bit kernels, with the decode
// w_hat = s (q - z) of "Quantization for LLM inference: FP8, INT4 (GPTQ, AWQ)
// and GGUF", section "The minimum maths".
//
// Formulation: D[n][m] = sum_k w_hat[n][k] * x[m][k], a 128 x BN tile per
// CTA at a time (MMA M = 128 weight rows, N = BN activation rows, K = 16 per
// instruction).  The weight operand A lives in tensor memory: dequant warps
// write bf16 w_hat there with tcgen05.st, so the dequantised tile never
// touches shared memory.  The activation operand B is loaded by TMA into
// shared memory with the 128-byte swizzle.  The accumulator D lives in
// tensor memory and is read back by the same warps for the epilogue.
//
// Warp roles (352 threads): warp 0 issues TMA loads of weight boxes
// [128 rows x 64 B] (64-byte swizzle) into a weight ring; warp 2 issues the
// activation boxes [BN rows x 64 elements] (128-byte swizzle) into an
// activation ring; warp 1 allocates tensor memory and one of its lanes issues
// the MMAs; warps 3..10 dequantise (two warps per 32-lane quarter of tensor
// memory, each taking half of the stage's 128 k), promote half of the
// accumulator columns and write the output.
//
// Dequantisation: natural k order.  A code word v (8 codes, k .. k+7) and
// v >> 4 give, with one byte permute and one LOP3 per pair, the bf16x2 pair
// (128 + q[2j], 128 + q[2j+1]); subtracting (128 + z) is exact, so the MMA
// operand is the exact integer q - z.  Each group of g consecutive k gets its
// own accumulator region in tensor memory, and the dequant warps, one stage
// behind the MMAs, add s * D_group into binary32 registers ("promotion"):
// (q - z) is never rounded and s is applied in binary32, as in the decode
// kernels.  A zero-point outside [0, 15] is split (zp_split in wq_common.cuh):
// the operand becomes q - z_lo, the dequant warp marks the stage, the MMA
// warp sums that stage's activations per group into shared memory, and the
// promotion adds -s z_hi times those sums.  Tensor memory: A 2 x 64 columns, D 2 stages x (128/g) groups x BN
// columns (BN = 128 for g = 128, 64 for g = 64, 32 for g = 32).
//
// Scheduling: stream-K over (tile, stage) units so every SM gets the same
// number of stages.  A tile split between CTAs leaves one binary32 partial
// per segment in the workspace; the CTA whose stages complete the tile sums
// the partials of the others and writes y.  Every barrier wait is bounded.
#include <algorithm>
#include <atomic>
#include <map>
#include <mutex>
#include <utility>

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

constexpr int kTileN = 128;         // weight rows per tile (MMA M)
constexpr int kStageK = 128;        // k per stage
constexpr int kWStages = 8;          // weight boxes in flight (released by the dequant warps)
constexpr int kDequantWarps = 8;
constexpr int kWPQ = kDequantWarps / 4;     // dequant warps per 32-lane quarter of tensor memory
constexpr int kKPerWarp = 128 / kWPQ;       // k of a stage each dequant warp handles
constexpr int kChunksPerWarp = kKPerWarp / 32;  // 16-byte code chunks per thread and stage
constexpr int kFirstDequantWarp = 3;  // warps 0, 1, 2: weight producer, MMA issuer, activation producer
constexpr int kThreads = (kFirstDequantWarp + kDequantWarps) * 32;
constexpr uint32_t kTmemCols = 512;  // A: kABufs x 64 columns, D: 2 x 128/g x BN = 256 columns
constexpr uint32_t kABufs = 4;       // dequantised weight tiles in tensor memory

// W8: int8 weights (W8A16), one byte per code, 128-byte rows per stage with the 128-byte swizzle;
// otherwise packed INT4, 64-byte rows with the 64-byte swizzle.
template <int BN, bool W8 = false>
struct Cfg {
    static constexpr int kWRowBytes = W8 ? 128 : 64;             // bytes of a weight row per stage
    static constexpr int kWStageBytes = kTileN * kWRowBytes;     // 16 KB or 8 KB
    static constexpr int kWSt = W8 ? 6 : kWStages;               // weight stages in flight
    static constexpr int kXAtomBytes = BN * 128;             // BN rows x 64 bf16
    static constexpr int kXStageBytes = 2 * kXAtomBytes;     // 128 k of activations
    static constexpr int kXStages = BN == 128 ? 3 : (BN == 64 ? 4 : 6);
    static constexpr size_t kWOff = (size_t)kXStages * kXStageBytes;
    static constexpr size_t kBarOff = kWOff + (size_t)kWSt * kWStageBytes;
    // x_full[XS], x_empty[XS], w_full[WS], w_empty[WS], a_full[A], a_empty[A], d_full[2], d_empty[2], done
    static constexpr size_t kFlagOff = kBarOff + (2 * kXStages + 2 * kWSt + 2 * kABufs + 4 + 1) * 8;
    // flags: abort, last-arrival, tensor-memory address, far-zero-point marks; then activation sums
    static constexpr size_t kXsumOff = kFlagOff + 64;
    static constexpr size_t kBytes = kXsumOff + 2 * 128 * 4;  // [2 D buffers][groups][BN], groups x BN <= 128
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

__device__ __forceinline__ uint32_t word_of4(const uint4 &v, int i)
{
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// (128 + q) - (128 + z) in bf16: exact for the integers involved (z in [0, 15], or z_lo of a split).
__device__ __forceinline__ uint32_t bf2_sub(uint32_t q128, uint32_t zc)
{
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162 *>(&q128);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&zc);
    a = __hsub2(a, b);
    return *reinterpret_cast<uint32_t *>(&a);
}

// t & mask | magic with both constants in registers (kernel arguments): one LOP3 instead of two.
__device__ __forceinline__ uint32_t lop_and_or(uint32_t t, uint32_t mask, uint32_t magic)
{
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(t), "r"(mask), "r"(magic));
    return d;
}

// Slot and phase of a ring of `n` buffers, advanced one use at a time.
struct Ring {
    uint32_t slot = 0, phase = 0;
    __device__ __forceinline__ void next(uint32_t n)
    {
        if (++slot == n) { slot = 0; phase ^= 1u; }
    }
};

// Eight int8 codes (two words) as four exact bf16 pairs (k, k + 1): each byte, flipped to q + 128, is placed
// under the exponent of 2^23 by one byte permute (2^23 + q + 128, exact in binary32), one subtraction gives q,
// and the pair is packed to bf16 (exact: |q| <= 128 has at most 8 significant bits).
__device__ __forceinline__ void int8x8_bf16(uint32_t w0, uint32_t w1, uint32_t out[4])
{
    const uint32_t u[2] = {w0 ^ 0x80808080u, w1 ^ 0x80808080u};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float f[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            f[j] = __fsub_rn(__uint_as_float(__byte_perm(u[h], 0x4B000000u, 0x7540u | (uint32_t)j)), 8388736.0f);
        out[2 * h] = pack_bf16x2(f[0], f[1]);
        out[2 * h + 1] = pack_bf16x2(f[2], f[3]);
    }
}

template <int BN, int GROUP, bool W8>
__global__ void __launch_bounds__(kThreads, 1)
gemm_w4a16_tc_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap xmap, int64_t M,
                     int64_t N, int64_t K, const uint16_t *__restrict__ sc, const uint16_t *__restrict__ zp,
                     uint16_t *__restrict__ y, float *__restrict__ ws, int *__restrict__ counters, int max_segs,
                     int *__restrict__ status, uint32_t nib_mask, uint32_t bf16_magic, int64_t skip_unit,
                     int s_per_row)
{
    using C = Cfg<BN, W8>;
    constexpr int kWStagesK = C::kWSt;
    constexpr int kWeightStageBytes = C::kWStageBytes;
    constexpr int NG = kStageK / GROUP;     // groups per stage
    constexpr int kDCols = NG * BN;         // accumulator columns per stage
    constexpr uint32_t XS = (uint32_t)C::kXStages;
    static_assert((int)kABufs * 64 + 2 * kDCols <= (int)kTmemCols, "tensor memory budget");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    uint64_t *x_full = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
    uint64_t *x_empty = x_full + XS;
    uint64_t *w_full = x_empty + XS;
    uint64_t *w_empty = w_full + kWStagesK;
    uint64_t *a_full = w_empty + kWStagesK;
    uint64_t *a_empty = a_full + kABufs;
    uint64_t *d_full = a_empty + kABufs;
    uint64_t *d_empty = d_full + 2;
    uint64_t *done = d_empty + 2;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kFlagOff);
    volatile int *last_flag = abort_flag + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kFlagOff + 16);
    // wide_mark[A buffer] = stage counter + 1 when a dequant warp split a zero-point of that stage;
    // xs_wide[D buffer] = 1 when the MMA warp wrote the stage's activation sums to xsum
    volatile int *wide_mark = reinterpret_cast<volatile int *>(smem + C::kFlagOff + 32);
    volatile int *xs_wide = wide_mark + kABufs;
    float *xsum = reinterpret_cast<float *>(smem + C::kXsumOff);
    static_assert(NG * BN <= 128, "activation-sum buffer");

    const int tid = threadIdx.x, wid = tid >> 5, lane = tid & 31;
    Sched S;
    S.n_tiles = (N + kTileN - 1) / kTileN;
    S.tiles = S.n_tiles * ((M + BN - 1) / BN);
    S.spt = K / kStageK;
    S.total = S.tiles * S.spt;
    S.per = S.total / gridDim.x;
    S.extra = S.total % gridDim.x;
    const int64_t beg = S.begin_of(blockIdx.x);
    const int64_t end = beg + S.per + ((int64_t)blockIdx.x < S.extra ? 1 : 0);
    const int spt = (int)S.spt;

    if (tid == 0) {
        for (uint32_t i = 0; i < XS; ++i) {
            mbar_init(&x_full[i], 1);
            mbar_init(&x_empty[i], 1);
        }
        for (int i = 0; i < kWStagesK; ++i) {
            mbar_init(&w_full[i], 1);
            mbar_init(&w_empty[i], kDequantWarps);
        }
        for (uint32_t i = 0; i < kABufs; ++i) {
            mbar_init(&a_full[i], kDequantWarps);
            mbar_init(&a_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&d_full[i], 2);  // the MMAs' completion, and the MMA warp's activation sums
            mbar_init(&d_empty[i], kDequantWarps);
        }
        for (uint32_t i = 0; i < kABufs; ++i) wide_mark[i] = 0;
        mbar_init(done, 1);
        *abort_flag = 0;
        *last_flag = 0;
        fence_mbar_init();
    }
    if (wid == 1) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t d_tmem = tmem + kABufs * 64u;  // accumulators: stage buffer b, group gi at (b * NG + gi) * BN

    if (wid == 0 || wid == 2) {
        // ------------------------------ TMA producers ------------------------------
        // warp 0: weight boxes into the weight ring; warp 2: activation boxes into the activation ring
        const bool weights = wid == 0;
        const uint32_t nst = weights ? (uint32_t)kWStagesK : XS;
        uint64_t *fullb = weights ? w_full : x_full;
        uint64_t *emptyb = weights ? w_empty : x_empty;
        if (lane == 0 && beg < end) {
            Ring rg;
            uint32_t issued = 0;
            int64_t tile = beg / spt;
            int ks = (int)(beg - tile * spt);
            for (int64_t u = beg; u < end; ++u) {
                if (issued >= nst && !mbar_wait_fast(&emptyb[rg.slot], rg.phase ^ 1u, status, abort_flag)) break;
                const int nt = (int)(tile % S.n_tiles), mt = (int)(tile / S.n_tiles);
                if (weights) {
                    // skip_unit (tests of the failure path only, -1 otherwise): this stage's weights are never
                    // requested, so the waits on them run out; no copy is left in flight
                    if (u != skip_unit) {
                        mbar_arrive_expect_tx(&fullb[rg.slot], kWeightStageBytes);
                        tma_load_2d(smem + C::kWOff + rg.slot * kWeightStageBytes, &wmap, &fullb[rg.slot],
                                    ks * C::kWRowBytes, nt * kTileN);
                    }
                } else {
                    uint8_t *st = smem + rg.slot * C::kXStageBytes;
                    mbar_arrive_expect_tx(&fullb[rg.slot], C::kXStageBytes);
                    tma_load_2d(st, &xmap, &fullb[rg.slot], ks * kStageK, mt * BN);
                    tma_load_2d(st + C::kXAtomBytes, &xmap, &fullb[rg.slot], ks * kStageK + 64, mt * BN);
                }
                ++issued;
                rg.next(nst);
                if (++ks == spt) { ks = 0; ++tile; }
            }
            // drain: every issued copy must land before the CTA may exit (bounded, ignoring abort); a skipped
            // stage was never requested and is not waited for
            for (uint32_t j = issued > nst ? issued - nst : 0; j < issued; ++j) {
                if (weights && beg + (int64_t)j == skip_unit) continue;
                const uint64_t t0 = global_ns();
                while (!mbar_try_wait(&fullb[j % nst], (j / nst) & 1u))
                    if (global_ns() - t0 > kWaitLimitNs) { record_timeout(status); break; }
            }
        }
    } else if (wid == 1) {
        // ------------------------------ MMA issuer ------------------------------
        // Lane 0 issues the MMAs.  For a stage whose weights have a zero-point outside [0, 15] (marked by
        // the dequant warps) the whole warp also sums the stage's activations per group, before the
        // activation slot is released, for the dequant warps' correction -z_hi * sum x.
        constexpr uint32_t idesc = idesc_bf16_f32(128, BN);
        constexpr int kStepsPerGroup = GROUP / 16;
        Ring xr, ar, dr;  // activation ring, A buffers, D double buffers
        uint32_t it = 0;
        const uint32_t xbase = smem_u32(smem);
        for (int64_t u = beg; u < end;) {
            const int64_t tile = u / spt;
            const int ks0 = (int)(u - tile * spt);
            const int ks1 = (int)std::min<int64_t>(spt, ks0 + (end - u));
            for (int ks = ks0; ks < ks1; ++ks, ++it) {
                mbar_wait_fast(&x_full[xr.slot], xr.phase, status, abort_flag);
                mbar_wait_fast(&a_full[ar.slot], ar.phase, status, abort_flag);
                if (it >= 2) mbar_wait_fast(&d_empty[dr.slot], dr.phase ^ 1u, status, abort_flag);
                tc_fence_after();
                const uint32_t xs = xbase + xr.slot * (uint32_t)C::kXStageBytes;
                if (lane == 0) {
                    const uint32_t a_col = tmem + ar.slot * 64u;
                    const uint32_t d_col = d_tmem + dr.slot * (uint32_t)kDCols;
#pragma unroll
                    for (int j = 0; j < kStageK / 16; ++j) {
                        const uint32_t baddr = xs + (uint32_t)(j >> 2) * C::kXAtomBytes + (uint32_t)(j & 3) * 32u;
                        tc_mma_ts(d_col + (uint32_t)((j / kStepsPerGroup) * BN), a_col + (uint32_t)j * 8u,
                                  smem_desc(baddr, 16, 1024, 2), idesc, (j % kStepsPerGroup) != 0 ? 1u : 0u);
                    }
                }
                const bool wide = wide_mark[ar.slot] == (int)(it + 1);
                if (wide) {
                    // rows m = lane, lane + 32, ...: two 128-byte-swizzled atoms of 64 k each
                    for (int m = lane; m < BN; m += 32) {
                        float xg[NG];
#pragma unroll
                        for (int gi = 0; gi < NG; ++gi) xg[gi] = 0.0f;
#pragma unroll
                        for (int a = 0; a < 2; ++a)
#pragma unroll
                            for (int c = 0; c < 8; ++c) {
                                uint4 v;
                                const uint32_t addr = xs + (uint32_t)a * C::kXAtomBytes + (uint32_t)m * 128u +
                                                      (((uint32_t)c ^ ((uint32_t)m & 7u)) << 4);
                                asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                             : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
                                xg[(a * 64 + c * 8) / GROUP] += sum_bf16x8(v);
                            }
#pragma unroll
                        for (int gi = 0; gi < NG; ++gi) xsum[(dr.slot * NG + gi) * BN + m] = xg[gi];
                    }
                }
                if (lane == 0) xs_wide[dr.slot] = wide ? 1 : 0;
                __syncwarp();
                if (lane == 0) {
                    tc_commit(&x_empty[xr.slot]);
                    tc_commit(&a_empty[ar.slot]);
                    tc_commit(&d_full[dr.slot]);
                    mbar_arrive(&d_full[dr.slot]);
                }
                xr.next(XS);
                ar.next(kABufs);
                dr.next(2);
            }
            u += ks1 - ks0;
        }
        if (lane == 0) {
            tc_commit(done);
            // every MMA must have completed before tensor memory is released
            const uint64_t t0 = global_ns();
            while (!mbar_try_wait(done, 0))
                if (global_ns() - t0 > kWaitLimitNs) { record_timeout(status); break; }
        }
    } else {
        // ------------------------------ dequant + promotion + epilogue ------------------------------
        const int dw = wid - kFirstDequantWarp;  // 0 .. kDequantWarps-1
        const int quarter = wid & 3;             // tensor-memory lanes 32*quarter .. +31
        const int kq = dw >> 2;                  // k part of each stage, column part of the accumulators
        const int r = quarter * 32 + lane;       // row of the tile
        const uint32_t lane_bits = (uint32_t)(quarter * 32) << 16;
        constexpr int kCols = BN / kWPQ;         // accumulator columns this warp promotes
        const int G = (int)(K / GROUP);
        // this thread's 16-byte code chunks in a weight slot: row r; INT4: chunks kq*2 + i of a 64-byte row
        // (64-byte swizzle); int8: chunks kq*4 + i of a 128-byte row (128-byte swizzle)
        constexpr int kCh = W8 ? 4 : kChunksPerWarp;
        uint32_t w_addr[kCh];
#pragma unroll
        for (int i = 0; i < kCh; ++i)
            w_addr[i] = W8 ? smem_u32(smem + C::kWOff) + (uint32_t)r * 128u + 16u * ((uint32_t)(kq * 4 + i) ^ (uint32_t)(r & 7))
                           : smem_u32(smem + C::kWOff) + (uint32_t)r * 64u +
                                 16u * ((uint32_t)(kq * kChunksPerWarp + i) ^ (uint32_t)((r >> 1) & 3));
        const uint32_t a_addr = tmem + lane_bits + (uint32_t)(kq * kKPerWarp / 2);
        const uint32_t dq_addr = d_tmem + lane_bits + (uint32_t)(kq * kCols);
        Ring wr, ar, pr;  // weight ring, A buffers, D buffers being promoted
        uint32_t it = 0;
        float acc[kCols];
        float sprev[NG];
        const uint16_t *zrow = zp;  // zero-points of this thread's row in the current tile

        // add s * D of the oldest unpromoted stage (stage ksp of the tile) to acc, then hand its buffer
        // back to the MMA warp.  If the stage had a zero-point outside [0, 15], the dequant warps wrote
        // q - z_lo (zp_split) and the MMA warp the activation sums: acc also takes -s * z_hi * sum x.
        auto promote = [&](int ksp) {
            mbar_wait_fast(&d_full[pr.slot], pr.phase, status, abort_flag);
            tc_fence_after();
            const bool wide = xs_wide[pr.slot] != 0;
#pragma unroll
            for (int gi = 0; gi < NG; ++gi) {
                const f32x2 s2{sprev[gi], sprev[gi]};
                // two tensor-memory loads in flight per wait
                constexpr int kChunk = kCols < 16 ? kCols : 16;
                constexpr int kBatch = kCols >= 2 * kChunk ? 2 : 1;
#pragma unroll
                for (int c0 = 0; c0 < kCols; c0 += kChunk * kBatch) {
                    uint32_t v[kBatch][kChunk];
#pragma unroll
                    for (int b = 0; b < kBatch; ++b) {
                        const uint32_t col =
                            dq_addr + pr.slot * (uint32_t)kDCols + (uint32_t)(gi * BN + c0 + b * kChunk);
                        if (kChunk == 16) tmem_ld16(col, v[b]);
                        else tmem_ld8(col, v[b]);
                    }
                    tmem_wait_ld();
#pragma unroll
                    for (int b = 0; b < kBatch; ++b)
#pragma unroll
                        for (int i = 0; i < kChunk; i += 2) {
                            const int cc = c0 + b * kChunk + i;
                            const f32x2 r2 = fma2_pairs(s2, f32x2{__uint_as_float(v[b][i]), __uint_as_float(v[b][i + 1])},
                                                        f32x2{acc[cc], acc[cc + 1]});
                            acc[cc] = r2.x;
                            acc[cc + 1] = r2.y;
                        }
                }
                if (wide) {
                    float zh;
                    zp_split(bf16_to_f32(zrow[ksp * NG + gi]), zh);
                    if (zh != 0.0f) {
                        const float t = -sprev[gi] * zh;
                        const float *xg = xsum + (pr.slot * NG + gi) * BN + kq * kCols;
#pragma unroll
                        for (int cc = 0; cc < kCols; ++cc) acc[cc] = fmaf(t, xg[cc], acc[cc]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&d_empty[pr.slot]);
            pr.next(2);
        };

        for (int64_t u = beg; u < end;) {
            const int64_t tile = u / spt;
            const int ks0 = (int)(u - tile * spt);
            const int ks1 = (int)std::min<int64_t>(spt, ks0 + (end - u));
            const int64_t nt = tile % S.n_tiles, mt = tile / S.n_tiles;
            const int64_t n = nt * kTileN + r;
            const int64_t nrow = n < N ? n : N - 1;
            // scales of the stage's groups (one scale per row when s_per_row: int8 per channel)
            const uint16_t *sp = s_per_row ? sc + nrow : sc + nrow * G + (int64_t)ks0 * NG;
            const int sp_step = s_per_row ? 0 : NG;
            const uint16_t *zbase = W8 ? nullptr : zp + nrow * G;    // zero-points of the row
            zrow = zbase;
            // a warp's k range of a stage lies in one group when the group is at least that long
            constexpr bool kOneZ = GROUP >= kKPerWarp;
            constexpr int kZ = kOneZ ? 1 : kChunksPerWarp;
            auto zidx = [&](int ks, int i) { return (ks * kStageK + (kq * kChunksPerWarp + i) * 32) / GROUP; };
            // scales and zero-points are loaded one stage ahead of their use
            uint16_t snext[NG], znext[kZ];
#pragma unroll
            for (int gi = 0; gi < NG; ++gi) snext[gi] = sp[s_per_row ? 0 : gi];
#pragma unroll
            for (int i = 0; i < kZ; ++i) znext[i] = W8 ? (uint16_t)0 : zbase[zidx(ks0, i)];
#pragma unroll
            for (int c = 0; c < kCols; ++c) acc[c] = 0.0f;

            for (int ks = ks0; ks < ks1; ++ks, ++it) {
                mbar_wait_fast(&w_full[wr.slot], wr.phase, status, abort_flag);
                if (it >= kABufs) {
                    mbar_wait_fast(&a_empty[ar.slot], ar.phase ^ 1u, status, abort_flag);
                    tc_fence_after();  // the tcgen05.st below must not move ahead of this wait
                }
                uint4 wv[kCh];
#pragma unroll
                for (int i = 0; i < kCh; ++i)
                    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(wv[i].x), "=r"(wv[i].y), "=r"(wv[i].z), "=r"(wv[i].w)
                                 : "r"(w_addr[i] + wr.slot * (uint32_t)kWeightStageBytes));
                float scur[NG];
                uint32_t z2s[kZ];
                bool wide = false;  // a zero-point outside [0, 15]: split by zp_split
#pragma unroll
                for (int gi = 0; gi < NG; ++gi) scur[gi] = bf16_to_f32(snext[gi]);
#pragma unroll
                for (int i = 0; i < kZ; ++i) {
                    float zl = bf16_to_f32(znext[i]);
                    if (!W8 && !(zl >= 0.0f && zl <= 15.0f)) {
                        float zh;
                        zl = zp_split(zl, zh);
                        wide = true;
                    }
                    const float zc = 128.0f + zl;  // 128 .. 143: exact in bf16
                    z2s[i] = pack_bf16x2(zc, zc);
                }
                sp += sp_step;
                if (ks + 1 < ks1) {
#pragma unroll
                    for (int gi = 0; gi < NG; ++gi) snext[gi] = sp[s_per_row ? 0 : gi];
                    if (!W8) {
#pragma unroll
                        for (int i = 0; i < kZ; ++i) znext[i] = zbase[zidx(ks + 1, i)];
                    }
                }
                uint32_t A[kKPerWarp / 2];
                if (W8) {
                    // int8 codes are the operand itself: q exactly in bf16, natural k order
#pragma unroll
                    for (int i = 0; i < kCh; ++i) {
                        int8x8_bf16(wv[i].x, wv[i].y, A + i * 8);
                        int8x8_bf16(wv[i].z, wv[i].w, A + i * 8 + 4);
                    }
                    tmem_st16(a_addr + ar.slot * 64u, A);
                    tmem_st16(a_addr + ar.slot * 64u + 16u, A + 16);
                } else
#pragma unroll
                for (int i = 0; i < kChunksPerWarp; ++i) {
                    // zero-point of this 32-k chunk (a chunk never straddles a group: g >= 32)
                    const uint32_t z2 = z2s[kOneZ ? 0 : i];
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const uint32_t v = word_of4(wv[i], w);
                        const uint32_t v4 = v >> 4;
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const uint32_t t = __byte_perm(v, v4, (uint32_t)(j | (j << 4) | ((4 + j) << 8) | ((4 + j) << 12)));
                            A[i * 16 + w * 4 + j] = bf2_sub(lop_and_or(t, nib_mask, bf16_magic), z2);
                        }
                    }
                    // each 32-k chunk goes to tensor memory as soon as it is ready
                    tmem_st16(a_addr + ar.slot * 64u + (uint32_t)(i * 16), A + i * 16);
                }
                tmem_wait_st();
                tc_fence_before();
                if (wide) wide_mark[ar.slot] = (int)it + 1;  // rare: tell the MMA warp to sum the activations
                __syncwarp();
                // tcgen05.st consumed the registers computed from the loaded codes, so no read of the
                // weight slot can still be pending: hand both the slot and the A buffer over
                if (lane == 0) {
                    mbar_arrive(&w_empty[wr.slot]);
                    mbar_arrive(&a_full[ar.slot]);
                }
                wr.next(kWStagesK);
                ar.next(kABufs);
                // promote the previous stage of this segment while this one is multiplied
                if (ks > ks0) promote(ks - 1);
#pragma unroll
                for (int gi = 0; gi < NG; ++gi) sprev[gi] = scur[gi];
            }
            promote(ks1 - 1);  // the segment's last stage

            // ---- segment output ----
            const int64_t mbase = mt * BN + kq * kCols;
            const bool whole = (ks0 == 0 && ks1 == spt);
            if (whole) {
                if (n < N) {
#pragma unroll
                    for (int c = 0; c < kCols; ++c)
                        if (mbase + c < M) y[(mbase + c) * N + n] = f32_to_bf16(acc[c]);
                }
            } else {
                // 32- and 64-column tiles: the CTA of the tile's first segment combines it (that segment ends its
                // range, while the tile's last segment starts the next CTA's, so it is usually among the last to
                // finish); the others write their slots and add their stage counts with release semantics, and
                // the first keeps its sums in registers and waits (bounded) until the counter shows every other
                // stage.  128-column tiles: the CTA that completes the tile combines it (the first-segment wait
                // measured much slower in this form).
                constexpr bool kFirstCombines = BN < 128;
                const int64_t cta_first = S.cta_of(tile * spt);
                const int64_t my_seg = (int64_t)blockIdx.x - cta_first;
                const int64_t cta_last = S.cta_of(tile * spt + spt - 1);
                if (!kFirstCombines || my_seg != 0) {
                    float *slot = ws + ((tile * max_segs + my_seg) * BN) * kTileN;
#pragma unroll
                    for (int c = 0; c < kCols; ++c) slot[(int64_t)(kq * kCols + c) * kTileN + r] = acc[c];
                    __threadfence();
                    named_bar_sync(1, kDequantWarps * 32);
                    if (tid == kFirstDequantWarp * 32) {
                        const int add = ks1 - ks0;
                        if (kFirstCombines) {
                            red_add_release(counters + tile, add);
                            *last_flag = 0;
                        } else {
                            const int prev = atomicAdd(counters + tile, add);
                            *last_flag = (prev + add == spt) ? 1 : 0;
                        }
                    }
                } else if (tid == kFirstDequantWarp * 32) {
                    const int others = spt - (ks1 - ks0);
                    int arrived = 1;
                    const uint64_t t0 = global_ns();
                    while (ld_acquire(counters + tile) != others) {
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
                named_bar_sync(1, kDequantWarps * 32);
                if (*last_flag) {
                    // sum the segments in segment order (this CTA's own from registers), so repeated calls round
                    // identically
                    __threadfence();
                    float tot[kCols];
#pragma unroll
                    for (int c = 0; c < kCols; ++c) tot[c] = 0.0f;
                    for (int64_t o = 0; o <= cta_last - cta_first; ++o) {
                        const float *other = ws + ((tile * max_segs + o) * BN) * kTileN;
#pragma unroll
                        for (int c = 0; c < kCols; ++c)
                            tot[c] += (o == my_seg) ? acc[c] : __ldcg(other + (int64_t)(kq * kCols + c) * kTileN + r);
                    }
#pragma unroll
                    for (int c = 0; c < kCols; ++c) acc[c] = tot[c];
                    if (n < N) {
#pragma unroll
                        for (int c = 0; c < kCols; ++c)
                            if (mbase + c < M) y[(mbase + c) * N + n] = f32_to_bf16(acc[c]);
                    }
                    named_bar_sync(1, kDequantWarps * 32);
                    if (tid == kFirstDequantWarp * 32) atomicExch(counters + tile, 0);
                }
            }
            u += ks1 - ks0;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (wid == 1) tmem_dealloc(tmem, kTmemCols);
}

// Failure-path tests: the (tile, stage) unit whose weight copy the next launch leaves out (-1: none).  Set
// by wq_test_skip_weight_copy, consumed by one launch.
std::atomic<int64_t> g_skip_unit{-1};

int64_t test_take_skip_unit() { return g_skip_unit.exchange(-1); }

template <int BN, int GROUP, bool W8>
int run(const uint16_t *x, int64_t M, int64_t N, int64_t K, const uint8_t *q, const uint16_t *s, const uint16_t *z,
        int s_per_row, uint16_t *y, void *workspace, int *status, cudaStream_t st)
{
    using C = Cfg<BN, W8>;
    CUtensorMap wmap, xmap;
    const uint64_t rowb = W8 ? (uint64_t)K : (uint64_t)(K / 2);
    if (!encode_tmap_2d(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, rowb, (uint64_t)N, rowb, C::kWRowBytes, kTileN,
                        W8 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
        return -1;
    if (!encode_tmap_2d(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, 64, BN,
                        CU_TENSOR_MAP_SWIZZLE_128B))
        return -1;
    auto kern = gemm_w4a16_tc_kernel<BN, GROUP, W8>;
    // at least 120 KB so that one CTA owns each SM (and its tensor memory)
    const size_t smem = std::max<size_t>(C::kBytes + 1024, 120 * 1024);
    static std::mutex mu;
    static std::map<int, int> sms_of;  // per device, for this instantiation: SM count once its attribute is set
    int dev = 0;
    cudaGetDevice(&dev);
    int sms;
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = sms_of.find(dev);
        if (it == sms_of.end()) {
            int v = 148, optin = 0;
            cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
            cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
            it = sms_of.emplace(dev, v).first;
        }
        sms = it->second;
    }
    const int64_t tiles = ((N + kTileN - 1) / kTileN) * ((M + BN - 1) / BN);
    const int64_t total = tiles * (K / kStageK);
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(total, sms));
    const int max_segs = (int)gemm_tc_max_segments(total, grid, K / kStageK);
    uint8_t *w8 = static_cast<uint8_t *>(workspace);
    int *counters = reinterpret_cast<int *>(w8);
    float *ws = reinterpret_cast<float *>(w8 + counter_region_bytes(tiles));
    if (clear_extra_counters(workspace, tiles, st) != cudaSuccess) return -2;
    kern<<<(unsigned)grid, kThreads, smem, st>>>(wmap, xmap, M, N, K, s, z, y, ws, counters, max_segs, status,
                                                  0x000F000Fu, 0x43004300u, W8 ? -1 : test_take_skip_unit(),
                                                  s_per_row);
    return 0;
}

}  // namespace

int gemm_tc_bn(int64_t M, int g)
{
    const int by_m = M <= 32 ? 32 : (M <= 64 ? 64 : 128);
    const int by_g = g; // tensor-memory budget: 2 stages x (128 / g) groups x BN <= 256 columns
    return by_m < by_g ? by_m : by_g;
}

int64_t gemm_tc_max_segments(int64_t total, int64_t grid, int64_t spt)
{
    const int64_t per = total / grid;  // >= 1
    return (spt + per - 1) / per + 1;
}

// Tile width (activation rows) of the W4A16 tensor-core call: 128 when the split-role kernel runs it
// (g = 128, K a multiple of 1024: for every M > 16, since a stage costs the tensor core the same for any
// N <= 128), else gemm_tc_bn.
int gemm_tc_w4_bn(int64_t M, int64_t K, int g)
{
    return (g == 128 && K % 1024 == 0) ? 128 : gemm_tc_bn(M, g);
}

size_t gemm_tc_partials_bytes(int64_t M, int64_t N, int64_t K, int BN)
{
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t tiles = ((N + kTileN - 1) / kTileN) * ((M + BN - 1) / BN);
    const int64_t spt = K / kStageK;
    const int64_t total = tiles * spt;
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(total, sms));
    const int64_t segs = gemm_tc_max_segments(total, grid, spt);
    const size_t b = sizeof(float) * (size_t)(tiles * segs * BN * kTileN);
    return (b + 255) / 256 * 256;
}

bool gemm_tc_eligible(int64_t M, int64_t N, int64_t K, int g)
{
    // M > 16; also 2 <= M <= 16 for groups of 32 and 64, which the TMA decode kernel does not take (the
    // tensor cores still beat the CUDA-core kernel there: it spends one FMA per code and row of x); and
    // 9 <= M <= 16 with g = 128 and K % 1024 == 0 (the 128 x 128-tile kernel), except up to 12 rows where the
    // persistent small-batch kernel runs with three weight stages.  Measured on B200 (K = 8192, N = 28672):
    // the 128 x 128-tile kernel takes 70 us at any M from 8 to 16; the small-batch kernels 43.8 us at M = 8
    // but 99-101 us at M = 12 and 16 (two column tiles of 8, and two stages or the older TMA kernel where the
    // activations take the room); on K = N = 8192 (three stages) the persistent one is ahead at M = 12 (29.1
    // against 31.4 us) and behind at M = 16 (33.9 against 31.3 us).
    const bool tc_small_batch =
        g == 128 && K % 1024 == 0 && M >= 9 && M <= 16 && !(M <= 12 && gemv_mt_stages(M, N, K, g) == 3);
    const bool m_ok = M > 16 || (M >= 2 && (g == 32 || g == 64)) || tc_small_batch;
    return m_ok && N >= kTileN && K >= kStageK && K % kStageK == 0 && (g == 32 || g == 64 || g == 128) &&
           K / 2 <= 0xffffffffLL && M <= 0x7fffffffLL;
}

size_t gemm_tc_workspace_bytes(int64_t M, int64_t N, int64_t K, int g)
{
    if (!gemm_tc_eligible(M, N, K, g)) return 0;
    const int BN = gemm_tc_w4_bn(M, K, g);
    const int64_t tiles = ((N + kTileN - 1) / kTileN) * ((M + BN - 1) / BN);
    return counter_region_bytes(tiles) + gemm_tc_partials_bytes(M, N, K, BN);
}

int launch_gemm_w4a16_tc(const uint16_t *x, int64_t M, int64_t N, int64_t K, const uint8_t *q, const uint16_t *s,
                         const uint16_t *z, int g, uint16_t *y, void *workspace, int *status, cudaStream_t st)
{
    const int bn = gemm_tc_bn(M, g);
    // g = 128 with K a multiple of 1024 runs the form with dequantisation and promotion in separate warps
    // (128 x 128 tiles for every M here; measured faster than the narrower tiles below at M = 32 too)
    if (gemm_tc_w4_bn(M, K, g) == 128 && g == 128 && K % 1024 == 0)
        return launch_gemm_w4a16_tc2(x, M, N, K, q, s, z, y, workspace, status, st, test_take_skip_unit());
    if (g == 32) return run<32, 32, false>(x, M, N, K, q, s, z, 0, y, workspace, status, st);
    if (g == 64) return bn == 32 ? run<32, 64, false>(x, M, N, K, q, s, z, 0, y, workspace, status, st)
                                 : run<64, 64, false>(x, M, N, K, q, s, z, 0, y, workspace, status, st);
    if (bn == 32) return run<32, 128, false>(x, M, N, K, q, s, z, 0, y, workspace, status, st);
    if (bn == 64) return run<64, 128, false>(x, M, N, K, q, s, z, 0, y, workspace, status, st);
    return run<128, 128, false>(x, M, N, K, q, s, z, 0, y, workspace, status, st);
}

bool gemm_tc_w8_eligible(int64_t M, int64_t N, int64_t K, int g)
{
    return M >= 2 && N >= kTileN && K >= kStageK && K % kStageK == 0 &&
           (g == 32 || g == 64 || g == 128 || (int64_t)g == K) && K <= 0x7fffffffLL && M <= 0x7fffffffLL;
}

// The promotion group of an int8 call: its group size, or 128 (one stage) for one scale per row.
static int w8_group(int64_t K, int g) { return (int64_t)g == K ? 128 : g; }

size_t gemm_tc_w8_workspace_bytes(int64_t M, int64_t N, int64_t K, int g)
{
    if (!gemm_tc_w8_eligible(M, N, K, g)) return 0;
    const int ge = w8_group(K, g);
    const int BN = gemm_tc_bn(M, ge);
    const int64_t tiles = ((N + kTileN - 1) / kTileN) * ((M + BN - 1) / BN);
    return counter_region_bytes(tiles) + gemm_tc_partials_bytes(M, N, K, BN);
}

int launch_gemm_w8a16_tc(const uint16_t *x, int64_t M, int64_t N, int64_t K, const int8_t *q8, const uint16_t *s,
                         int g, uint16_t *y, void *workspace, int *status, cudaStream_t st)
{
    const uint8_t *q = reinterpret_cast<const uint8_t *>(q8);
    const int ge = w8_group(K, g);
    const int per_row = (int64_t)g == K ? 1 : 0;
    const int bn = gemm_tc_bn(M, ge);
    if (ge == 32) return run<32, 32, true>(x, M, N, K, q, s, nullptr, per_row, y, workspace, status, st);
    if (ge == 64) return bn == 32 ? run<32, 64, true>(x, M, N, K, q, s, nullptr, per_row, y, workspace, status, st)
                                  : run<64, 64, true>(x, M, N, K, q, s, nullptr, per_row, y, workspace, status, st);
    if (bn == 32) return run<32, 128, true>(x, M, N, K, q, s, nullptr, per_row, y, workspace, status, st);
    if (bn == 64) return run<64, 128, true>(x, M, N, K, q, s, nullptr, per_row, y, workspace, status, st);
    return run<128, 128, true>(x, M, N, K, q, s, nullptr, per_row, y, workspace, status, st);
}

}  // namespace wq

// Test hook of the failure path (declared in wq.h): the next tensor-core W4A16 launch leaves out the weight
// copy of (tile, stage) unit `unit`, so the waits on it run out.
extern "C" void wq_test_skip_weight_copy(int64_t unit) { wq::g_skip_unit.store(unit); }

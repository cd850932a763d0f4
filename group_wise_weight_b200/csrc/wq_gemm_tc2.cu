// wq_gemm_tc2.cu -- W4A16 matmul at batch sizes above 16 with groups of 128
// (a 128 x 128 tile per CTA), on the 5th-generation tensor cores, with
// dequantisation and promotion in separate warps.
//
// The arithmetic is that of wq_gemm_tc.cu ("Quantization for LLM inference:
// FP8, INT4 (GPTQ, AWQ) and GGUF", "The minimum maths": w_hat = s (q - z);
// "Quantization Methods Compared ...", "Hardware, formats and the roofline":
// at batch 128 the matmul is a dense contraction, 4-bit weights are expanded
// inside the kernel): the MMA takes the exact integers q - z from tensor
// memory, each group of 128 k accumulates into its own tensor-memory region,
// and s is applied in binary32 ("promotion", y += s * D_group).  What differs
// is who does what:
//  * warp 0 loads weight stages (TMA, 64-byte swizzle) and the scale and
//    zero-point windows, warp 2 activation stages (TMA, 128-byte swizzle),
//    warp 1 allocates tensor memory, and lane 0 of warps 1 and 3 issue the
//    MMAs of alternate stages (A from tensor memory, B from shared memory);
//  * warps 4..11 (two warpgroups) only dequantise: codes from shared memory
//    to bf16 q - z in registers, stored into one of two tensor-memory A
//    buffers as soon as the MMA two stages back has freed it;
//  * warps 12..19 (two warpgroups) only promote, each thread holding 64 of its
//    row's binary32 accumulators (warpgroup c has columns 64c .. 64c + 63),
//    and write the output.
// Per stage an MMA lane waits twice (activations landed; the stage's A
// written and its D buffer promoted, one barrier that the dequantisation and
// promotion warps both arrive on) and commits once: a single "MMA done"
// barrier tells the activation producer, the dequantisation warps and the
// promotion warps alike that the stage's buffers may be reused or read.
// (Measured: a 128 x 128 x 16 MMA with A in tensor memory occupies the tensor
// core ~94 cycles, so 8 per stage ~750; issuing them blocks the lane for about
// that long, and the lane's commit, arrive and next waits then took ~400
// cycles in which the tensor core had nothing queued -- hence two lanes.)
// Register budgets follow the roles (setmaxnreg): 640 threads at launch x 96
// registers = 61,440 = 128 x 48 + 256 x 72 + 256 x 144.  Waits
// are inlined (no calls): ptxas allocates registers per role only for
// straight-line code.
// Scales and zero-points reach shared memory by TMA in windows of 8 groups x
// 128 rows, issued by the weight producer (needs K % 1024 == 0 for the
// windows' row stride; other K take wq_gemm_tc.cu).  Tensor memory: two A
// buffers of 64 columns and three D buffers of 128, so the MMAs of a stage
// wait for the promotion of the stage three back (with two, the chain of MMA
// completion, promotion and the next issue set the stage time; three were
// measured 5.7% faster on the 8-layer step, a fourth does not fit).  A zero-point outside [0, 15]
// is split as in wq_gemm_tc.cu: the dequantisation warps record z_hi per row
// and mark the stage; when a promotion warp finishes a window's stages it sums
// each marked stage's activations for its 64 columns from global memory (in k
// order) and adds -s z_hi times the sums.  A window's 8 scales reach the
// promotion warps' registers in one load, so no stage waits on a scale.  The dequantisation and promotion warps do not leave their loops
// when a wait fails (the abort flag makes every later wait return at once), so
// their warp-level and named barriers stay matched.
// Stream-K over (tile, stage) units, per-segment binary32 partials summed in
// segment order.  Every wait is bounded.
#include <algorithm>
#include <atomic>
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
constexpr int kBN = 128;        // activation rows per tile (MMA N)
constexpr int kStageK = 128;    // k per stage = one group
constexpr int kWStages = 6;
constexpr int kXStages = 4;
constexpr int kABufs = 2;        // dequantised A stages in tensor memory (64 columns each)
constexpr int kDBufs = 3;        // accumulator stages in tensor memory (128 columns each)
constexpr int kRing = 4;        // stage-ready / MMA-done barriers, indexed by stage % kRing
constexpr int kWideRing = 16;   // far-zero-point records, indexed by stage % kWideRing
constexpr int kThreads = 640;
constexpr int kFirstDq = 4, kDqWarps = 8, kFirstPr = 12, kPrWarps = 8;
constexpr int kRegCtl = 48, kRegDq = 72, kRegPr = 144;
constexpr int kWeightStageBytes = kTileN * (kStageK / 2);  // 8 KB
constexpr int kXAtomBytes = kBN * 128;                     // 128 rows x 64 bf16
constexpr int kXStageBytes = 2 * kXAtomBytes;              // 32 KB
constexpr uint32_t kTmemCols = 512;                        // A 2 x 64, D 3 x 128
constexpr int kWinGroups = 8;                              // groups (stages) per s / z window
constexpr int kWinSlots = 2;                               // windows in flight per ring
constexpr int kWinBytes = kTileN * kWinGroups * 2;         // 128 rows x 8 bf16 = 2 KB
constexpr size_t kWOff = (size_t)kXStages * kXStageBytes;
constexpr size_t kZwOff = kWOff + (size_t)kWStages * kWeightStageBytes;  // zero-point windows
constexpr size_t kSwOff = kZwOff + (size_t)kWinSlots * kWinBytes;        // scale windows
constexpr size_t kBarOff = kSwOff + (size_t)kWinSlots * kWinBytes;
// x_full[XS]; w_full, w_empty [WS]; ready, done [R]; zw_full, zw_empty, sw_full, sw_empty [2]; drain
constexpr int kBars = kXStages + 2 * kWStages + 2 * kRing + 4 * kWinSlots + 1;
constexpr size_t kFlagOff = kBarOff + (size_t)kBars * 8;
// flags: abort, last-arrival, tensor-memory address
constexpr size_t kMarkOff = kFlagOff + 64;                    // [kWideRing] far-zero-point marks
constexpr size_t kZhiOff = kMarkOff + kWideRing * 4;          // [kWideRing][row] z_hi
constexpr size_t kSmemBytes = kZhiOff + kWideRing * kTileN * 4;

static_assert(kRing >= kXStages && kRing >= kABufs && kRing > kDBufs, "stage rings must cover the buffers");
static_assert(kABufs * 64 + kDBufs * kBN <= (int)kTmemCols, "tensor memory");
// a record is read when the promotion finishes its stage's window (at most 7 stages later); the dequantisation
// warps reach stage j + kWideRing only after the promotion has freed the D buffer of stage j + kWideRing - 6
static_assert(kWideRing >= kWinGroups + kABufs + kDBufs, "far-zero-point records must outlive their window's promotion");
static_assert(kWOff % 1024 == 0 && kZwOff % 128 == 0 && kSwOff % 128 == 0, "TMA destinations");
static_assert(4 * kRegCtl + kDqWarps * kRegDq + kPrWarps * kRegPr <= (65536 / kThreads) / 8 * 8 * (kThreads / 32),
              "register budgets exceed the launch's registers");

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

template <int N>
__device__ __forceinline__ void setmaxnreg_dec()
{
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void setmaxnreg_inc()
{
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

__device__ __forceinline__ uint32_t word_of4(const uint4 &v, int i)
{
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

__device__ __forceinline__ uint32_t lop_and_or(uint32_t t, uint32_t mask, uint32_t magic)
{
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(t), "r"(mask), "r"(magic));
    return d;
}

// `count` arrivals at once (the promotion warps' share of the first two stages, whose D buffers start free).
__device__ __forceinline__ void mbar_arrive_n(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Programmatic dependent launch: let the next kernel in the stream start launching, and wait until the
// preceding one has completed and its memory is visible.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity, int *status)
{
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_ns() - t0 > kWaitLimitNs) { record_timeout(status); return; }
}

__global__ void __launch_bounds__(kThreads, 1)
gemm_w4a16_tc2_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap xmap,
                      const __grid_constant__ CUtensorMap smap, const __grid_constant__ CUtensorMap zmap,
                      const uint16_t *__restrict__ x, int64_t M, int64_t N, int64_t K, uint16_t *__restrict__ y,
                      float *__restrict__ ws, int *__restrict__ counters, int max_segs, int *__restrict__ status,
                      uint32_t nib_mask, uint32_t bf16_magic, int64_t skip_unit)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    uint64_t *x_full = reinterpret_cast<uint64_t *>(smem + kBarOff);
    uint64_t *w_full = x_full + kXStages;
    uint64_t *w_empty = w_full + kWStages;
    uint64_t *ready = w_empty + kWStages;  // stage A written (8 dequant warps) and its D buffer free (8 promotion)
    uint64_t *done = ready + kRing;        // the stage's MMAs completed (commit) and the MMA lane's release
    uint64_t *zw_full = done + kRing;
    uint64_t *zw_empty = zw_full + kWinSlots;
    uint64_t *sw_full = zw_empty + kWinSlots;
    uint64_t *sw_empty = sw_full + kWinSlots;
    uint64_t *drain = sw_empty + kWinSlots;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kFlagOff);
    volatile int *last_flag = abort_flag + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kFlagOff + 16);
    volatile int *wide_mark = reinterpret_cast<volatile int *>(smem + kMarkOff);       // [kWideRing]
    float *zhi = reinterpret_cast<float *>(smem + kZhiOff);                             // [kWideRing][row]

    const int tid = threadIdx.x, wid = tid >> 5, lane = tid & 31;
    Sched S;
    S.n_tiles = (N + kTileN - 1) / kTileN;
    S.tiles = S.n_tiles * ((M + kBN - 1) / kBN);
    S.spt = K / kStageK;
    S.total = S.tiles * S.spt;
    S.per = S.total / gridDim.x;
    S.extra = S.total % gridDim.x;
    const int64_t beg = S.begin_of(blockIdx.x);
    const int64_t end = beg + S.per + ((int64_t)blockIdx.x < S.extra ? 1 : 0);
    const int spt = (int)S.spt;

    // The next call's CTAs may start as this grid's CTAs leave their SMs: they set up, load weights, scales
    // and zero-points and dequantise, and wait for this grid to finish before they read x or write anything
    // to global memory (y, the workspace).
    pdl_launch_dependents();
    if (tid == 0) {
        for (int i = 0; i < kXStages; ++i) mbar_init(&x_full[i], 1);
        for (int i = 0; i < kWStages; ++i) {
            mbar_init(&w_full[i], 1);
            mbar_init(&w_empty[i], kDqWarps);
        }
        for (int i = 0; i < kRing; ++i) {
            mbar_init(&ready[i], kDqWarps + kPrWarps);
            mbar_init(&done[i], 2);  // the MMAs' completion and the MMA lane's arrive
        }
        for (int i = 0; i < kWinSlots; ++i) {
            mbar_init(&zw_full[i], 1);
            mbar_init(&zw_empty[i], kDqWarps);
            mbar_init(&sw_full[i], 1);
            mbar_init(&sw_empty[i], kPrWarps);
        }
        mbar_init(drain, 2);  // one commit per MMA lane
        for (int i = 0; i < kWideRing; ++i) wide_mark[i] = 0;
        *abort_flag = 0;
        *last_flag = 0;
        fence_mbar_init();
        // the first kDBufs stages find their D buffers free
        for (int i = 0; i < kDBufs; ++i) mbar_arrive_n(&ready[i], kPrWarps);
    }
    if (wid == 1) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t d_tmem = tmem + kABufs * 64u;  // D buffer b at column kABufs * 64 + b * 128

    if (wid < kFirstDq) {
        setmaxnreg_dec<kRegCtl>();
        if (wid == 0 && lane == 0 && beg < end) {
            // ------------------------------ weight and s / z producer ------------------------------
            Ring rg;
            uint32_t issued = 0, wins = 0;
            int64_t tile = beg / spt;
            int ks = (int)(beg - tile * spt);
            for (int64_t u = beg; u < end; ++u) {
                if (issued >= (uint32_t)kWStages && !mbar_wait(&w_empty[rg.slot], rg.phase ^ 1u, status, abort_flag))
                    break;
                const int nt = (int)(tile % S.n_tiles);
                if (u == beg || (ks % kWinGroups) == 0) {
                    // the s and z of groups (ks & ~7) .. + 7 of the tile's 128 rows, one window each
                    const uint32_t ws_ = wins % kWinSlots, wph = (wins / kWinSlots) & 1u;
                    if (wins >= (uint32_t)kWinSlots &&
                        (!mbar_wait(&zw_empty[ws_], wph ^ 1u, status, abort_flag) ||
                         !mbar_wait(&sw_empty[ws_], wph ^ 1u, status, abort_flag)))
                        break;
                    mbar_arrive_expect_tx(&zw_full[ws_], kWinBytes);
                    tma_load_2d(smem + kZwOff + ws_ * kWinBytes, &zmap, &zw_full[ws_], ks & ~(kWinGroups - 1), nt * kTileN);
                    mbar_arrive_expect_tx(&sw_full[ws_], kWinBytes);
                    tma_load_2d(smem + kSwOff + ws_ * kWinBytes, &smap, &sw_full[ws_], ks & ~(kWinGroups - 1), nt * kTileN);
                    ++wins;
                }
                // skip_unit (failure-path tests only, -1 otherwise): these weights are never requested
                if (u != skip_unit) {
                    mbar_arrive_expect_tx(&w_full[rg.slot], kWeightStageBytes);
                    tma_load_2d(smem + kWOff + rg.slot * kWeightStageBytes, &wmap, &w_full[rg.slot],
                                ks * (kStageK / 2), nt * kTileN);
                }
                ++issued;
                rg.next(kWStages);
                if (++ks == spt) { ks = 0; ++tile; }
            }
            for (uint32_t j = issued > (uint32_t)kWStages ? issued - kWStages : 0; j < issued; ++j) {
                if (beg + (int64_t)j == skip_unit) continue;
                drain_wait(&w_full[j % kWStages], (j / kWStages) & 1u, status);
            }
            for (uint32_t j = wins > (uint32_t)kWinSlots ? wins - kWinSlots : 0; j < wins; ++j) {
                drain_wait(&zw_full[j % kWinSlots], (j / kWinSlots) & 1u, status);
                drain_wait(&sw_full[j % kWinSlots], (j / kWinSlots) & 1u, status);
            }
        } else if (wid == 2 && lane == 0 && beg < end) {
            // ------------------------------ activation producer ------------------------------
            pdl_wait();  // x may be the preceding call's y
            uint32_t it = 0;
            int64_t tile = beg / spt;
            int ks = (int)(beg - tile * spt);
            for (int64_t u = beg; u < end; ++u, ++it) {
                // the slot's previous stage (it - kXStages) has been multiplied
                if (it >= (uint32_t)kXStages) {
                    const uint32_t p = it - kXStages;
                    if (!mbar_wait(&done[p % kRing], (p / kRing) & 1u, status, abort_flag)) break;
                }
                const int mt = (int)(tile / S.n_tiles);
                uint8_t *st = smem + (it % kXStages) * kXStageBytes;
                uint64_t *bar = &x_full[it % kXStages];
                mbar_arrive_expect_tx(bar, kXStageBytes);
                tma_load_2d(st, &xmap, bar, ks * kStageK, mt * kBN);
                tma_load_2d(st + kXAtomBytes, &xmap, bar, ks * kStageK + 64, mt * kBN);
                if (++ks == spt) { ks = 0; ++tile; }
            }
            for (uint32_t j = it > (uint32_t)kXStages ? it - kXStages : 0; j < it; ++j)
                drain_wait(&x_full[j % kXStages], (j / kXStages) & 1u, status);
        } else if ((wid == 1 || wid == 3) && lane == 0) {
            // ------------------------------ MMA issuers ------------------------------
            // Two lanes take alternate stages (warp 1 the even ones, warp 3 the odd ones): issuing a stage's
            // MMAs blocks a lane until the tensor core has nearly run them, so a single lane left the tensor
            // core idle while it committed and waited for the next stage.  Stages have their own A, D and
            // activation buffers, so the order in which the two lanes' MMAs run does not matter (making the
            // lanes take turns was measured slower), and each lane's commits track its own MMAs.
            constexpr uint32_t idesc = idesc_bf16_f32(128, kBN);
            const uint32_t xbase = smem_u32(smem);
            const uint32_t n_units = (uint32_t)(end - beg);
            for (uint32_t it = wid == 1 ? 0u : 1u; it < n_units; it += 2) {
                if (!mbar_wait(&x_full[it % kXStages], (it / kXStages) & 1u, status, abort_flag) ||
                    !mbar_wait(&ready[it % kRing], (it / kRing) & 1u, status, abort_flag))
                    break;
                tc_fence_after();
                const uint32_t xs = xbase + (it % kXStages) * (uint32_t)kXStageBytes;
                const uint32_t a_col = tmem + (it % kABufs) * 64u;
                const uint32_t d_col = d_tmem + (it % (uint32_t)kDBufs) * (uint32_t)kBN;
#pragma unroll
                for (int j = 0; j < kStageK / 16; ++j) {
                    const uint32_t baddr = xs + (uint32_t)(j >> 2) * kXAtomBytes + (uint32_t)(j & 3) * 32u;
                    tc_mma_ts(d_col, a_col + (uint32_t)j * 8u, smem_desc(baddr, 16, 1024, 2), idesc, j != 0 ? 1u : 0u);
                }
                tc_commit(&done[it % kRing]);
                // the second arrival on the stage's MMA-done barrier: a release by the thread that acquired
                // the stage's ready phase, so the promotion warps also see what the dequantisation warps wrote
                mbar_arrive(&done[it % kRing]);
            }
            tc_commit(drain);
            drain_wait(drain, 0, status);  // every MMA (both lanes') completes before tensor memory is released
        }
    } else if (wid < kFirstPr) {
        setmaxnreg_dec<kRegDq>();
        // ------------------------------ dequantisation ------------------------------
        const int dw = wid - kFirstDq;
        const int quarter = wid & 3;  // tensor-memory lanes 32 * quarter ..
        const int kq = dw >> 2;       // k half of each stage
        const int r = quarter * 32 + lane;
        const uint32_t lane_bits = (uint32_t)(quarter * 32) << 16;
        uint32_t w_addr[2];
#pragma unroll
        for (int i = 0; i < 2; ++i)
            w_addr[i] = smem_u32(smem + kWOff) + (uint32_t)r * 64u + 16u * ((uint32_t)(kq * 2 + i) ^ (uint32_t)((r >> 1) & 3));
        const uint32_t a_addr = tmem + lane_bits + (uint32_t)(kq * 32);
        Ring wr;
        uint32_t it = 0;
        int ks = (int)(beg % spt);
        int win = -1;  // s / z window in use (the producer's sequence: a new one at the start and every 8th group)
        const uint32_t zw_row = smem_u32(smem + kZwOff) + (uint32_t)r * (kWinGroups * 2);
        for (int64_t u = beg; u < end; ++u, ++it) {
            if (u == beg || (ks % kWinGroups) == 0) {
                if (win >= 0) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&zw_empty[win % kWinSlots]);
                }
                ++win;
                mbar_wait(&zw_full[win % kWinSlots], (uint32_t)(win / kWinSlots) & 1u, status, abort_flag);
            }
            uint16_t zraw;
            asm volatile("ld.shared.u16 %0, [%1];"
                         : "=h"(zraw)
                         : "r"(zw_row + (uint32_t)(win % kWinSlots) * kWinBytes + (uint32_t)(ks % kWinGroups) * 2u));
            mbar_wait(&w_full[wr.slot], wr.phase, status, abort_flag);
            uint4 wv[2];
#pragma unroll
            for (int i = 0; i < 2; ++i)
                asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(wv[i].x), "=r"(wv[i].y), "=r"(wv[i].z), "=r"(wv[i].w)
                             : "r"(w_addr[i] + wr.slot * (uint32_t)kWeightStageBytes));
            float zl = bf16_to_f32(zraw), zh = 0.0f;
            bool wide = false;
            if (!(zl >= 0.0f && zl <= 15.0f)) {
                zl = zp_split(zl, zh);
                wide = true;
            }
            const uint32_t z2 = bf16_pair_128_plus(zl);
            // the stage's q - z are formed in registers before the A buffer is waited for, so the stores
            // follow the MMA that frees it at once
            uint32_t A[32];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const uint32_t v = word_of4(wv[i], w);
                    const uint32_t v4 = v >> 4;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t t = __byte_perm(v, v4, (uint32_t)(j | (j << 4) | ((4 + j) << 8) | ((4 + j) << 12)));
                        A[i * 16 + w * 4 + j] = sub_bf16x2(lop_and_or(t, nib_mask, bf16_magic), z2);
                    }
                }
            }
            if (it >= (uint32_t)kABufs) {
                // the A buffer's previous stage (it - kABufs) has been multiplied
                const uint32_t p = it - kABufs;
                mbar_wait(&done[p % kRing], (p / kRing) & 1u, status, abort_flag);
                tc_fence_after();
            }
            const uint32_t a_slot = a_addr + (it % kABufs) * 64u;
            tmem_st16(a_slot, A);
            tmem_st16(a_slot + 16u, A + 16);
            if (kq == 0) zhi[(it % kWideRing) * kTileN + r] = zh;  // read by the promotion of a marked stage
            if (wide) wide_mark[it % kWideRing] = (int)it + 1;
            // announce the stage: stores complete, weights consumed
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&ready[it % kRing]);
                mbar_arrive(&w_empty[wr.slot]);
            }
            wr.next(kWStages);
            if (++ks == spt) ks = 0;
        }
        tmem_wait_st();
    } else {
        setmaxnreg_inc<kRegPr>();
        // ------------------------------ promotion and output ------------------------------
        const int pw = wid - kFirstPr;
        const int quarter = wid & 3;
        const int ch = pw >> 2;  // columns 64 ch .. 64 ch + 63
        const int r = quarter * 32 + lane;
        const uint32_t lane_bits = (uint32_t)(quarter * 32) << 16;
        const int ptid = tid - kFirstPr * 32;  // 0 .. 255
        uint32_t it = 0;
        int win = -1;  // s window in use (same sequence as the producer's)
        const uint32_t sw_row = smem_u32(smem + kSwOff) + (uint32_t)r * (kWinGroups * 2);
        // This row's 8 scales of the window in use (bf16; group g of the window at bits 16 (g % 4) of
        // sw[g / 4]), read with one 16-byte load when the window opens: a new window at the first unit and at
        // every 8th group, the previous one released (all of its scales are in registers by then).
        uint64_t sw[2] = {0, 0};
        auto open_window = [&]() {
            if (win >= 0) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&sw_empty[win % kWinSlots]);
            }
            ++win;
            mbar_wait(&sw_full[win % kWinSlots], (uint32_t)(win / kWinSlots) & 1u, status, abort_flag);
            uint4 w4;
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(w4.x), "=r"(w4.y), "=r"(w4.z), "=r"(w4.w)
                         : "r"(sw_row + (uint32_t)(win % kWinSlots) * kWinBytes));
            sw[0] = ((uint64_t)w4.y << 32) | w4.x;
            sw[1] = ((uint64_t)w4.w << 32) | w4.z;
        };
        auto scale_of = [&](int ks) -> float {
            const int g = ks & (kWinGroups - 1);
            const uint64_t w = g < 4 ? sw[0] : sw[1];
            return __uint_as_float((uint32_t)((w >> (16 * (g & 3))) & 0xFFFFu) << 16);
        };
        if (beg < end) open_window();
        pdl_wait();  // y and the workspace may still be in use by the preceding call until it completes
        // A failed wait does not end the loop: the abort flag makes every later wait return at once, and all
        // promotion warps keep taking the same named barriers.
        for (int64_t u = beg; u < end;) {
            const int64_t tile = u / spt;
            const int ks0 = (int)(u - tile * spt);
            const int ks1 = (int)std::min<int64_t>(spt, ks0 + (end - u));
            const int64_t nt = tile % S.n_tiles, mt = tile / S.n_tiles;
            const int64_t n = nt * kTileN + r;
            float acc[64];
#pragma unroll
            for (int c = 0; c < 64; ++c) acc[c] = 0.0f;
            int ks_w0 = ks0;  // first group of the window's stages not yet checked for far zero-points
            for (int ks = ks0; ks < ks1; ++ks, ++it) {
                // the stage's MMAs are complete (and, through the MMA lane's arrive, the dequantisation warps'
                // far-zero-point record of the stage is visible)
                mbar_wait(&done[it % kRing], (it / kRing) & 1u, status, abort_flag);
                tc_fence_after();
                const uint32_t dcol = d_tmem + lane_bits + (it % (uint32_t)kDBufs) * (uint32_t)kBN + (uint32_t)(ch * 64);
                uint32_t v[64];
                tmem_ld32(dcol, v);
                tmem_ld32(dcol + 32u, v + 32);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                // the D buffer is free for stage it + kDBufs as soon as it is in registers
                if (lane == 0) mbar_arrive(&ready[(it + kDBufs) % kRing]);
                const float s = scale_of(ks);
                const f32x2 s2{s, s};
#pragma unroll
                for (int i = 0; i < 64; i += 2) {
                    const f32x2 r2 = fma2_pairs(s2, f32x2{__uint_as_float(v[i]), __uint_as_float(v[i + 1])},
                                                f32x2{acc[i], acc[i + 1]});
                    acc[i] = r2.x;
                    acc[i + 1] = r2.y;
                }
                if ((ks & (kWinGroups - 1)) == kWinGroups - 1 || ks + 1 == ks1) {
                    // the window's last stage here: its marked stages get -s z_hi times their activation sums
                    // (lane l sums tokens 64 ch + l and 64 ch + 32 + l over the stage's 128 k, 16-byte chunks in
                    // k order, from global memory); lane 0 reads each mark, so branches are warp-uniform
                    // lane l looks at the window's l-th checked stage; one ballot gives the marked ones
                    const int nchk = ks - ks_w0 + 1;  // 1 .. 8
                    const uint32_t jl = it - (uint32_t)(ks - ks_w0) + (uint32_t)lane;
                    const uint32_t marked =
                        __ballot_sync(0xffffffffu, lane < nchk && wide_mark[jl % kWideRing] == (int)jl + 1);
                    for (uint32_t mbits = marked; mbits != 0u; mbits &= mbits - 1u) {
                        const int kw = ks_w0 + __ffs((int)mbits) - 1;
                        const uint32_t jt = it - (uint32_t)(ks - kw);
                        float tsum[2];
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int64_t row = mt * kBN + ch * 64 + h * 32 + lane;
                            float t = 0.0f;
                            if (row < M) {
                                const uint4 *p = reinterpret_cast<const uint4 *>(x + row * K + (int64_t)kw * kStageK);
                                for (int c = 0; c < kStageK / 8; ++c) t += sum_bf16x8(__ldg(p + c));
                            }
                            tsum[h] = t;
                        }
                        const float zh = zhi[(jt % kWideRing) * kTileN + r];
                        const float t = -scale_of(kw) * zh;
#pragma unroll
                        for (int c = 0; c < 64; ++c) {
                            const float xs = __shfl_sync(0xffffffffu, tsum[c >> 5], c & 31);
                            if (zh != 0.0f) acc[c] = fmaf(t, xs, acc[c]);
                        }
                    }
                    ks_w0 = ks + 1;
                    // the next unit opens a new window (a multiple of 8 groups, or a new tile at group 0)
                    if ((int64_t)beg + it + 1 < end) open_window();
                }
            }

            // ---- segment output (this warpgroup's 64 columns) ----
            const int64_t mbase = mt * kBN + ch * 64;
            if (ks0 == 0 && ks1 == spt) {
                if (n < N) {
                    uint16_t *yp = y + mbase * N + n;
                    const int mlim = (int)std::max<int64_t>(0, std::min<int64_t>(64, M - mbase));
#pragma unroll
                    for (int c = 0; c < 64; ++c, yp += N)
                        if (c < mlim) *yp = f32_to_bf16(acc[c]);
                }
            } else {
                // Partial sums of a split tile: segment slot [column / 4][row][4] floats, so each thread writes
                // and reads its 64 columns as 16 float4 and a warp's access is 512 contiguous bytes.
                const int64_t cta_first = S.cta_of(tile * spt);
                const int64_t my_seg = (int64_t)blockIdx.x - cta_first;
                const int64_t nseg = S.cta_of(tile * spt + spt - 1) - cta_first + 1;
                auto seg_ptr = [&](int64_t o, int q) -> float4 * {  // this thread's float4 q (columns 4q..4q+3)
                    return reinterpret_cast<float4 *>(ws) +
                           ((tile * max_segs + o) * (kBN / 4) + ch * 16 + q) * kTileN + r;
                };
                // The CTA of the tile's first segment combines it: that segment ends its range, while the tile's
                // last segment starts the next CTA's, so it is usually among the last to finish.  The others write
                // their slots and add their stage counts with release semantics (no round trip); the first
                // keeps its sums in registers and waits (bounded) until the counter shows every other stage.
                if (my_seg != 0) {
#pragma unroll
                    for (int q = 0; q < 16; ++q)
                        *seg_ptr(my_seg, q) = make_float4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
                    __threadfence();
                    named_bar_sync(1, kPrWarps * 32);
                    if (ptid == 0) red_add_release(counters + tile, ks1 - ks0);
                    u += ks1 - ks0;
                    continue;
                }
                if (ptid == 0) {
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
                named_bar_sync(1, kPrWarps * 32);
                if (*last_flag) {
                    // sum the segments in segment order (this CTA's own first, from registers); 16 columns at a
                    // time, the next segment's values requested before the current ones are added
                    __threadfence();
#pragma unroll
                    for (int c0 = 0; c0 < 64; c0 += 16) {
                        float tot[16];
#pragma unroll
                        for (int c = 0; c < 16; ++c) tot[c] = 0.0f;
                        float4 nxt[4];
                        auto fetch = [&](int64_t o) {
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                nxt[q] = o == my_seg ? make_float4(0.f, 0.f, 0.f, 0.f) : __ldcg(seg_ptr(o, c0 / 4 + q));
                        };
                        fetch(0);
                        for (int64_t o = 0; o < nseg; ++o) {
                            float4 cur[4];
#pragma unroll
                            for (int q = 0; q < 4; ++q) cur[q] = nxt[q];
                            if (o + 1 < nseg) fetch(o + 1);
                            if (o == my_seg) {
#pragma unroll
                                for (int c = 0; c < 16; ++c) tot[c] += acc[c0 + c];
                            } else {
#pragma unroll
                                for (int q = 0; q < 4; ++q) {
                                    tot[4 * q] += cur[q].x;
                                    tot[4 * q + 1] += cur[q].y;
                                    tot[4 * q + 2] += cur[q].z;
                                    tot[4 * q + 3] += cur[q].w;
                                }
                            }
                        }
                        if (n < N) {
                            uint16_t *yp = y + (mbase + c0) * N + n;
                            const int mlim = (int)std::max<int64_t>(0, std::min<int64_t>(16, M - mbase - c0));
#pragma unroll
                            for (int c = 0; c < 16; ++c, yp += N)
                                if (c < mlim) *yp = f32_to_bf16(tot[c]);
                        }
                    }
                    named_bar_sync(1, kPrWarps * 32);
                    if (ptid == 0) atomicExch(counters + tile, 0);
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

}  // namespace

size_t gemm_tc2_smem_bytes() { return std::max<size_t>(kSmemBytes + 1024, 120 * 1024); }

int launch_gemm_w4a16_tc2(const uint16_t *x, int64_t M, int64_t N, int64_t K, const uint8_t *q, const uint16_t *s,
                          const uint16_t *z, uint16_t *y, void *workspace, int *status, cudaStream_t st,
                          int64_t skip_unit)
{
    CUtensorMap wmap, xmap;
    if (!encode_tmap_2d(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, (uint64_t)(K / 2), (uint64_t)N, (uint64_t)(K / 2),
                        kStageK / 2, kTileN, CU_TENSOR_MAP_SWIZZLE_64B))
        return -1;
    if (!encode_tmap_2d(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, 64, kBN,
                        CU_TENSOR_MAP_SWIZZLE_128B))
        return -1;
    // scales and zero-points [N][G] bf16 in windows of 8 groups x 128 rows (the row stride G * 2 bytes is a
    // multiple of 16 because K % 1024 == 0)
    CUtensorMap smap, zmap;
    const uint64_t G = (uint64_t)K / kStageK;
    if (!encode_tmap_2d(&smap, CU_TENSOR_MAP_DATA_TYPE_UINT16, s, G, (uint64_t)N, G * 2, kWinGroups, kTileN,
                        CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_tmap_2d(&zmap, CU_TENSOR_MAP_DATA_TYPE_UINT16, z, G, (uint64_t)N, G * 2, kWinGroups, kTileN,
                        CU_TENSOR_MAP_SWIZZLE_NONE))
        return -1;
    static std::mutex mu;
    static std::map<int, int> sms_of;
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
            cudaFuncSetAttribute(gemm_w4a16_tc2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
            it = sms_of.emplace(dev, v).first;
        }
        sms = it->second;
    }
    const int64_t tiles = ((N + kTileN - 1) / kTileN) * ((M + kBN - 1) / kBN);
    const int64_t total = tiles * (K / kStageK);
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(total, sms));
    const int max_segs = (int)gemm_tc_max_segments(total, grid, K / kStageK);
    uint8_t *w8 = static_cast<uint8_t *>(workspace);
    int *counters = reinterpret_cast<int *>(w8);
    float *ws = reinterpret_cast<float *>(w8 + counter_region_bytes(tiles));
    if (clear_extra_counters(workspace, tiles, st) != cudaSuccess) return -2;
    // programmatic dependent launch: this grid may start while the previous kernel in the stream finishes;
    // it reads nothing that kernel may write, and writes nothing, before griddepcontrol.wait
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = gemm_tc2_smem_bytes();
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, gemm_w4a16_tc2_kernel, wmap, xmap, smap, zmap, x, M, N, K, y, ws, counters,
                           max_segs, status, 0x000F000Fu, 0x43004300u, skip_unit) != cudaSuccess)
        return -2;
    return 0;
}

}  // namespace wq

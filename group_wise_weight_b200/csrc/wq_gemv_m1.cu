// wq_gemv_m1.cu -- W4A16, group 128, a single activation row (M = 1): the
// decode step of an LLM, bound by streaming the packed weights from HBM once.
//
// "Quantization Methods Compared: INT8, GPTQ, AWQ, FP8, FP4 and KV-Cache
// Quantization", section "Hardware, formats and the roofline": at batch 1 a
// decode step reads every weight once and does two flops per weight, so the
// kernel has to keep HBM streaming while spending as few issue slots per
// weight as possible on the dequantisation w_hat = s (q - z) ("Quantization
// for LLM inference: FP8, INT4 (GPTQ, AWQ) and GGUF", "The minimum maths").
//
// Why mma.sync at M = 1.  On CUDA cores every code costs one mixed
// bf16 x bf16 -> binary32 FMA, and that pipe saturates near 4.5 TB/s of
// packed weights on B200, below the HBM roofline.  One m16n8k16 tensor
// instruction instead takes the 256 codes of a 16-row x 16-k block (the
// activation vector fills all 8 columns of the other operand, so every lane
// ends up holding its rows' sums), leaving the LOP3 code extraction as the
// only per-code work.
//
// Memory pipeline.  TMA throughput on B200 depends on the size of each copy:
// copies of 2 KB stream at about 4 TB/s, copies of 8 KB and more at over
// 6 TB/s.  So one producer warp per CTA moves 32 KB per copy: a stage is 256
// rows x 2 groups, fetched through a 3-D view of the packed codes (64-byte
// group slices, rows, groups; the group stride is 64 bytes) that lands in
// shared memory as [group][row][64 B], so the consumers' 16-byte reads are
// free of bank conflicts.  Three stages are in flight; the scales and
// zero-points follow in [256 rows x 8 groups] boxes, double buffered.
//
// Work layout.
//  * A unit is (tile of 256 rows, pair of groups).  The grid is persistent
//    (one CTA per SM) and every CTA takes an equal contiguous range of units,
//    tile by tile along K (stream-K), so no SM idles behind a short last wave.
//  * Consumer warp w (16 of them) owns rows 16w .. 16w+15 of the tile.  Lane
//    (g, t) (g = lane / 4, t = lane % 4) reads 16 bytes -- codes 32t .. 32t+31
//    of the group -- of rows g and g + 8.  Each 32-bit word gives, with one
//    shift and one LOP3 per pair, the bf16 pairs (128 + q_i, 128 + q_{i+4})
//    of its part of the A operand of eight k16 steps; the k order inside a
//    step is permuted accordingly and the activation pairs are staged in
//    shared memory in the same permuted order.
//  * Subtracting the bf16 pair (128 + z, 128 + z) from each code pair gives
//    the exact integers q - z, so the tensor core sums x (q - z) per group and
//    the binary32 accumulator takes s * D: no term carries an offset that has
//    to cancel later, rows whose weights are all zero give exactly zero, and
//    the rounding error stays proportional to sum |x w_hat|.  A zero-point
//    outside [0, 15] is split (zp_split in wq_common.cuh): the operand is
//    q - z_lo and the lane adds -s z_hi times the group's activation sum.
//  * A tile split between CTAs leaves one binary32 partial per segment in the
//    workspace.  The consumers never wait on global memory for this: each
//    warp drops its 16 row sums into a double-buffered shared-memory tile and
//    moves on, and a separate combiner warp copies the tile to the
//    segment's slot, bumps the tile's arrival counter and, if it is the last
//    to arrive, sums the slots in segment order, writes y and re-zeroes the
//    counter -- a fixed order, so results do not depend on timing.
//  * x is copied into shared memory with one bulk asynchronous copy, then
//    permuted in place.
//  * Launched with programmatic dependent launch: in a stream of linears the
//    next kernel's CTAs start as SMs free up, initialise their barriers and
//    prefetch their first weight stages into L2 while this one finishes; they
//    read x and write anything only after griddepcontrol.wait.
//  * Every mbarrier wait is bounded; on a timeout the kernel records it in the
//    status word, the producer stops issuing, and every later wait returns at
//    once: the consumers finish their loop (on garbage) with unchanged control
//    flow, the producer waits (bounded) for its copies in flight, and the CTA
//    exits.  The workspace must then be zero-filled again before reuse.

#include "wq_common.cuh"
#include "wq_internal.h"
#include "wq_sm100.cuh"

#include <algorithm>
#include <map>
#include <mutex>

namespace wq {

namespace {

constexpr int kC = 16;                            // consumer warps
constexpr int kProducer = kC;                     // warp roles: consumers 0 .. kC-1, then these two
constexpr int kCombiner = kC + 1;
constexpr int kT = (kC + 2) * 32;                 // threads
constexpr int kTile = 16 * kC;                    // rows per tile (256)
constexpr int kStages = 3;                        // weight stages in flight
constexpr uint32_t kStageBytes = kTile * 128;     // 256 rows x 2 groups x 64 B
constexpr uint32_t kSzBytes = kTile * 16;         // 256 rows x 8 groups x 2 B (one of s or z)
constexpr uint32_t kBulkPiece = 16384;            // bytes per bulk copy of x
constexpr int kPairsPerWindow = 4;                // 8 groups of s/z = 4 units

// shared memory: [x pairs 2K][pad to 1024][stages][s/z windows][2 partial tiles][barriers]
__host__ __device__ __forceinline__ size_t m1_ring_offset(int64_t K)
{
    return ((size_t)K * 2 + 1023) & ~(size_t)1023;
}
__host__ __device__ __forceinline__ size_t m1_sz_offset(int64_t K) { return m1_ring_offset(K) + kStages * kStageBytes; }
__host__ __device__ __forceinline__ size_t m1_part_offset(int64_t K) { return m1_sz_offset(K) + 2 * 2 * kSzBytes; }
__host__ __device__ __forceinline__ size_t m1_bar_offset(int64_t K) { return m1_part_offset(K) + 2 * kTile * 4; }
// full/empty per stage, s/z full/empty x2, partial full/empty x2, x, flags (2 x 8 B)
constexpr int kBars = 2 * kStages + 4 + 4 + 1 + 2;
__host__ __device__ __forceinline__ size_t m1_smem_bytes(int64_t K) { return m1_bar_offset(K) + kBars * 8 + 1024; }

// (v >> sh) & mask | magic with both constants in registers: one LOP3.
__device__ __forceinline__ uint32_t nib_pair(uint32_t v, int sh, uint32_t mask, uint32_t magic)
{
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(v >> sh), "r"(mask), "r"(magic));
    return d;
}

// D += A B for one m16n8k16 step (bf16 in, binary32 accumulate); no side effects.
__device__ __forceinline__ void mma_bf16(float c[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 :: "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar, int x, int y, int z)
{
    asm volatile("cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];"
                 :: "r"(smem_u32(dst)), "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
                 : "memory");
}

// Bring a tensor-map box into L2 (no shared-memory destination, nothing to wait for).
__device__ __forceinline__ void tma_prefetch_l2_3d(const CUtensorMap *map, int x, int y, int z)
{
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global [%0, {%1, %2, %3}];" ::"l"(map), "r"(x), "r"(y), "r"(z)
                 : "memory");
}

// Programmatic dependent launch: let the next kernel in the stream start launching now, and wait until
// the previous kernel has completed and its writes are visible (no-ops for a normal launch).
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ uint4 lds128(uint32_t addr)
{
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(addr));
    return r;
}

__device__ __forceinline__ uint32_t lds_u32(uint32_t addr)
{
    uint32_t r;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(r) : "r"(addr));
    return r;
}

__device__ __forceinline__ uint32_t add_bf16x2(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t word_of(const uint4 &v, int i)
{
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// Device-scope add with acquire-release semantics: orders the writes that happen before it (this thread's,
// and through the preceding CTA barrier the other consumers') before the add, and later reads after it.
__device__ __forceinline__ int atom_add_acq_rel(int *p, int v)
{
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// The CTA whose equal share [units * b / B, units * (b + 1) / B) holds unit u.
__host__ __device__ __forceinline__ int64_t cta_of(int64_t u, int64_t units, int64_t B)
{
    return ((u + 1) * B - 1) / units;
}

// Eight activations divided by their input channels' scales: bf16(x / s) with an IEEE binary32 quotient
// (the activation side of per-input-channel scaling, wq_gemm_w4a16_colscaled).
__device__ __forceinline__ uint4 colscale8(uint4 v, const float *s)
{
    const float4 s0 = __ldg(reinterpret_cast<const float4 *>(s)), s1 = __ldg(reinterpret_cast<const float4 *>(s) + 1);
    const float sc[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
        w[i] = pack_bf16x2(__fdiv_rn(__uint_as_float(w[i] << 16), sc[2 * i]),
                           __fdiv_rn(__uint_as_float(w[i] & 0xffff0000u), sc[2 * i + 1]));
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Bounded wait used on the drain path (ignores the abort flag).
__device__ __forceinline__ void wait_drain(uint64_t *bar, uint32_t parity, int *status)
{
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_ns() - t0 > kWaitLimitNs) { record_timeout(status); return; }
}

// 18 warps put five on one SM sub-partition, whose register file holds 16K registers: at most 96 each.
__global__ void __maxnreg__(96)
gemv_w4a16_m1_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap smap,
                     const __grid_constant__ CUtensorMap zmap, const uint16_t *__restrict__ x, int N, int K,
                     uint16_t *__restrict__ y, float *__restrict__ ws, int *__restrict__ cnt, int max_segs,
                     int *__restrict__ status, uint32_t nib_mask, uint32_t bf16_magic,
                     const float *__restrict__ col_scale)
{
    extern __shared__ __align__(1024) uint8_t m1_raw[];
    // TMA destinations want 128-byte (we keep 1024-byte) alignment: align the base explicitly
    uint8_t *sm = m1_raw + ((1024u - (smem_u32(m1_raw) & 1023u)) & 1023u);
    uint4 *xp = reinterpret_cast<uint4 *>(sm);                    // K / 8 chunks of 8 activations
    uint8_t *ring = sm + m1_ring_offset(K);
    uint8_t *szr = sm + m1_sz_offset(K);                          // [2 windows][s, z][256 rows][8 groups]
    float *part = reinterpret_cast<float *>(sm + m1_part_offset(K));  // [2][256 rows] partial sums
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + m1_bar_offset(K));
    uint64_t *full = bars, *empty = bars + kStages;
    uint64_t *szfull = bars + 2 * kStages, *szempty = szfull + 2;
    uint64_t *pfull = szempty + 2, *pempty = pfull + 2;
    uint64_t *xbar = pempty + 2;
    volatile int *flags = reinterpret_cast<volatile int *>(xbar + 1);  // [0] abort, [1] last-arrival broadcast
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int G = K >> 7;
    const int P = G >> 1;  // group pairs (units) per tile

    pdl_launch_dependents();
    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kC);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&szfull[i], 1);
            mbar_init(&szempty[i], kC);
            mbar_init(&pfull[i], kC);
            mbar_init(&pempty[i], 1);
        }
        mbar_init(xbar, 1);
        flags[0] = 0;
        flags[1] = 0;
        fence_mbar_init();
    }
    __syncthreads();

    // ---- this CTA's equal share of the units ----
    const int ntiles = (N + kTile - 1) / kTile;
    const int64_t units = (int64_t)ntiles * P;
    const int64_t B = min((int64_t)gridDim.x, units);  // participating CTAs, each with >= 1 unit
    const int64_t bid = blockIdx.x;
    const int64_t beg = bid < B ? units * bid / B : units, end = bid < B ? units * (bid + 1) / B : units;
    const int n = (int)(end - beg);  // a CTA's share stays far below 2^31
    const int tile0 = (int)(beg / P), pair0 = (int)(beg - (int64_t)tile0 * P);

    // Under programmatic dependent launch the previous kernel may still be running.  Nothing it writes may
    // be read before pdl_wait().  The packed weights, scales and zero-points are inputs that the preceding
    // call does not write (a call of this kernel writes only y and its workspace; the library's other
    // kernels do not launch dependents early), so the producer issues the first stages and the first s/z
    // window into shared memory now, and only the activations wait.
    int pt = tile0, pp = pair0;  // producer position: tile, group pair
    int wins = 0;                // s/z windows issued
    int pi = 0;                  // stages issued
    auto issue_window = [&](int slot) {
        mbar_arrive_expect_tx(&szfull[slot], 2 * kSzBytes);
        uint8_t *d = szr + (uint32_t)slot * 2u * kSzBytes;
        const int g8 = (2 * pp) & ~7;
        tma_load_2d(d, &smap, &szfull[slot], g8, pt * kTile);
        tma_load_2d(d + kSzBytes, &zmap, &szfull[slot], g8, pt * kTile);
        ++wins;
    };
    if (wid == kProducer && lane == 0) {
        // at most two windows start within the first kStages pairs, so no window slot needs a wait here
        for (; pi < kStages && pi < n; ++pi) {
            if (pi == 0 || (pp & (kPairsPerWindow - 1)) == 0) issue_window(wins & 1);
            mbar_arrive_expect_tx(&full[pi], kStageBytes);
            tma_load_3d(ring + (uint32_t)pi * kStageBytes, &wmap, &full[pi], 0, pt * kTile, 2 * pp);
            if (++pp == P) { pp = 0; ++pt; }
        }
    }
    pdl_wait();

    if (wid == kProducer) {
        // ================================ producer ================================
        if (lane == 0 && n > 0) {
            // the part of x this CTA's units read (512 bytes per group pair): its pairs of the first tile,
            // and those of the next tile if the range wraps; all of x once the range spans a whole tile
            const uint32_t xbytes = (uint32_t)K * 2u;
            uint32_t r0 = 0, r1 = xbytes, w1 = 0;  // [r0, r1) and, when wrapping, [0, w1)
            if (n < P) {
                r0 = (uint32_t)pair0 * 512u;
                if (pair0 + n <= P) {
                    r1 = (uint32_t)(pair0 + n) * 512u;
                } else {
                    w1 = (uint32_t)(pair0 + n - P) * 512u;
                    if (w1 >= r0) { r0 = 0; w1 = 0; }  // the two pieces meet: all of x
                }
            }
            mbar_arrive_expect_tx(xbar, (r1 - r0) + w1);
            for (uint32_t o = r0; o < r1; o += kBulkPiece)
                bulk_g2s(sm + o, reinterpret_cast<const uint8_t *>(x) + o, min(kBulkPiece, r1 - o), xbar);
            for (uint32_t o = 0; o < w1; o += kBulkPiece)
                bulk_g2s(sm + o, reinterpret_cast<const uint8_t *>(x) + o, min(kBulkPiece, w1 - o), xbar);
            int i = pi;
            for (; i < n; ++i) {
                // s/z window: at every 4th pair of a tile
                if ((pp & (kPairsPerWindow - 1)) == 0) {
                    const int slot = wins & 1;
                    if (wins >= 2 && !mbar_wait(&szempty[slot], (uint32_t)((wins >> 1) - 1) & 1u, status, flags)) break;
                    issue_window(slot);
                }
                const int s = i % kStages;
                if (!mbar_wait(&empty[s], (uint32_t)(i / kStages - 1) & 1u, status, flags)) break;
                mbar_arrive_expect_tx(&full[s], kStageBytes);
                tma_load_3d(ring + (uint32_t)s * kStageBytes, &wmap, &full[s], 0, pt * kTile, 2 * pp);
                if (++pp == P) { pp = 0; ++pt; }
            }
            // drain: the copies issued last must land before the CTA can end (bounded, ignores abort)
            for (int j = max(0, i - kStages); j < i; ++j) wait_drain(&full[j % kStages], (uint32_t)(j / kStages) & 1u, status);
            for (int j = max(0, wins - 2); j < wins; ++j) wait_drain(&szfull[j & 1], (uint32_t)(j >> 1) & 1u, status);
            wait_drain(xbar, 0, status);
        }
        __syncthreads();
        return;
    }

    if (wid == kCombiner) {
        // ================================ combiner ================================
        // The CTA's range splits a tile wherever it starts or ends inside one; walk those tiles in the
        // consumers' order.  Lane l handles rows 8l .. 8l + 7 of the tile.
        int pseg = 0;
        for (int64_t tt = beg / P; tt * P < end; ++tt) {
            if (tt * P >= beg && tt * P + P <= end) continue;  // whole tile: the consumers wrote y
            const int b = pseg & 1;
            const bool ok = __all_sync(0xffffffffu, mbar_wait(&pfull[b], (uint32_t)(pseg >> 1) & 1u, status, flags));
            if (!ok) break;
            const float4 v0 = *reinterpret_cast<const float4 *>(part + b * kTile + 8 * lane);
            const float4 v1 = *reinterpret_cast<const float4 *>(part + b * kTile + 8 * lane + 4);
            __syncwarp();
            if (lane == 0) mbar_arrive(&pempty[b]);  // the shared tile is in registers: free it
            ++pseg;
            const int64_t c_first = cta_of(tt * P, units, B);
            const int nseg = (int)(cta_of(tt * P + P - 1, units, B) - c_first) + 1;
            float *slots = ws + (size_t)tt * max_segs * kTile;
            float4 *mine = reinterpret_cast<float4 *>(slots + (bid - c_first) * kTile + 8 * lane);
            mine[0] = v0;
            mine[1] = v1;
            // the release of the add below covers every lane's slot writes (ordered by the warp barrier)
            __syncwarp();
            int last = 0;
            if (lane == 0) last = (atom_add_acq_rel(cnt + tt, 1) + 1 == nseg) ? 1 : 0;
            last = __shfl_sync(0xffffffffu, last, 0);
            if (last) {
                // sum the segments' slots in segment order (independent of which CTA arrived last)
                float v[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
                const float4 *q = reinterpret_cast<const float4 *>(slots + 8 * lane);
                int o = 0;
                for (; o + 4 <= nseg; o += 4) {
                    float4 a[8];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        a[2 * j] = __ldcg(q + (size_t)(o + j) * (kTile / 4));
                        a[2 * j + 1] = __ldcg(q + (size_t)(o + j) * (kTile / 4) + 1);
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        v[0] += a[2 * j].x; v[1] += a[2 * j].y; v[2] += a[2 * j].z; v[3] += a[2 * j].w;
                        v[4] += a[2 * j + 1].x; v[5] += a[2 * j + 1].y; v[6] += a[2 * j + 1].z; v[7] += a[2 * j + 1].w;
                    }
                }
                for (; o < nseg; ++o) {
                    const float4 a0 = __ldcg(q + (size_t)o * (kTile / 4)), a1 = __ldcg(q + (size_t)o * (kTile / 4) + 1);
                    v[0] += a0.x; v[1] += a0.y; v[2] += a0.z; v[3] += a0.w;
                    v[4] += a1.x; v[5] += a1.y; v[6] += a1.z; v[7] += a1.w;
                }
                const int64_t row = tt * kTile + 8 * lane;
                if (row + 8 <= N) {
                    uint4 pk;
                    pk.x = (uint32_t)f32_to_bf16(v[0]) | ((uint32_t)f32_to_bf16(v[1]) << 16);
                    pk.y = (uint32_t)f32_to_bf16(v[2]) | ((uint32_t)f32_to_bf16(v[3]) << 16);
                    pk.z = (uint32_t)f32_to_bf16(v[4]) | ((uint32_t)f32_to_bf16(v[5]) << 16);
                    pk.w = (uint32_t)f32_to_bf16(v[6]) | ((uint32_t)f32_to_bf16(v[7]) << 16);
                    *reinterpret_cast<uint4 *>(y + row) = pk;
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        if (row + j < N) y[row + j] = f32_to_bf16(v[j]);
                }
                __syncwarp();
                if (lane == 0) atomicExch(cnt + tt, 0);
            }
        }
        __syncthreads();
        return;
    }

    // ================================ consumers ================================
    if (n > 0) {
        // ---- x: wait for the bulk copy, permute each chunk in place (chunks that were not copied hold
        // stale bytes and are never read) ----
        mbar_wait(xbar, 0, status, flags);
        for (int c = tid; c < K / 8; c += kC * 32) {
            {
                uint4 v = xp[c];
                if (col_scale) v = colscale8(v, col_scale + 8 * c);
                uint4 pr;
                pr.x = __byte_perm(v.x, v.z, 0x5410);  // (x0, x4)
                pr.y = __byte_perm(v.x, v.z, 0x7632);  // (x1, x5)
                pr.z = __byte_perm(v.y, v.w, 0x5410);  // (x2, x6)
                pr.w = __byte_perm(v.y, v.w, 0x7632);  // (x3, x7)
                xp[c] = pr;
            }
        }
        named_bar_sync(1, kC * 32);

        const int gq = lane >> 2, tq = lane & 3;
        const uint32_t ring_u32 = smem_u32(ring), szr_u32 = smem_u32(szr), xp_u32 = smem_u32(xp);
        const int r0 = 16 * wid + gq;  // this lane's rows in the tile: r0 and r0 + 8
        float acc[2] = {0.0f, 0.0f};
        int t = tile0, p = pair0, seg_first = pair0;
        int win = -1;
        int pseg = 0;  // partial segments handed to the combiner
        int s = 0;     // stage slot of unit i, and the parity of its fill
        uint32_t ph = 0, w_off = 0;
        const uint32_t w_lane = ring_u32 + (uint32_t)r0 * 64u + (uint32_t)tq * 16u;
        const uint32_t sz_lane = szr_u32 + (uint32_t)r0 * 16u;
        const uint32_t x_lane = xp_u32 + (uint32_t)tq * 64u;
        // A wait that runs out sets the abort flag and every later wait returns at once: the loop then runs
        // to its end on garbage, with the same control flow in every warp, so the barriers below still meet.
        for (int i = 0; i < n; ++i) {
            // ---- s/z window ----
            if (i == 0 || (p & (kPairsPerWindow - 1)) == 0) {
                if (win >= 0) {  // the previous window is consumed
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&szempty[win & 1]);
                }
                ++win;
                mbar_wait(&szfull[win & 1], (uint32_t)(win >> 1) & 1u, status, flags);
            }
            mbar_wait(&full[s], ph, status, flags);
            // ---- loads from the stage: rows r0, r0 + 8 of both groups; their s, z ----
            const uint32_t wsrc = w_lane + w_off;
            uint4 wv[2][2];  // [group h][row r0, row r0 + 8]
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int a = 0; a < 2; ++a) wv[h][a] = lds128(wsrc + (uint32_t)h * (kTile * 64u) + (uint32_t)a * 8u * 64u);
            const int kg = 2 * p;
            const uint32_t szsrc = sz_lane + (uint32_t)(win & 1) * 2u * kSzBytes + (uint32_t)(kg & 7) * 2u;
            // s and z of groups kg, kg + 1 are adjacent in the window box (kg is even): one 32-bit load per
            // row and array; (128 + z) is formed by one bf16 addition, exact when z is in [0, 15]
            float sv[2][2];
            uint32_t zz[2][2];  // bf16 pairs (128 + z, 128 + z)
            uint32_t zraw[2], zin = 0u;  // zin & 0xFFF0FFF0: some z of this lane outside [0, 15]
#pragma unroll
            for (int a = 0; a < 2; ++a) {
                const uint32_t o = szsrc + (uint32_t)a * 8u * 16u;
                zraw[a] = lds_u32(o + kSzBytes);
                const uint32_t s2 = lds_u32(o), z2 = add_bf16x2(zraw[a], 0x43004300u);
                sv[0][a] = __uint_as_float(s2 << 16);
                sv[1][a] = __uint_as_float(s2 & 0xffff0000u);
                zz[0][a] = __byte_perm(z2, 0u, 0x1010);
                zz[1][a] = __byte_perm(z2, 0u, 0x3232);
                zin |= z2 ^ 0x43004300u;
            }
            // a zero-point of this lane outside [0, 15] (rare): split it (zp_split) and add -s z_hi times the
            // group's activation sum (all 128 values, in a fixed order) to the row sums right away
            if ((zin & 0xFFF0FFF0u) != 0u) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float xs = 0.0f;
                    for (int j = 0; j < 16; ++j) xs += sum_bf16x8(lds128(xp_u32 + (uint32_t)(kg + h) * 256u + (uint32_t)j * 16u));
#pragma unroll
                    for (int a = 0; a < 2; ++a) {
                        const float zf = __uint_as_float(h ? (zraw[a] & 0xffff0000u) : (zraw[a] << 16));
                        float zh;
                        zz[h][a] = bf16_pair_128_plus(zp_split(zf, zh));
                        acc[a] = fmaf(-sv[h][a] * zh, xs, acc[a]);
                    }
                }
            }
            // the stage's weight bytes are in registers: hand the slot back to the producer
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            if (++s == kStages) { s = 0; ph ^= 1u; w_off = 0; } else { w_off += kStageBytes; }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint4 Pw[4];
#pragma unroll
                for (int w = 0; w < 4; ++w) Pw[w] = lds128(x_lane + (uint32_t)(kg + h) * 256u + (uint32_t)w * 16u);
                float C0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, C1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const uint32_t va = word_of(wv[h][0], w), vb = word_of(wv[h][1], w);
                    float *C = (w & 1) ? C1 : C0;
                    const uint32_t za = zz[h][0], zb = zz[h][1];
                    mma_bf16(C, sub_bf16x2(nib_pair(va, 0, nib_mask, bf16_magic), za),
                             sub_bf16x2(nib_pair(vb, 0, nib_mask, bf16_magic), zb),
                             sub_bf16x2(nib_pair(va, 4, nib_mask, bf16_magic), za),
                             sub_bf16x2(nib_pair(vb, 4, nib_mask, bf16_magic), zb), Pw[w].x, Pw[w].y);
                    mma_bf16(C, sub_bf16x2(nib_pair(va, 8, nib_mask, bf16_magic), za),
                             sub_bf16x2(nib_pair(vb, 8, nib_mask, bf16_magic), zb),
                             sub_bf16x2(nib_pair(va, 12, nib_mask, bf16_magic), za),
                             sub_bf16x2(nib_pair(vb, 12, nib_mask, bf16_magic), zb), Pw[w].z, Pw[w].w);
                }
                // every column of D carries the same x: C[0] is row r0, C[2] row r0 + 8
                acc[0] = fmaf(sv[h][0], C0[0] + C1[0], acc[0]);
                acc[1] = fmaf(sv[h][1], C0[2] + C1[2], acc[1]);
            }
            // ---- end of a segment: the tile's last pair, or the end of this CTA's range ----
            const bool tile_done = (p + 1 == P);
            if (tile_done || i + 1 == n) {
                const int row0 = t * kTile + r0;
                if (seg_first == 0 && tile_done) {
                    if (tq == 0) {
                        if (row0 < N) y[row0] = f32_to_bf16(acc[0]);
                        if (row0 + 8 < N) y[row0 + 8] = f32_to_bf16(acc[1]);
                    }
                } else {
                    // partial: this warp's 16 row sums go to the shared tile of this segment; the combiner
                    // warp takes it from there (tiles alternate between two buffers)
                    const int b = pseg & 1;
                    if (pseg >= 2) mbar_wait(&pempty[b], (uint32_t)((pseg >> 1) - 1) & 1u, status, flags);
                    if (tq == 0) {
                        part[b * kTile + r0] = acc[0];
                        part[b * kTile + r0 + 8] = acc[1];
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&pfull[b]);
                    ++pseg;
                }
                acc[0] = acc[1] = 0.0f;
            }
            if (++p == P) { p = 0; ++t; seg_first = 0; }
        }
    }
    __syncthreads();
}

// Grid of the persistent kernel for this shape on the current device: one CTA per SM, fewer when there
// is less work.  Cached per device.
int m1_grid(int64_t N, int64_t K)
{
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
            cudaFuncSetAttribute(gemv_w4a16_m1_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
            it = sms_of.emplace(dev, v).first;
        }
        sms = it->second;
    }
    const int64_t units = ((N + kTile - 1) / kTile) * (K / 256);
    return (int)std::max<int64_t>(1, std::min<int64_t>(units, sms));
}

// Most segments (CTAs) any tile is split into, for this grid.
int m1_max_segments(int64_t N, int64_t K, int grid)
{
    const int64_t P = K / 256;
    const int64_t units = ((N + kTile - 1) / kTile) * P;
    const int64_t per = units / std::min<int64_t>(grid, units);  // >= 1 unit per CTA
    return (int)std::min<int64_t>((P + per - 1) / per + 1, P);
}

size_t m1_slots_bytes(int64_t N, int64_t K, int grid)
{
    const int64_t ntiles = (N + kTile - 1) / kTile;
    return ((size_t)ntiles * m1_max_segments(N, K, grid) * kTile * 4 + 255) / 256 * 256;
}

}  // namespace

bool gemv_m1_eligible(int64_t M, int64_t N, int64_t K, int g)
{
    // K % 1024: the s/z row stride (K / 128 bf16) must be a multiple of 16 bytes for their tensor maps;
    // K <= 32768: x and the stages fit in shared memory
    return M == 1 && g == 128 && K >= 1024 && K % 1024 == 0 && K <= 32768 && N >= 1 && N <= 0x7fffffffLL;
}

size_t gemv_m1_workspace_bytes(int64_t M, int64_t N, int64_t K, int g)
{
    if (!gemv_m1_eligible(M, N, K, g)) return 0;
    const int64_t ntiles = (N + kTile - 1) / kTile;
    return m1_slots_bytes(N, K, m1_grid(N, K)) + ((size_t)ntiles * 4 + 255) / 256 * 256;
}

int launch_gemv_w4a16_m1(const uint16_t *x, int64_t N, int64_t K, const uint8_t *q, const uint16_t *s,
                         const uint16_t *z, uint16_t *y, void *workspace, int *status, cudaStream_t st,
                         const float *col_scale)
{
    // packed codes seen as (64-byte group slice, row, group): strides K/2 bytes (row) and 64 bytes (group)
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qr) != cudaSuccess ||
            qr != cudaDriverEntryPointSuccess || fn == nullptr)
            return -1;
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    CUtensorMap wmap, smap, zmap;
    const uint64_t G = (uint64_t)K / 128;
    cuuint64_t dims[3] = {64, (cuuint64_t)N, G};
    cuuint64_t strides[2] = {(cuuint64_t)K / 2, 64};
    cuuint32_t box[3] = {64, (cuuint32_t)kTile, 2};
    cuuint32_t estr[3] = {1, 1, 1};
    if (encode(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t *>(q), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return -1;
    if (!encode_tmap_2d(&smap, CU_TENSOR_MAP_DATA_TYPE_UINT16, s, G, (uint64_t)N, G * 2, 8, kTile,
                        CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_tmap_2d(&zmap, CU_TENSOR_MAP_DATA_TYPE_UINT16, z, G, (uint64_t)N, G * 2, 8, kTile,
                        CU_TENSOR_MAP_SWIZZLE_NONE))
        return -1;
    const int grid = m1_grid(N, K);
    const int max_segs = m1_max_segments(N, K, grid);
    uint8_t *w8 = static_cast<uint8_t *>(workspace);
    float *ws = reinterpret_cast<float *>(w8);
    int *cnt = reinterpret_cast<int *>(w8 + m1_slots_bytes(N, K, grid));
    // programmatic dependent launch: this grid may start while the previous kernel in the stream finishes;
    // the kernel reads nothing that kernel may write, and writes nothing, before griddepcontrol.wait
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kT);
    cfg.dynamicSmemBytes = m1_smem_bytes(K);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, gemv_w4a16_m1_kernel, wmap, smap, zmap, x, (int)N, (int)K, y, ws, cnt, max_segs,
                           status, 0x000F000Fu, 0x43004300u, col_scale) != cudaSuccess)
        return -2;
    return 0;
}

}  // namespace wq

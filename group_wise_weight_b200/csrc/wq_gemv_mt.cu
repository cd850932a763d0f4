// wq_gemv_mt.cu -- W4A16, group 128, 2 <= M <= 16 activation rows: the decode
// step at small batch, still bound by streaming the packed weights from HBM.
//
// "Quantization Methods Compared: INT8, GPTQ, AWQ, FP8, FP4 and KV-Cache
// Quantization", section "Hardware, formats and the roofline": up to a batch
// of a few dozen rows a decode step reads every weight once and the 4-bit
// kernel stays memory-bound, so one pass over the weights serves all M rows.
// w_hat = s (q - z) ("Quantization for LLM inference: FP8, INT4 (GPTQ, AWQ)
// and GGUF", "The minimum maths").
//
// The weight stream is the one of the M = 1 kernel (wq_gemv_m1.cu): a
// persistent grid, one CTA per SM, 16 consumer warps, a TMA producer warp
// moving 32 KB stages of 256 rows x 2 groups through a 3-D view of the codes,
// s/z windows of 8 groups, stream-K over (256-row tile, group pair) units,
// split tiles combined in segment order by a combiner warp, programmatic
// dependent launch.  What differs is the activation operand: the M rows fill
// the 8 (NT = 1) or 16 (NT = 2) columns of mma.sync m16n8k16, so there is no
// room for the integer digit planes of the M = 1 kernel, and the codes enter
// as exact bf16 integers instead:
//  * a 32-bit word of codes c_0 .. c_7 yields the bf16 pairs (128 + c_i,
//    128 + c_{i+4}), i = 0 .. 3, one shift and one LOP3 each; subtracting the
//    pair (128 + z, 128 + z) leaves the exact q - z, so the tensor core sums
//    x (q - z) per group and s multiplies the binary32 result;
//  * the k order inside a step is permuted to match, and x is staged once per
//    CTA in shared memory as the matching pairs (x_i, x_{i+4}), only for the
//    group pairs the CTA's units touch;
//  * a zero-point outside [0, 15] is split (zp_split in wq_common.cuh): the
//    operand holds q - z_lo and -s z_hi times the group's activation sum is
//    added in binary32.
#include <algorithm>
#include <map>
#include <mutex>

#include "wq_common.cuh"
#include "wq_internal.h"
#include "wq_sm100.cuh"

namespace wq {

namespace {

constexpr int kC = 16;                         // consumer warps
constexpr int kProducer = kC;                  // warp roles: consumers 0 .. kC-1, then these two
constexpr int kCombiner = kC + 1;
constexpr int kT = (kC + 2) * 32;              // threads
constexpr int kTile = 16 * kC;                 // rows per tile (256)
constexpr int kMaxStages = 3;
constexpr uint32_t kStageBytes = kTile * 128;  // 256 rows x 2 groups x 64 B
constexpr uint32_t kSzBytes = kTile * 16;      // 256 rows x 8 groups x 2 B (one of s or z)
constexpr int kPairsPerWindow = 4;             // 8 groups of s/z = 4 units

// shared memory: [stages][s/z windows][2 partial tiles of M x 256][x pairs][barriers]
struct MtLayout {
    size_t sz, part, xs, bar, total;
    __host__ __device__ MtLayout(int stages, int M, int npairs)
    {
        sz = (size_t)stages * kStageBytes;
        part = sz + 2 * 2 * kSzBytes;
        xs = part + (size_t)2 * M * kTile * 4;
        bar = xs + (size_t)npairs * 2 * M * 256;  // per pair, group and row: 128 bf16
        total = bar + (2 * kMaxStages + 4 + 4 + 2) * 8 + 1024;
    }
};

__device__ __forceinline__ uint32_t nib_pair(uint32_t v, int sh)
{
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(v >> sh), "r"(0x000F000Fu), "r"(0x43004300u));
    return d;
}

__device__ __forceinline__ void mma_bf16(float c[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar, int x, int y, int z)
{
    asm volatile("cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];"
                 :: "r"(smem_u32(dst)), "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
                 : "memory");
}

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

__device__ __forceinline__ int atom_add_acq_rel(int *p, int v)
{
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

__host__ __device__ __forceinline__ int cta_of(int64_t u, int64_t units, int64_t B)
{
    return (int)(((u + 1) * B - 1) / units);
}

__device__ __forceinline__ void wait_drain(uint64_t *bar, uint32_t parity, int *status)
{
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_ns() - t0 > kWaitLimitNs) { record_timeout(status); return; }
}

// 18 warps put five on one SM sub-partition, whose register file holds 16K registers: at most 96 each.
template <int NT, int STAGES>
__global__ void __maxnreg__(96)
gemv_w4a16_mt_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap smap,
                     const __grid_constant__ CUtensorMap zmap, const uint16_t *__restrict__ x, int M, int N, int K,
                     uint16_t *__restrict__ y, float *__restrict__ ws, int *__restrict__ cnt, int max_segs,
                     int *__restrict__ status, int npairs)
{
    extern __shared__ __align__(1024) uint8_t mt_raw[];
    uint8_t *sm = mt_raw + ((1024u - (smem_u32(mt_raw) & 1023u)) & 1023u);
    const MtLayout L(STAGES, M, npairs);
    uint8_t *ring = sm;
    uint8_t *szr = sm + L.sz;                                  // [2 windows][s, z][256 rows][8 groups]
    float *part = reinterpret_cast<float *>(sm + L.part);      // [2][M][256 rows] partial sums
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L.bar);
    uint64_t *full = bars, *empty = bars + kMaxStages;
    uint64_t *szfull = bars + 2 * kMaxStages, *szempty = szfull + 2;
    uint64_t *pfull = szempty + 2, *pempty = pfull + 2;
    volatile int *flags = reinterpret_cast<volatile int *>(pempty + 2);  // [0] abort
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int G = K >> 7;
    const int P = G >> 1;  // group pairs (units) per tile

    pdl_launch_dependents();
    if (tid == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kC);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&szfull[i], 1);
            mbar_init(&szempty[i], kC);
            mbar_init(&pfull[i], kC);
            mbar_init(&pempty[i], 1);
        }
        flags[0] = 0;
        flags[1] = 0;
        fence_mbar_init();
    }
    __syncthreads();

    const int ntiles = (N + kTile - 1) / kTile;
    const int64_t units = (int64_t)ntiles * P;
    const int64_t B = min((int64_t)gridDim.x, units);
    const int64_t bid = blockIdx.x;
    const int64_t beg = bid < B ? units * bid / B : units, end = bid < B ? units * (bid + 1) / B : units;
    const int n = (int)(end - beg);
    const int tile0 = (int)(beg / P), pair0 = (int)(beg - (int64_t)tile0 * P);

    // The weights, scales and zero-points are inputs the preceding call does not write: the first stages and
    // s/z window are requested before the grid-dependency wait; x waits.
    int pt = tile0, pp = pair0;
    int wins = 0, pi = 0;
    auto issue_window = [&](int slot) {
        mbar_arrive_expect_tx(&szfull[slot], 2 * kSzBytes);
        uint8_t *d = szr + (uint32_t)slot * 2u * kSzBytes;
        const int g8 = (2 * pp) & ~7;
        tma_load_2d(d, &smap, &szfull[slot], g8, pt * kTile);
        tma_load_2d(d + kSzBytes, &zmap, &szfull[slot], g8, pt * kTile);
        ++wins;
    };
    if (wid == kProducer && lane == 0) {
        // at most two windows start within the first STAGES pairs
        for (; pi < STAGES && pi < n; ++pi) {
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
            int i = pi;
            for (; i < n; ++i) {
                if ((pp & (kPairsPerWindow - 1)) == 0) {
                    const int slot = wins & 1;
                    if (wins >= 2 && !mbar_wait(&szempty[slot], (uint32_t)((wins >> 1) - 1) & 1u, status, flags)) break;
                    issue_window(slot);
                }
                const int s = i % STAGES;
                if (!mbar_wait(&empty[s], (uint32_t)(i / STAGES - 1) & 1u, status, flags)) break;
                mbar_arrive_expect_tx(&full[s], kStageBytes);
                tma_load_3d(ring + (uint32_t)s * kStageBytes, &wmap, &full[s], 0, pt * kTile, 2 * pp);
                if (++pp == P) { pp = 0; ++pt; }
            }
            for (int j = max(0, i - STAGES); j < i; ++j) wait_drain(&full[j % STAGES], (uint32_t)(j / STAGES) & 1u, status);
            for (int j = max(0, wins - 2); j < wins; ++j) wait_drain(&szfull[j & 1], (uint32_t)(j >> 1) & 1u, status);
        }
        __syncthreads();
        return;
    }

    if (wid == kCombiner) {
        // ================================ combiner ================================
        // Split tiles in the consumers' order.  Lane l handles rows 8l .. 8l + 7 of the tile, for every m.
        int pseg = 0;
        for (int64_t tt = beg / P; tt * P < end; ++tt) {
            if (tt * P >= beg && tt * P + P <= end) continue;  // whole tile: the consumers wrote y
            const int b = pseg & 1;
            const bool ok = __all_sync(0xffffffffu, mbar_wait(&pfull[b], (uint32_t)(pseg >> 1) & 1u, status, flags));
            if (!ok) break;
            const int c_first = cta_of(tt * P, units, B);
            const int nseg = cta_of(tt * P + P - 1, units, B) - c_first + 1;
            float *slots = ws + (size_t)tt * max_segs * M * kTile;  // [segment][m][256]
            float *mine = slots + (size_t)(bid - c_first) * M * kTile + 8 * lane;
            const float *src = part + (size_t)b * M * kTile + 8 * lane;
            for (int m = 0; m < M; ++m) {
                const float4 v0 = *reinterpret_cast<const float4 *>(src + m * kTile);
                const float4 v1 = *reinterpret_cast<const float4 *>(src + m * kTile + 4);
                reinterpret_cast<float4 *>(mine + m * kTile)[0] = v0;
                reinterpret_cast<float4 *>(mine + m * kTile)[1] = v1;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&pempty[b]);  // the shared tile is copied out: free it
            ++pseg;
            int last = 0;
            if (lane == 0) last = (atom_add_acq_rel(cnt + tt, 1) + 1 == nseg) ? 1 : 0;
            last = __shfl_sync(0xffffffffu, last, 0);
            if (last) {
                // sum the segments' slots in segment order (independent of which CTA arrived last)
                const int64_t row = tt * kTile + 8 * lane;
                const size_t sstride = (size_t)M * (kTile / 4);  // float4 between segments
                for (int m = 0; m < M; ++m) {
                    float v[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
                    const float4 *q = reinterpret_cast<const float4 *>(slots + (size_t)m * kTile + 8 * lane);
                    // segments 4 at a time: the loads of a batch are in flight together
                    int o = 0;
                    for (; o + 4 <= nseg; o += 4) {
                        float4 a[8];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            a[2 * j] = __ldcg(q + (size_t)(o + j) * sstride);
                            a[2 * j + 1] = __ldcg(q + (size_t)(o + j) * sstride + 1);
                        }
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            v[0] += a[2 * j].x; v[1] += a[2 * j].y; v[2] += a[2 * j].z; v[3] += a[2 * j].w;
                            v[4] += a[2 * j + 1].x; v[5] += a[2 * j + 1].y; v[6] += a[2 * j + 1].z; v[7] += a[2 * j + 1].w;
                        }
                    }
                    {
                        float4 a[6];
                        const int rem = nseg - o;  // 0 .. 3
#pragma unroll
                        for (int j = 0; j < 3; ++j)
                            if (j < rem) {
                                a[2 * j] = __ldcg(q + (size_t)(o + j) * sstride);
                                a[2 * j + 1] = __ldcg(q + (size_t)(o + j) * sstride + 1);
                            }
#pragma unroll
                        for (int j = 0; j < 3; ++j)
                            if (j < rem) {
                                v[0] += a[2 * j].x; v[1] += a[2 * j].y; v[2] += a[2 * j].z; v[3] += a[2 * j].w;
                                v[4] += a[2 * j + 1].x; v[5] += a[2 * j + 1].y; v[6] += a[2 * j + 1].z; v[7] += a[2 * j + 1].w;
                            }
                    }
                    uint16_t *yr = y + (size_t)m * N;
                    if (row + 8 <= N) {
                        uint4 pk;
                        pk.x = (uint32_t)f32_to_bf16(v[0]) | ((uint32_t)f32_to_bf16(v[1]) << 16);
                        pk.y = (uint32_t)f32_to_bf16(v[2]) | ((uint32_t)f32_to_bf16(v[3]) << 16);
                        pk.z = (uint32_t)f32_to_bf16(v[4]) | ((uint32_t)f32_to_bf16(v[5]) << 16);
                        pk.w = (uint32_t)f32_to_bf16(v[6]) | ((uint32_t)f32_to_bf16(v[7]) << 16);
                        if ((N & 7) == 0) {
                            *reinterpret_cast<uint4 *>(yr + row) = pk;
                        } else {
                            const uint32_t w4[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                yr[row + 2 * j] = (uint16_t)(w4[j] & 0xffffu);
                                yr[row + 2 * j + 1] = (uint16_t)(w4[j] >> 16);
                            }
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            if (row + j < N) yr[row + j] = f32_to_bf16(v[j]);
                    }
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
        const uint32_t xs_u32 = smem_u32(sm + L.xs);
        // ---- x of the group pairs this CTA touches, pair (pair0 + j) mod P in slot j: for slot j, group h
        // and row m, 16 chunks of 8 activations each permuted to the pairs (x0, x4), (x1, x5), (x2, x6),
        // (x3, x7).  Chunk u is stored at u ^ (2 ((u >> 3) & 1) + (m & 1)): the 8 lanes of a shared-memory
        // phase (rows 2j, 2j + 1, quads tq = 0 .. 3, chunk 4 tq + w) then read 8 different bank groups ----
        const int nslots = min(n, P);
        const int nchunks = nslots * 2 * M * 16;
        for (int c0 = tid; c0 < nchunks; c0 += 4 * kC * 32) {
            uint4 v[4];
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int c = c0 + b * kC * 32;
                if (c < nchunks) {
                    const int u = c & 15, m = (c >> 4) % M, jh = (c >> 4) / M, js = jh >> 1, h = jh & 1;
                    int pj = pair0 + js;
                    if (pj >= P) pj -= P;
                    v[b] = *reinterpret_cast<const uint4 *>(x + (size_t)m * K + (size_t)(2 * pj + h) * 128 + 8 * u);
                }
            }
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int c = c0 + b * kC * 32;
                if (c < nchunks) {
                    uint4 pr;
                    pr.x = __byte_perm(v[b].x, v[b].z, 0x5410);  // (x0, x4)
                    pr.y = __byte_perm(v[b].x, v[b].z, 0x7632);  // (x1, x5)
                    pr.z = __byte_perm(v[b].y, v[b].w, 0x5410);  // (x2, x6)
                    pr.w = __byte_perm(v[b].y, v[b].w, 0x7632);  // (x3, x7)
                    const int u = c & 15, m = (c >> 4) % M;
                    const uint32_t phys = (uint32_t)((c & ~15) | (u ^ ((((u >> 3) & 1) << 1) | (m & 1))));
                    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(xs_u32 + phys * 16u),
                                 "r"(pr.x), "r"(pr.y), "r"(pr.z), "r"(pr.w)
                                 : "memory");
                }
            }
        }
        named_bar_sync(1, kC * 32);

        const int gq = lane >> 2, tq = lane & 3;
        const uint32_t ring_u32 = smem_u32(ring), szr_u32 = smem_u32(szr);
        const int r0 = 16 * wid + gq;  // this lane's weight rows in the tile: r0 and r0 + 8
        // B operand: activation row m = 8 nt + gq (zero when m >= M); its 32 values of a group at lane tq
        bool bok[NT];
        uint32_t b_lane[NT], b_sw[NT];  // row base + 64 tq, and the chunk swizzle of (row, tq)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int m = 8 * nt + gq;
            bok[nt] = m < M;
            b_lane[nt] = xs_u32 + (uint32_t)((bok[nt] ? m : 0) * 256 + tq * 64);
            b_sw[nt] = (uint32_t)((((tq >> 1) & 1) << 1) | (m & 1));
        }
        float acc[2][NT][2];  // [row r0, r0 + 8][tile nt][activation row 8 nt + 2 tq + e]
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) acc[a][nt][0] = acc[a][nt][1] = 0.0f;
        int t = tile0, p = pair0, seg_first = pair0;
        int win = -1, pseg = 0, s = 0, di = 0;
        uint32_t ph = 0, w_off = 0;
        const uint32_t w_lane = ring_u32 + (uint32_t)r0 * 64u + (uint32_t)tq * 16u;
        const uint32_t sz_lane = szr_u32 + (uint32_t)r0 * 16u;
        const uint32_t xrow = (uint32_t)M * 256u;  // bytes per (slot, group)
        for (int i = 0; i < n; ++i) {
            if (i == 0 || (p & (kPairsPerWindow - 1)) == 0) {
                if (win >= 0) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&szempty[win & 1]);
                }
                ++win;
                mbar_wait(&szfull[win & 1], (uint32_t)(win >> 1) & 1u, status, flags);
            }
            mbar_wait(&full[s], ph, status, flags);
            const uint32_t wsrc = w_lane + w_off;
            uint4 wv[2][2];  // [group h][row r0, row r0 + 8]
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int a = 0; a < 2; ++a) wv[h][a] = lds128(wsrc + (uint32_t)h * (kTile * 64u) + (uint32_t)a * 8u * 64u);
            const int kg = 2 * p;
            const uint32_t szsrc = sz_lane + (uint32_t)(win & 1) * 2u * kSzBytes + (uint32_t)(kg & 7) * 2u;
            float sv[2][2];
            uint32_t zz[2][2];           // bf16 pairs (128 + z, 128 + z)
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
            const uint32_t xslot = (uint32_t)di * 2u * xrow;
            // a zero-point outside [0, 15] (rare): split it and add -s z_hi times the group's activation sums of
            // this lane's columns (rows 8 nt + 2 tq + e, all 128 values, in a fixed order)
            if ((zin & 0xFFF0FFF0u) != 0u) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float xsum[NT][2];
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int m = 8 * nt + 2 * tq + e;
                            float v = 0.0f;
                            if (m < M)
                                for (int j = 0; j < 16; ++j) {
                                    const uint32_t pj = (uint32_t)(j ^ ((((j >> 3) & 1) << 1) | (m & 1)));
                                    v += sum_bf16x8(lds128(xs_u32 + xslot + (uint32_t)h * xrow + (uint32_t)m * 256u + pj * 16u));
                                }
                            xsum[nt][e] = v;
                        }
#pragma unroll
                    for (int a = 0; a < 2; ++a) {
                        const float zf = __uint_as_float(h ? (zraw[a] & 0xffff0000u) : (zraw[a] << 16));
                        float zh;
                        zz[h][a] = bf16_pair_128_plus(zp_split(zf, zh));
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                            for (int e = 0; e < 2; ++e) acc[a][nt][e] = fmaf(-sv[h][a] * zh, xsum[nt][e], acc[a][nt][e]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            if (++s == STAGES) { s = 0; ph ^= 1u; w_off = 0; } else { w_off += kStageBytes; }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint4 Pw[NT][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        Pw[nt][w] = bok[nt] ? lds128(b_lane[nt] + xslot + (uint32_t)h * xrow + ((uint32_t)w ^ b_sw[nt]) * 16u)
                                            : make_uint4(0u, 0u, 0u, 0u);
                float C[NT][2][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) C[nt][0][e] = C[nt][1][e] = 0.0f;
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    // word w of rows r0, r0 + 8: the exact bf16 pairs q - z, formed once for all column tiles
                    uint32_t A[4][2];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        A[j][0] = sub_bf16x2(nib_pair(word_of(wv[h][0], w), 4 * j), zz[h][0]);
                        A[j][1] = sub_bf16x2(nib_pair(word_of(wv[h][1], w), 4 * j), zz[h][1]);
                    }
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        mma_bf16(C[nt][w & 1], A[0][0], A[0][1], A[1][0], A[1][1], Pw[nt][w].x, Pw[nt][w].y);
                        mma_bf16(C[nt][w & 1], A[2][0], A[2][1], A[3][0], A[3][1], Pw[nt][w].z, Pw[nt][w].w);
                    }
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    // D: (row r0, column 2 tq), (r0, 2 tq + 1), (r0 + 8, 2 tq), (r0 + 8, 2 tq + 1)
                    acc[0][nt][0] = fmaf(sv[h][0], C[nt][0][0] + C[nt][1][0], acc[0][nt][0]);
                    acc[0][nt][1] = fmaf(sv[h][0], C[nt][0][1] + C[nt][1][1], acc[0][nt][1]);
                    acc[1][nt][0] = fmaf(sv[h][1], C[nt][0][2] + C[nt][1][2], acc[1][nt][0]);
                    acc[1][nt][1] = fmaf(sv[h][1], C[nt][0][3] + C[nt][1][3], acc[1][nt][1]);
                }
            }
            if (++di == P) di = 0;
            // ---- end of a segment: the tile's last pair, or the end of this CTA's range ----
            const bool tile_done = (p + 1 == P);
            if (tile_done || i + 1 == n) {
                const int row0 = t * kTile + r0;
                if (seg_first == 0 && tile_done) {
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int m = 8 * nt + 2 * tq + e;
                            if (m < M) {
                                if (row0 < N) y[(size_t)m * N + row0] = f32_to_bf16(acc[0][nt][e]);
                                if (row0 + 8 < N) y[(size_t)m * N + row0 + 8] = f32_to_bf16(acc[1][nt][e]);
                            }
                        }
                } else {
                    // partial: this warp's 16 rows for every m go to the shared tile of this segment
                    const int b = pseg & 1;
                    if (pseg >= 2) mbar_wait(&pempty[b], (uint32_t)((pseg >> 1) - 1) & 1u, status, flags);
                    float *pb = part + (size_t)b * M * kTile;
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int m = 8 * nt + 2 * tq + e;
                            if (m < M) {
                                pb[m * kTile + r0] = acc[0][nt][e];
                                pb[m * kTile + r0 + 8] = acc[1][nt][e];
                            }
                        }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&pfull[b]);
                    ++pseg;
                }
#pragma unroll
                for (int a = 0; a < 2; ++a)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) acc[a][nt][0] = acc[a][nt][1] = 0.0f;
            }
            if (++p == P) { p = 0; ++t; seg_first = 0; }
        }
    }
    __syncthreads();
}

// Launch parameters per (device, M, N, K): grid (one CTA per SM, fewer when there is less work), the x slots a
// CTA needs, the stage count that fits shared memory (0: the shape does not fit).
struct MtConfig {
    int grid, npairs, stages;
    size_t smem;
};

MtConfig mt_config(int64_t M, int64_t N, int64_t K)
{
    static std::mutex mu;
    static std::map<int, std::pair<int, int>> dev_of;  // SMs, opt-in shared memory per block
    int dev = 0;
    cudaGetDevice(&dev);
    int sms, optin;
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = dev_of.find(dev);
        if (it == dev_of.end()) {
            // without a device (a workspace query on a build host) assume a B200: 148 SMs, 227 KB per block
            int v = 148, o = 232448;
            cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
            cudaDeviceGetAttribute(&o, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
            cudaGetLastError();
            cudaFuncSetAttribute(gemv_w4a16_mt_kernel<1, 3>, cudaFuncAttributeMaxDynamicSharedMemorySize, o);
            cudaFuncSetAttribute(gemv_w4a16_mt_kernel<1, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, o);
            cudaFuncSetAttribute(gemv_w4a16_mt_kernel<2, 3>, cudaFuncAttributeMaxDynamicSharedMemorySize, o);
            cudaFuncSetAttribute(gemv_w4a16_mt_kernel<2, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, o);
            it = dev_of.emplace(dev, std::make_pair(v, o)).first;
        }
        sms = it->second.first;
        optin = it->second.second;
    }
    const int64_t P = K / 256;
    const int64_t units = ((N + kTile - 1) / kTile) * P;
    MtConfig c;
    c.grid = (int)std::max<int64_t>(1, std::min<int64_t>(units, sms));
    const int64_t per = (units + c.grid - 1) / c.grid;
    c.npairs = (int)std::min<int64_t>(per, P);
    c.stages = MtLayout(3, (int)M, c.npairs).total <= (size_t)optin ? 3
               : MtLayout(2, (int)M, c.npairs).total <= (size_t)optin ? 2
                                                                       : 0;
    c.smem = c.stages ? MtLayout(c.stages, (int)M, c.npairs).total : 0;
    return c;
}

int mt_max_segments(int64_t N, int64_t K, int grid)
{
    const int64_t P = K / 256;
    const int64_t units = ((N + kTile - 1) / kTile) * P;
    const int64_t per = units / std::min<int64_t>(grid, units);
    return (int)std::min<int64_t>((P + per - 1) / per + 1, P);
}

size_t mt_slots_bytes(int64_t M, int64_t N, int64_t K, int grid)
{
    const int64_t ntiles = (N + kTile - 1) / kTile;
    return ((size_t)ntiles * mt_max_segments(N, K, grid) * M * kTile * 4 + 255) / 256 * 256;
}

}  // namespace

bool gemv_mt_eligible(int64_t M, int64_t N, int64_t K, int g)
{
    // K % 1024: the s/z row stride must be a multiple of 16 bytes for their tensor maps; the CTA's x pairs
    // and at least two stages must fit shared memory
    if (!(g == 128 && M >= 2 && M <= 16 && K >= 1024 && K % 1024 == 0 && K <= 32768 && N >= 1 && N <= 0x7fffffffLL))
        return false;
    return mt_config(M, N, K).stages != 0;
}

int gemv_mt_stages(int64_t M, int64_t N, int64_t K, int g)
{
    return gemv_mt_eligible(M, N, K, g) ? mt_config(M, N, K).stages : 0;
}

size_t gemv_mt_workspace_bytes(int64_t M, int64_t N, int64_t K, int g)
{
    if (!gemv_mt_eligible(M, N, K, g)) return 0;
    const int64_t ntiles = (N + kTile - 1) / kTile;
    return counter_region_bytes(ntiles) + mt_slots_bytes(M, N, K, mt_config(M, N, K).grid);
}

int launch_gemv_w4a16_mt(const uint16_t *x, int64_t M, int64_t N, int64_t K, const uint8_t *q, const uint16_t *s,
                         const uint16_t *z, uint16_t *y, void *workspace, int *status, cudaStream_t st)
{
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
    const MtConfig c = mt_config(M, N, K);
    const int max_segs = mt_max_segments(N, K, c.grid);
    const int64_t ntiles = (N + kTile - 1) / kTile;
    uint8_t *w8 = static_cast<uint8_t *>(workspace);
    int *cnt = reinterpret_cast<int *>(w8);
    float *ws = reinterpret_cast<float *>(w8 + counter_region_bytes(ntiles));
    if (clear_extra_counters(workspace, ntiles, st) != cudaSuccess) return -2;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)c.grid);
    cfg.blockDim = dim3(kT);
    cfg.dynamicSmemBytes = c.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const int Mi = (int)M, Ni = (int)N, Ki = (int)K;
    cudaError_t e;
    if (M <= 8)
        e = c.stages == 3 ? cudaLaunchKernelEx(&cfg, gemv_w4a16_mt_kernel<1, 3>, wmap, smap, zmap, x, Mi, Ni, Ki, y, ws,
                                               cnt, max_segs, status, c.npairs)
                          : cudaLaunchKernelEx(&cfg, gemv_w4a16_mt_kernel<1, 2>, wmap, smap, zmap, x, Mi, Ni, Ki, y, ws,
                                               cnt, max_segs, status, c.npairs);
    else
        e = c.stages == 3 ? cudaLaunchKernelEx(&cfg, gemv_w4a16_mt_kernel<2, 3>, wmap, smap, zmap, x, Mi, Ni, Ki, y, ws,
                                               cnt, max_segs, status, c.npairs)
                          : cudaLaunchKernelEx(&cfg, gemv_w4a16_mt_kernel<2, 2>, wmap, smap, zmap, x, Mi, Ni, Ki, y, ws,
                                               cnt, max_segs, status, c.npairs);
    return e == cudaSuccess ? 0 : -2;
}

}  // namespace wq

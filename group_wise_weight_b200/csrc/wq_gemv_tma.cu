// wq_gemv_tma.cu -- W4A16, group 128, M <= 16: the decode-regime matmul fed
// by a TMA pipeline (sm_100a).
//
// "Quantization Methods Compared: INT8, GPTQ, AWQ, FP8, FP4 and KV-Cache
// Quantization", section "Hardware, formats and the roofline": at decode
// batch sizes the step is bound by reading the weights once from HBM, and
// the 4-bit kernel dequantises inside the matmul.  Decode w_hat = s (q - z)
// ("Quantization for LLM inference: FP8, INT4 (GPTQ, AWQ) and GGUF", "The
// minimum maths").
//
// Structure (one CTA = 8 consumer warps + 1 producer warp, persistent):
//  * Work is the flattened sequence of (128-row tile, 128-k chunk) units; CTA
//    b takes an equal contiguous share of it (stream-K), so every shape
//    keeps all SMs streaming and no CTA idles behind a short last wave.
//  * The producer keeps kStages TMA loads of [128 rows x 64 bytes] weight
//    boxes in flight into a shared-memory ring (mbarrier full/empty pairs);
//    the consumers never wait on global-memory latency for weights.
//  * Consumer warp w owns rows 16w..16w+15 of the tile.  Each lane reads the
//    16 bytes of rows n and n+8 it needs (512 contiguous bytes per warp, no
//    bank conflicts), turns every code pair into bf16 128 + q with one LOP3
//    and subtracts the pair (128 + z, 128 + z), which leaves the exact
//    integers q - z, and issues mma.sync m16n8k16 with the weights as the
//    16-row operand and the activations as the 8-column operand.  A 32-bit
//    word of codes c_0 .. c_7 yields the bf16 pairs (c_i, c_{i+4}),
//    i = 0 .. 3, one shift and one LOP3 each, so the k order inside an MMA
//    step is permuted to put such a pair in each operand register; the
//    activations are staged in shared memory as the matching pairs
//    (x_i, x_{i+4}), and a dot product does not depend on the k order.
//  * Per chunk (= group) the binary32 accumulator takes s * C: (q - z) is
//    exact, s is applied in binary32, and no term carries an offset that
//    would have to cancel later (rows of zeros give exactly zero).  A warp
//    that meets a zero-point outside [0, 15] splits it (zp_split in
//    wq_common.cuh) and adds -z_hi times the group's activation sums, which
//    the lanes form from the activation operand they already hold.
//  * A tile split between CTAs is combined in a binary32 workspace with
//    atomics; the CTA whose contribution completes the tile's K range
//    converts it to bf16, re-zeroes the workspace and resets the tile's
//    counter, leaving the workspace ready for the next call.
//  * Every barrier wait is bounded (see mbar_wait); on a timeout the kernel
//    records it in the status word and winds down without hanging.
#include <algorithm>
#include <atomic>
#include <map>
#include <mutex>
#include <utility>

#include "wq_internal.h"
#include "wq_sm100.cuh"

namespace wq {

// cuTensorMapEncodeTiled from the driver, or nullptr.
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    // looked up once (host threads may race to fill it; they store the same pointer), retried on failure
    static std::atomic<PFN_cuTensorMapEncodeTiled_v12000> cached{nullptr};
    PFN_cuTensorMapEncodeTiled_v12000 fn = cached.load(std::memory_order_acquire);
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || p == nullptr)
            return nullptr;
        fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        cached.store(fn, std::memory_order_release);
    }
    return fn;
}

bool encode_tmap_2d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base, uint64_t inner, uint64_t outer,
                    uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle)
{
    const PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_stride_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(map, dtype, 2, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

namespace {

constexpr int kTileRows = 128;
constexpr int kChunkBytes = 64;  // 128 codes of one row = one group of 128
constexpr int kPair = 2;         // chunks per stage
constexpr int kStageRowBytes = kPair * kChunkBytes;
constexpr int kStageBytes = kTileRows * kStageRowBytes;
constexpr int kStages = 4;
constexpr int kConsumers = 8;
constexpr int kThreads = (kConsumers + 1) * 32;

struct SmemLayout {
    size_t bars, flags, xp, total;
};

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

__host__ __device__ inline SmemLayout smem_layout(int64_t M, int64_t K, bool xsmem)
{
    SmemLayout L;
    const int64_t G = K >> 7;
    L.bars = (size_t)kStages * kStageBytes;
    L.flags = L.bars + 2 * kStages * sizeof(uint64_t);
    L.xp = align_up(L.flags + 16, 16);
    // k-permuted activations of the M real rows, then one zero row (4 lanes x 4 words) for padding
    L.total = L.xp + (xsmem ? ((size_t)G * M * 16 + 16) * sizeof(uint4) : 0);
    return L;
}

__device__ __forceinline__ void pair_x(const uint4 xv, uint32_t P[4])
{
    P[0] = __byte_perm(xv.x, xv.z, 0x5410);
    P[1] = __byte_perm(xv.x, xv.z, 0x7632);
    P[2] = __byte_perm(xv.y, xv.w, 0x5410);
    P[3] = __byte_perm(xv.y, xv.w, 0x7632);
}

__device__ __forceinline__ void mma16816(float c[4], const uint32_t a[4], uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
                 "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t word_i(const uint4 &v, int i)
{
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// Bounded wait that ignores the abort flag: used to drain in-flight copies.
__device__ __forceinline__ void mbar_drain(uint64_t *bar, uint32_t parity, int *status)
{
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_ns() - t0 > kWaitLimitNs) {
            record_timeout(status);
            return;
        }
    }
}

__device__ __forceinline__ uint4 lds128(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

template <int NT, bool XSMEM, bool EVEN_G>
__global__ void __launch_bounds__(kThreads)
gemv_w4a16_tma_kernel(const __grid_constant__ CUtensorMap tmap, const uint16_t *__restrict__ x, int64_t M,
                      int64_t N, int64_t K, const uint16_t *__restrict__ sc, const uint16_t *__restrict__ zp,
                      uint16_t *__restrict__ y, float *__restrict__ ws, int *__restrict__ counters,
                      int *__restrict__ status)
{
    extern __shared__ uint8_t smem_raw[];
    // 1 KB-align the ring (TMA destinations want 128 B at least)
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const SmemLayout L = smem_layout(M, K, XSMEM);
    uint8_t *stage = smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bars);
    uint64_t *empty = full + kStages;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L.flags);
    volatile int *last_flag = abort_flag + 1;
    volatile int *zero_word = abort_flag + 2;  // written once (0) at start, never again
    uint4 *xp = reinterpret_cast<uint4 *>(smem + L.xp);

    const int G = (int)(K >> 7);
    const int GP = (G + kPair - 1) / kPair;  // chunk pairs per tile (the last may be half empty)
    const int64_t tiles = (N + kTileRows - 1) / kTileRows;
    const int64_t total = tiles * GP;
    const int64_t b = blockIdx.x;
    const int64_t per = total / gridDim.x, extra = total % gridDim.x;
    const int64_t beg = b * per + (b < extra ? b : extra);
    const int64_t end = beg + per + (b < extra ? 1 : 0);

    const int tid = threadIdx.x, wid = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumers);
        }
        *abort_flag = 0;
        *last_flag = 0;
        *zero_word = 0;
        fence_mbar_init();
    }
    if (XSMEM) {
        // xp[((ch * M + m) * 4 + c) * 4 + i] = k-permuted pairs of x[m][ch*128 + 32c + 8i .. +8],
        // followed by a zero row that lanes of padded rows m >= M read instead
        const int Mi = (int)M;
        for (int t = tid; t < G * Mi * 16; t += kThreads) {
            const int i = t & 3, c = (t >> 2) & 3, cm = t >> 4;
            const int m = cm % Mi, ch = cm / Mi;
            const uint4 xv = *reinterpret_cast<const uint4 *>(x + (int64_t)m * K + ch * 128 + c * 32 + i * 8);
            uint32_t P[4];
            pair_x(xv, P);
            xp[t] = make_uint4(P[0], P[1], P[2], P[3]);
        }
        if (tid < 16) xp[G * Mi * 16 + tid] = make_uint4(0u, 0u, 0u, 0u);
    }
    __syncthreads();

    if (wid == kConsumers) {
        // ---------------- producer ----------------
        if (lane == 0 && beg < end) {
            int64_t issued = 0;
            int s = 0;
            uint32_t phase = 0;
            int64_t tile = beg / GP;
            int cp = (int)(beg - tile * GP);
            for (int64_t u = beg; u < end; ++u) {
                if (issued >= kStages && !mbar_wait_fast(&empty[s], phase ^ 1u, status, abort_flag)) break;
                mbar_arrive_expect_tx(&full[s], kStageBytes);
                tma_load_2d(stage + s * kStageBytes, &tmap, &full[s], cp * kStageRowBytes, (int)(tile * kTileRows));
                ++issued;
                if (++s == kStages) { s = 0; phase ^= 1u; }
                if (++cp == GP) { cp = 0; ++tile; }
            }
            // every issued copy must land before this CTA may exit
            const int64_t first = issued > kStages ? issued - kStages : 0;
            for (int64_t j = first; j < issued; ++j)
                mbar_drain(&full[(int)(j % kStages)], (uint32_t)((j / kStages) & 1), status);
        }
        return;
    }

    // ---------------- consumers ----------------
    const uint32_t opaque_zero = (uint32_t)*zero_word;  // always 0, but opaque to the compiler
    const int r4 = lane >> 2, c = lane & 3;
    const uint32_t stage0 = smem_u32(stage) + (uint32_t)((wid * 16 + r4) * kStageRowBytes + c * 16);
    // k-permuted activations of this lane's rows m = nt*8 + r4 (the zero row when m >= M)
    uint32_t xp_row[NT], xp_step[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int m = nt * 8 + r4;
        const bool ok = m < M;
        xp_row[nt] = smem_u32(xp) + 16u * (uint32_t)(ok ? (m * 4 + c) * 4 : G * (int)M * 16 + c * 4);
        xp_step[nt] = ok ? 16u * (uint32_t)(M * 16) : 0u;  // bytes per chunk
    }
    const uint16_t *xg[NT];
    bool xok[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int64_t m = nt * 8 + r4;
        xok[nt] = m < M;
        xg[nt] = x + (xok[nt] ? m : 0) * K + c * 32;
    }

    int s = 0;
    uint32_t phase = 0;
    for (int64_t u = beg; u < end;) {
        const int64_t tile = u / GP;
        const int cp0 = (int)(u - tile * GP);
        const int cp1 = (int)((cp0 + (end - u) < GP) ? cp0 + (end - u) : GP);
        const int ch0 = cp0 * kPair, ch1 = cp1 * kPair < G ? cp1 * kPair : G;
        const int64_t n_a = tile * kTileRows + wid * 16 + r4, n_b = n_a + 8;
        const int64_t na = n_a < N ? n_a : N - 1, nb = n_b < N ? n_b : N - 1;
        const uint16_t *sa_p = sc + na * G, *sb_p = sc + nb * G;
        const uint16_t *za_p = zp + na * G, *zb_p = zp + nb * G;

        float acc[2][NT][2];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) acc[h][nt][0] = acc[h][nt][1] = 0.0f;

        // Scales and zero-points of the stage's two chunks: with an even group count the pair
        // (ch, ch+1) of a row is one aligned 32-bit word (low half = chunk ch).  Loaded two
        // stages ahead into raw registers that are not touched until their stage is consumed;
        // loads past the segment are predicated off.
        const uint32_t *s32a = reinterpret_cast<const uint32_t *>(sa_p), *s32b = reinterpret_cast<const uint32_t *>(sb_p);
        const uint32_t *z32a = reinterpret_cast<const uint32_t *>(za_p), *z32b = reinterpret_cast<const uint32_t *>(zb_p);
        auto ldsz = [&](int chq, uint32_t v[4]) {
            if (chq < ch1) {
                if (EVEN_G) {
                    v[0] = ld_nc_u32(s32a + (chq >> 1));
                    v[1] = ld_nc_u32(s32b + (chq >> 1));
                    v[2] = ld_nc_u32(z32a + (chq >> 1));
                    v[3] = ld_nc_u32(z32b + (chq >> 1));
                } else {
                    const int c2 = chq + 1 < G ? chq + 1 : chq;
                    v[0] = (uint32_t)ld_nc_u16(sa_p + chq) | ((uint32_t)ld_nc_u16(sa_p + c2) << 16);
                    v[1] = (uint32_t)ld_nc_u16(sb_p + chq) | ((uint32_t)ld_nc_u16(sb_p + c2) << 16);
                    v[2] = (uint32_t)ld_nc_u16(za_p + chq) | ((uint32_t)ld_nc_u16(za_p + c2) << 16);
                    v[3] = (uint32_t)ld_nc_u16(zb_p + chq) | ((uint32_t)ld_nc_u16(zb_p + c2) << 16);
                }
            }
        };
        uint32_t szc[4] = {0u, 0u, 0u, 0u}, szn[4] = {0u, 0u, 0u, 0u}, szm[4] = {0u, 0u, 0u, 0u};
        ldsz(ch0, szc);
        ldsz(ch0 + kPair, szn);
        ldsz(ch0 + 2 * kPair, szm);

        for (int ch = ch0; ch < ch1; ch += kPair) {
            mbar_wait_fast(&full[s], phase, status, abort_flag);
            const uint32_t wsrc = stage0 + (uint32_t)s * kStageBytes;
            uint4 wa[kPair], wb[kPair];
#pragma unroll
            for (int pc = 0; pc < kPair; ++pc) {
                wa[pc] = lds128(wsrc + pc * kChunkBytes);
                wb[pc] = lds128(wsrc + pc * kChunkBytes + 8 * kStageRowBytes);
            }
            // Release the slot as soon as every lane's reads have landed: the xor below cannot
            // execute before all 16 loaded words are in registers, the vote waits for every lane,
            // and the arrive takes the vote's result as an operand, so it cannot issue earlier.
            {
                uint32_t d = (wa[0].x ^ wa[0].y ^ wa[0].z) ^ (wa[0].w ^ wb[0].x ^ wb[0].y) ^ (wb[0].z ^ wb[0].w);
                d ^= (wa[1].x ^ wa[1].y ^ wa[1].z) ^ (wa[1].w ^ wb[1].x ^ wb[1].y) ^ (wb[1].z ^ wb[1].w);
                const uint32_t all = __ballot_sync(0xffffffffu, d == 0x9e3779b9u);
                if (lane == 0) mbar_arrive_after(&empty[s], all, opaque_zero);
            }
            if (++s == kStages) { s = 0; phase ^= 1u; }

#pragma unroll
            for (int pc = 0; pc < kPair; ++pc) {
                const int chc = ch + pc;
                if (pc > 0 && chc >= ch1) break;  // odd group count: the last stage is half empty
                // bf16 of chunk ch + pc: low half for pc = 0, high half for pc = 1
                const float s_a = __uint_as_float(pc ? (szc[0] & 0xffff0000u) : (szc[0] << 16));
                const float s_b = __uint_as_float(pc ? (szc[1] & 0xffff0000u) : (szc[1] << 16));
                float zl_a = __uint_as_float(pc ? (szc[2] & 0xffff0000u) : (szc[2] << 16));
                float zl_b = __uint_as_float(pc ? (szc[3] & 0xffff0000u) : (szc[3] << 16));
                // a zero-point outside [0, 15] anywhere in the warp: split it (zp_split) for this group
                const bool wide = __any_sync(0xffffffffu, !(zl_a >= 0.0f && zl_a <= 15.0f && zl_b >= 0.0f && zl_b <= 15.0f));
                float zh_a = 0.0f, zh_b = 0.0f;
                if (wide) {
                    zl_a = zp_split(zl_a, zh_a);
                    zl_b = zp_split(zl_b, zh_b);
                }
                const uint32_t zz_a = bf16_pair_128_plus(zl_a), zz_b = bf16_pair_128_plus(zl_b);
                uint32_t P[NT][4][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if (XSMEM) {
                        const uint32_t base = xp_row[nt] + (uint32_t)chc * xp_step[nt];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const uint4 v = lds128(base + 16u * i);
                            P[nt][i][0] = v.x; P[nt][i][1] = v.y; P[nt][i][2] = v.z; P[nt][i][3] = v.w;
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            uint4 xv = ld_nc_v4(xg[nt] + (int64_t)chc * 128 + i * 8);
                            if (!xok[nt]) xv = make_uint4(0u, 0u, 0u, 0u);
                            pair_x(xv, P[nt][i]);
                        }
                    }
                }
                float C[2][NT][4];
#pragma unroll
                for (int e = 0; e < 2; ++e)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) C[e][nt][0] = C[e][nt][1] = C[e][nt][2] = C[e][nt][3] = 0.0f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t va = word_i(wa[pc], i), vb = word_i(wb[pc], i);
                    uint32_t RA[4], RB[4];
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        RA[t] = sub_bf16x2(nib_pair_bf16(va, 4 * t), zz_a);  // exact q - z
                        RB[t] = sub_bf16x2(nib_pair_bf16(vb, 4 * t), zz_b);
                    }
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint32_t a[4] = {RA[2 * h], RB[2 * h], RA[2 * h + 1], RB[2 * h + 1]};
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) mma16816(C[i & 1][nt], a, P[nt][i][2 * h], P[nt][i][2 * h + 1]);
                    }
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    float d[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) d[e] = C[0][nt][e] + C[1][nt][e];
                    if (wide) {
                        // activation sums of this group: lane (r4, c) holds 32 values of row nt*8 + r4, the
                        // four lanes of a quad the whole group; D's columns 2c, 2c + 1 need rows 2c, 2c + 1
                        float xs = 0.0f;
#pragma unroll
                        for (int i = 0; i < 4; ++i) xs += sum_bf16x8(make_uint4(P[nt][i][0], P[nt][i][1], P[nt][i][2], P[nt][i][3]));
                        xs += __shfl_xor_sync(0xffffffffu, xs, 1);
                        xs += __shfl_xor_sync(0xffffffffu, xs, 2);
                        const float x0 = __shfl_sync(0xffffffffu, xs, 8 * c), x1 = __shfl_sync(0xffffffffu, xs, 8 * c + 4);
                        d[0] = fmaf(-zh_a, x0, d[0]);
                        d[1] = fmaf(-zh_a, x1, d[1]);
                        d[2] = fmaf(-zh_b, x0, d[2]);
                        d[3] = fmaf(-zh_b, x1, d[3]);
                    }
                    acc[0][nt][0] = fmaf(s_a, d[0], acc[0][nt][0]);
                    acc[0][nt][1] = fmaf(s_a, d[1], acc[0][nt][1]);
                    acc[1][nt][0] = fmaf(s_b, d[2], acc[1][nt][0]);
                    acc[1][nt][1] = fmaf(s_b, d[3], acc[1][nt][1]);
                }
            }
            // advance the scale/zero window by one stage, fetching two stages ahead
#pragma unroll
            for (int q = 0; q < 4; ++q) { szc[q] = szn[q]; szn[q] = szm[q]; }
            ldsz(ch + 3 * kPair, szm);
            (void)szm;
        }

        // ---- tile output ----
        const bool whole = (ch0 == 0 && ch1 == G);
        if (whole) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int64_t n = h ? n_b : n_a;
                if (n >= N) continue;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int64_t m = nt * 8 + 2 * c + e;
                        if (m < M) y[m * N + n] = f32_to_bf16(acc[h][nt][e]);
                    }
            }
        } else {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int64_t n = h ? n_b : n_a;
                if (n >= N) continue;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int64_t m = nt * 8 + 2 * c + e;
                        if (m < M) atomicAdd(ws + m * N + n, acc[h][nt][e]);
                    }
            }
            __threadfence();
            named_bar_sync(1, kConsumers * 32);
            if (tid == 0) {
                const int add = ch1 - ch0;
                const int prev = atomicAdd(counters + tile, add);
                *last_flag = (prev + add == G) ? 1 : 0;
            }
            named_bar_sync(1, kConsumers * 32);
            if (*last_flag) {
                __threadfence();
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int64_t n = h ? n_b : n_a;
                    if (n >= N) continue;
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int64_t m = nt * 8 + 2 * c + e;
                            if (m < M) y[m * N + n] = f32_to_bf16(atomicExch(ws + m * N + n, 0.0f));
                        }
                }
                named_bar_sync(1, kConsumers * 32);
                if (tid == 0) atomicExch(counters + tile, 0);
            }
        }
        u += cp1 - cp0;
    }
}

template <int NT, bool XSMEM, bool EVEN_G>
int run(const uint16_t *x, int64_t M, int64_t N, int64_t K, const uint8_t *q, const uint16_t *s, const uint16_t *z,
        uint16_t *y, float *ws, int *counters, int *status, cudaStream_t st)
{
    CUtensorMap map;
    if (!encode_tmap_2d(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, (uint64_t)(K / 2), (uint64_t)N, (uint64_t)(K / 2),
                        kStageRowBytes, kTileRows, CU_TENSOR_MAP_SWIZZLE_NONE))
        return -1;
    auto kern = gemv_w4a16_tma_kernel<NT, XSMEM, EVEN_G>;
    const size_t smem = smem_layout(M, K, XSMEM).total + 1024;
    // launch shape per (device, shared-memory size), computed once
    static std::mutex mu;
    static std::map<std::pair<int, size_t>, int> capacity;
    int dev = 0;
    cudaGetDevice(&dev);
    int cap;
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = capacity.find({dev, smem});
        if (it == capacity.end()) {
            int sms = 148, per_sm = 1, optin = 0;
            // allow the largest opt-in size once, so any later size launches too
            cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
            it = capacity.emplace(std::make_pair(dev, smem), sms * std::max(per_sm, 1)).first;
        }
        cap = it->second;
    }
    const int64_t total = ((N + kTileRows - 1) / kTileRows) * ((K / 128 + kPair - 1) / kPair);
    const unsigned grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>(total, cap));
    kern<<<grid, kThreads, smem, st>>>(map, x, M, N, K, s, z, y, ws, counters, status);
    return 0;
}

}  // namespace

size_t gemv_tma_workspace_bytes(int64_t M, int64_t N, int64_t K, int g)
{
    if (!gemv_tma_eligible(M, N, K, g)) return 0;
    const int64_t tiles = (N + kTileRows - 1) / kTileRows;
    return counter_region_bytes(tiles) + align_up(sizeof(float) * (size_t)(M * N), 256);
}

bool gemv_tma_eligible(int64_t M, int64_t N, int64_t K, int g)
{
    // M = 1 runs faster on the CUDA-core kernel (measured); the pipeline serves 2 <= M <= 16
    return g == 128 && M >= 2 && M <= 16 && N >= kTileRows && K >= 256 && K / 128 <= 0x7fffffff / 64;
}

size_t gemv_tma_compact_bytes(int64_t M, int64_t N, int64_t K, int g)
{
    if (!gemv_tma_eligible(M, N, K, g)) return 0;
    const int64_t tiles = (N + kTileRows - 1) / kTileRows;
    return align_up(sizeof(float) * (size_t)(M * N), 256) + align_up(sizeof(int) * (size_t)tiles, 256);
}

int launch_gemv_w4a16_tma(const uint16_t *x, int64_t M, int64_t N, int64_t K, const uint8_t *q, const uint16_t *s,
                          const uint16_t *z, uint16_t *y, void *workspace, int *status, cudaStream_t st, bool compact)
{
    const int64_t tiles = (N + kTileRows - 1) / kTileRows;
    uint8_t *w8 = static_cast<uint8_t *>(workspace);
    int *counters;
    float *ws;
    if (compact) {  // a private scratch area cleared before every call: partial sums first, counters after
        ws = reinterpret_cast<float *>(w8);
        counters = reinterpret_cast<int *>(w8 + align_up(sizeof(float) * (size_t)(M * N), 256));
    } else {
        counters = reinterpret_cast<int *>(w8);
        ws = reinterpret_cast<float *>(w8 + counter_region_bytes(tiles));
        if (clear_extra_counters(workspace, tiles, st) != cudaSuccess) return -2;
        // the partial sums meet in binary32 atomics, so they must start at zero; in a workspace shared with
        // other shapes this region may hold their partial sums
        if (cudaMemsetAsync(ws, 0, sizeof(float) * (size_t)(M * N), st) != cudaSuccess) return -2;
    }
    const bool xsmem = (size_t)M * (size_t)K * 2 <= 32 * 1024;
    const bool even = ((K / 128) & 1) == 0;
#define WQ_RUN(NT, XS, EV) return run<NT, XS, EV>(x, M, N, K, q, s, z, y, ws, counters, status, st)
    if (M <= 8) {
        if (xsmem) { if (even) WQ_RUN(1, true, true); WQ_RUN(1, true, false); }
        if (even) WQ_RUN(1, false, true);
        WQ_RUN(1, false, false);
    }
    if (xsmem) { if (even) WQ_RUN(2, true, true); WQ_RUN(2, true, false); }
    if (even) WQ_RUN(2, false, true);
    WQ_RUN(2, false, false);
#undef WQ_RUN
}

}  // namespace wq

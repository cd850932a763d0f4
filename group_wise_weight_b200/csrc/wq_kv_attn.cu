// wq_kv_attn.cu -- the decode-attention read of a quantised KV cache.
//
// "Quantization Methods Compared: INT8, GPTQ, AWQ, FP8, FP4 and KV-Cache
// Quantization", section "Hardware, formats and the roofline": every decode
// step reads the whole KV cache of every sequence, and at batch 128 with
// 8,000-token contexts those reads (335.5 GB for a 70B model) outweigh the
// weights -- which is why 4-bit weights alone stop paying off there.
// "Quantization for LLM inference: FP8, INT4 (GPTQ, AWQ) and GGUF", section
// "KV cache quantization": the cache is kept in fp8 (one byte per value) or
// in int4 with blocks of 128 values (half a byte plus the scale overhead).
//
// Formats (the pages give sizes only; the reading taken here):
//  * K and V of one layer are each [B][T][H][D] (sequences, token slots, KV
//    heads, head_dim), D = 128.
//  * int4: each (b, t, h) vector is one block of 128 values in the weight
//    format of wq_quantize_int4 with g = 128 -- codes [B][T][H][64] bytes,
//    bf16 scale and zero-point per vector ([B][T][H] each): v_hat = s (q - z).
//  * fp8: E4M3 codes [B][T][H][128] with one binary32 scale per tensor, as
//    wq_quantize_fp8_tensor writes them: v_hat = s * e4m3(code).
// The read is decode attention (scaled dot-product attention, Vaswani et al.
// 2017, section 3.2.1) of one new query token per sequence over its first
// len_b cached tokens, query head j reading KV head j / (Hq / H):
//   score_t = (q_j . k_hat_t) / sqrt(D),  p = softmax(score),  o_j = sum_t p_t v_hat_t.
// A sequence with len_b = 0 gives o = 0.
//
// Design.  The pass is bound by reading the cache (int4: 136 bytes per token
// and KV head for K and V together), and at 4,096 flop per 136 bytes it needs
// tensor cores to keep up with HBM.  The query heads that share a KV head
// (r = Hq / H <= 8) share every cache read.
//  * Kernel 1: one CTA (4 warps) per (KV head, chunk of 1,024 tokens,
//    sequence).  Phase 1: each warp takes 16-token tiles, dequantises K into
//    the A operand of mma.sync m16n8k16 (tokens x d) and multiplies by the r
//    queries (d x heads, padded to 8).  int4 codes become the exact integers
//    q - z in bf16 (a LOP3 per code pair gives 128 + q, one bf16 subtraction
//    of 128 + z), so each token's scale s multiplies its row of scores in
//    binary32 afterwards.  The chunk's scores stay in shared memory.  Phase
//    2, after the chunk's exact per-head maximum is known: p = exp(score -
//    max) for every token, and o^T (d x heads) = V^T P^T with V^T the A
//    operand (d x tokens, again the exact q - z for int4) and
//    p_t * s_t (the token's V scale folded in, rounded to bf16) the B
//    operand.  The chunk writes its unnormalised o, its maxima and its sums
//    of p to the workspace.
//  * Kernel 2 merges the chunks of each (sequence, query head):
//    o = sum_c e^(m_c - m) o_c / sum_c e^(m_c - m) l_c, in binary32.
//  * fp8: the codes convert exactly to f16 pairs (cvt.rn.f16x2.e4m3x2) and
//    the MMAs run in f16; each query head is scaled by a power of two into
//    f16's range (exact) and the scale is undone in binary32.
// A zero-point outside [0, 15] (a vector on one side of zero) is split as in
// the matmul kernels: the operand holds q - z_lo and the term -s z_hi times
// the query sum (K) or the weight sum (V) is added in binary32.
#include <algorithm>

#include "wq_common.cuh"
#include "wq_internal.h"

namespace wq {

namespace {

constexpr int kD = 128;          // head_dim
constexpr int kChunk = 1024;     // tokens per CTA: 256 per warp (128 measured 25% slower, 512 slower again)
constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kTokPerWarp = kChunk / kWarps;  // 256
constexpr int kR = 8;            // query heads per KV head, padded

__device__ __forceinline__ void mma_bf16(float c[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16(float c[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                        uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two E4M3 codes (low byte first) as an exact f16 pair.
__device__ __forceinline__ uint32_t e4m3x2_f16x2(uint32_t two_codes)
{
    uint32_t r;
    asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(r) : "r"(two_codes));
    return r;
}

__device__ __forceinline__ uint32_t f16x2_of(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ uint32_t word_of4(const uint4 &v, int i)
{
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

__device__ __forceinline__ uint32_t lop_nib(uint32_t v)  // (v & 0x000F000F) | 0x43004300: 128 + nibble pairs
{
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(v), "r"(0x000F000Fu), "r"(0x43004300u));
    return d;
}

struct KvArgs {
    const uint16_t *q;                  // [B][Hq][D] bf16
    const uint8_t *kc, *vc;             // codes
    const uint16_t *ks, *kz, *vs, *vz;  // int4: per-vector bf16 scale / zero-point [B][T][H]
    const float *k8s, *v8s;             // fp8: per-tensor scales
    const int *lengths;                 // [B]
    int B, T, H, Hq, r, nchunk;
    float *part;                        // [B][H][nchunk][kR][D + 2]: o (unnormalised), max, sum
};

// Query heads of KV head h as B operands of the QK^T MMA, in the k order the int4 A operand uses:
// step s = 2w + e takes from thread (g, tq) the d values 32 tq + 8 w + 2 e + {0, 4} (first register) and
// + {1, 5} (second register) of query head g.  Also returns the query sum of head g (for far zero-points).
template <bool F16>
__device__ __forceinline__ float load_q(const KvArgs &a, int b, int h, int g, int tq, uint32_t qf[8][2], float &qscale)
{
    const int j = h * a.r + g;
    float qv[32];
    if (g < a.r) {
        const uint4 *src = reinterpret_cast<const uint4 *>(a.q + ((size_t)b * a.Hq + j) * kD + 32 * tq);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint4 u = src[c];
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                qv[8 * c + 2 * i] = __uint_as_float(w[i] << 16);
                qv[8 * c + 2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) qv[i] = 0.0f;
    }
    // fp8: scale the head by a power of two so that its largest magnitude lies in [2^14, 2^15) (exact)
    qscale = 1.0f;
    if (F16) {
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(qv[i]));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        if (amax > 0.0f) {
            const int e = 14 - ((int)((__float_as_uint(amax) >> 23) & 0xff) - 127);
            qscale = __uint_as_float((uint32_t)(127 + e) << 23);
        }
    }
    float qsum = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) qsum += qv[i];
#pragma unroll
    for (int s = 0; s < 8; ++s) {
        const int w = s >> 1, e = s & 1;
        const float *v = qv + 8 * w + 2 * e;
        if (F16) {
            qf[s][0] = f16x2_of(v[0] * qscale, v[4] * qscale);
            qf[s][1] = f16x2_of(v[1] * qscale, v[5] * qscale);
        } else {
            qf[s][0] = pack_bf16x2(v[0], v[4]);
            qf[s][1] = pack_bf16x2(v[1], v[5]);
        }
    }
    qsum += __shfl_xor_sync(0xffffffffu, qsum, 1);
    qsum += __shfl_xor_sync(0xffffffffu, qsum, 2);
    return qsum;
}

// int4 A operand of one token row: 16 code bytes (d = 32 tq .. 32 tq + 31) minus the zero-point pair, in
// the k order of load_q: a[s][0] = pair (d0 + 8w + 2e, +4), a[s][1] = (+1, +5), s = 2w + e.
__device__ __forceinline__ void int4_row(const uint4 c, uint32_t zz, uint32_t a[8][2])
{
    const uint32_t w4[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const uint32_t v = w4[w];
        const uint32_t p0 = sub_bf16x2(lop_nib(v), zz);        // (c0, c4)
        const uint32_t p1 = sub_bf16x2(lop_nib(v >> 4), zz);   // (c1, c5)
        const uint32_t p2 = sub_bf16x2(lop_nib(v >> 8), zz);   // (c2, c6)
        const uint32_t p3 = sub_bf16x2(lop_nib(v >> 12), zz);  // (c3, c7)
        a[2 * w][0] = p0;
        a[2 * w][1] = p1;
        a[2 * w + 1][0] = p2;
        a[2 * w + 1][1] = p3;
    }
}

// fp8 A operand of one token row: 32 code bytes (d = 32 tq .. 32 tq + 31) in the same k order as int4_row
// (pairs (d, d + 4) and (d + 1, d + 5) of each group of 8).
__device__ __forceinline__ void fp8_row(const uint4 c0, const uint4 c1, uint32_t a[8][2])
{
    const uint32_t w8[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const uint32_t lo = w8[2 * w], hi = w8[2 * w + 1];  // codes d0..d3, d4..d7
        a[2 * w][0] = e4m3x2_f16x2(__byte_perm(lo, hi, 0x0040));      // (d0, d4)
        a[2 * w][1] = e4m3x2_f16x2(__byte_perm(lo, hi, 0x0051));      // (d1, d5)
        a[2 * w + 1][0] = e4m3x2_f16x2(__byte_perm(lo, hi, 0x0062));  // (d2, d6)
        a[2 * w + 1][1] = e4m3x2_f16x2(__byte_perm(lo, hi, 0x0073));  // (d3, d7)
    }
}

template <bool FP8>
__global__ void __launch_bounds__(kThreads)
kv_attn_chunk_kernel(const KvArgs a)
{
    __shared__ float sc[kChunk][kR];  // scores, then the cross-warp reduction of o
    __shared__ float red[kWarps][2 * kR];
    __shared__ float hmax[kR];
    const int h = blockIdx.x, chunk = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, wid = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, tq = lane & 3;
    const int len = min(max(a.lengths[b], 0), a.T);
    const int t0 = chunk * kChunk;
    const int tend = min(t0 + kChunk, len);
    float *out = a.part + ((((size_t)b * a.H + h) * a.nchunk + chunk) * kR) * (kD + 2);
    if (t0 >= tend) {
        // no token of this chunk is live: an empty partial (sum 0, maximum -inf)
        for (int i = tid; i < kR * (kD + 2); i += kThreads)
            out[i] = (i % (kD + 2)) == kD ? -INFINITY : 0.0f;
        return;
    }
    const float rsqrt_d = 0.08838834764831845f;  // 1 / sqrt(128)
    const float k8 = FP8 ? *a.k8s : 1.0f, v8 = FP8 ? *a.v8s : 1.0f;
    uint32_t qf[8][2];
    float qscale;
    const float qsum = load_q<FP8>(a, b, h, g, tq, qf, qscale);  // sum of query head g
    // thread (g, tq) needs the query sums of heads 2 tq and 2 tq + 1 (held by lanes 8 tq .. and 8 tq + 4 ..)
    const float qsum0 = __shfl_sync(0xffffffffu, qsum, (2 * tq) * 4);
    const float qsum1 = __shfl_sync(0xffffffffu, qsum, (2 * tq + 1) * 4);
    const float inv_q0 = FP8 ? 1.0f / __shfl_sync(0xffffffffu, qscale, (2 * tq) * 4) : 1.0f;
    const float inv_q1 = FP8 ? 1.0f / __shfl_sync(0xffffffffu, qscale, (2 * tq + 1) * 4) : 1.0f;
    const size_t row_stride = (size_t)a.H;  // vectors between consecutive tokens
    const size_t vec0 = ((size_t)b * a.T) * a.H + h;  // vector index of token 0 of this (b, h)
    constexpr int kRowBytes = FP8 ? kD : kD / 2;

    // ---------------- phase 1: scores of this warp's tokens ----------------
    const int wt0 = t0 + wid * kTokPerWarp;
    // the next 16-token tile's loads are issued before the current tile is dequantised and multiplied
    struct KRaw {
        uint4 c0, c1, d0, d1;  // code bytes of tokens base + g (c) and base + g + 8 (d); int4 uses c0, d0
        uint16_t sa, za, sb, zb;
    };
    auto load_k = [&](int base) {
        KRaw t;
        t.c0 = t.c1 = t.d0 = t.d1 = make_uint4(0, 0, 0, 0);
        t.sa = t.sb = 0;
        t.za = t.zb = 0;
        const int ta = base + g, tb = base + g + 8;
        if (ta < tend) {
            const size_t v = vec0 + (size_t)ta * row_stride;
            if (FP8) {
                const uint4 *p = reinterpret_cast<const uint4 *>(a.kc + v * kRowBytes + 32 * tq);
                t.c0 = ld_nc_v4(p);
                t.c1 = ld_nc_v4(p + 1);
            } else {
                t.c0 = ld_nc_v4(a.kc + v * kRowBytes + 16 * tq);
                t.sa = ld_nc_u16(a.ks + v);
                t.za = ld_nc_u16(a.kz + v);
            }
        }
        if (tb < tend) {
            const size_t v = vec0 + (size_t)tb * row_stride;
            if (FP8) {
                const uint4 *p = reinterpret_cast<const uint4 *>(a.kc + v * kRowBytes + 32 * tq);
                t.d0 = ld_nc_v4(p);
                t.d1 = ld_nc_v4(p + 1);
            } else {
                t.d0 = ld_nc_v4(a.kc + v * kRowBytes + 16 * tq);
                t.sb = ld_nc_u16(a.ks + v);
                t.zb = ld_nc_u16(a.kz + v);
            }
        }
        return t;
    };
    KRaw nxt = load_k(wt0);
#pragma unroll 1
    for (int base = wt0; base < wt0 + kTokPerWarp && base < tend; base += 16) {
        const int ta = base + g, tb = base + g + 8;
        const bool la = ta < tend, lb = tb < tend;
        const KRaw cur = nxt;
        if (base + 16 < wt0 + kTokPerWarp && base + 16 < tend) nxt = load_k(base + 16);
        uint32_t A0[8][2], A1[8][2];
        float sa = 0.0f, sb = 0.0f, zha = 0.0f, zhb = 0.0f;
        if (FP8) {
            fp8_row(cur.c0, cur.c1, A0);
            fp8_row(cur.d0, cur.d1, A1);
            sa = k8;
            sb = k8;
        } else {
            sa = bf16_to_f32(cur.sa);
            sb = bf16_to_f32(cur.sb);
            float za = bf16_to_f32(cur.za), zb = bf16_to_f32(cur.zb);
            if (!(za >= 0.0f && za <= 15.0f)) za = zp_split(za, zha);
            if (!(zb >= 0.0f && zb <= 15.0f)) zb = zp_split(zb, zhb);
            int4_row(cur.c0, bf16_pair_128_plus(za), A0);
            int4_row(cur.d0, bf16_pair_128_plus(zb), A1);
        }
        float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            if (FP8) mma_f16(acc, A0[s][0], A1[s][0], A0[s][1], A1[s][1], qf[s][0], qf[s][1]);
            else mma_bf16(acc, A0[s][0], A1[s][0], A0[s][1], A1[s][1], qf[s][0], qf[s][1]);
        }
        // score = s_t (D - z_hi qsum) / sqrt(D); rows g (acc 0, 1) and g + 8 (acc 2, 3); heads 2 tq, 2 tq + 1
        const float s0 = (acc[0] * inv_q0 - zha * qsum0) * sa * rsqrt_d;
        const float s1 = (acc[1] * inv_q1 - zha * qsum1) * sa * rsqrt_d;
        const float s2 = (acc[2] * inv_q0 - zhb * qsum0) * sb * rsqrt_d;
        const float s3 = (acc[3] * inv_q1 - zhb * qsum1) * sb * rsqrt_d;
        const int ra = base + g - t0, rb = base + g + 8 - t0;
        sc[ra][2 * tq] = la ? s0 : -INFINITY;
        sc[ra][2 * tq + 1] = la ? s1 : -INFINITY;
        sc[rb][2 * tq] = lb ? s2 : -INFINITY;
        sc[rb][2 * tq + 1] = lb ? s3 : -INFINITY;
    }
    __syncthreads();

    // ---------------- the chunk's maximum per head ----------------
    {
        const int j = tid & 7;  // head
        float m = -INFINITY;
        for (int t = tid >> 3; t < tend - t0; t += kThreads / 8) m = fmaxf(m, sc[t][j]);
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
        if (lane < 8) red[wid][lane] = m;
        __syncthreads();
        if (tid < kR) {
            float mm = red[0][tid];
            for (int w = 1; w < kWarps; ++w) mm = fmaxf(mm, red[w][tid]);
            hmax[tid] = mm;
        }
        __syncthreads();
    }

    // ---------------- phase 2: o^T = V^T P^T over this warp's tokens ----------------
    // thread (g, tq): d values 16 g .. 16 g + 15 (m tile i holds d = 16 g + 2 i in row g and 16 g + 2 i + 1 in
    // row g + 8), tokens 4 tq .. 4 tq + 3 of each 16-token step (k = 2 tq, 2 tq + 1 -> tokens 4 tq, 4 tq + 1;
    // k = 2 tq + 8, 2 tq + 9 -> tokens 4 tq + 2, 4 tq + 3), query head g for the B operand.
    float o[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
    float lsum = 0.0f;   // sum of p over this thread's tokens, head g
    float zcorr = 0.0f;  // sum of p' z_hi over this thread's tokens, head g (zero-points outside [0, 15])
    const float mg = g < a.r ? hmax[g] : 0.0f;
    // V codes (and, int4, the V scales and zero-points) of the 4 tokens 4 tq + u of a 16-token step: the
    // next step's are loaded before the current one is used
    struct VRaw {
        uint4 c[4];  // fp8: 16 bytes (d = 16 g ..) per token; int4: 8 bytes in .x, .y
        uint16_t s[4], z[4];
    };
    auto load_v = [&](int base) {
        VRaw t;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int tt = base + 4 * tq + u;
            t.c[u] = make_uint4(0, 0, 0, 0);
            t.s[u] = 0;
            t.z[u] = 0;
            if (tt < tend) {
                const size_t v = vec0 + (size_t)tt * row_stride;
                if (FP8) {
                    t.c[u] = ld_nc_v4(a.vc + v * kRowBytes + 16 * g);
                } else {
                    const uint2 w2 = *reinterpret_cast<const uint2 *>(a.vc + v * kRowBytes + 8 * g);
                    t.c[u].x = w2.x;
                    t.c[u].y = w2.y;
                    t.s[u] = ld_nc_u16(a.vs + v);
                    t.z[u] = ld_nc_u16(a.vz + v);
                }
            }
        }
        return t;
    };
    VRaw vnext = load_v(wt0);
#pragma unroll 1
    for (int base = wt0; base < wt0 + kTokPerWarp && base < tend; base += 16) {
        const VRaw vcur = vnext;
        if (base + 16 < wt0 + kTokPerWarp && base + 16 < tend) vnext = load_v(base + 16);
        float pv[4];  // p' of tokens 4 tq + u, head g: p * s_t (int4) or p (fp8; its scale is applied at the end)
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int t = base + 4 * tq + u;
            const float p = (t < tend && g < a.r) ? __expf(sc[t - t0][g] - mg) : 0.0f;
            lsum += p;
            pv[u] = p;
        }
        if constexpr (FP8) {
            const uint32_t b0 = f16x2_of(pv[0], pv[1]), b1 = f16x2_of(pv[2], pv[3]);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                // m tile i: row g takes d = 16 g + 2 i, row g + 8 takes d = 16 g + 2 i + 1 (bytes 2 i, 2 i + 1)
                const int wi = i >> 1;
                const uint32_t s_lo = (i & 1) ? 0x0062u : 0x0040u, s_hi = (i & 1) ? 0x0073u : 0x0051u;
                const uint32_t x0 = word_of4(vcur.c[0], wi), x1 = word_of4(vcur.c[1], wi);
                const uint32_t x2 = word_of4(vcur.c[2], wi), x3 = word_of4(vcur.c[3], wi);
                mma_f16(o[i], e4m3x2_f16x2(__byte_perm(x0, x1, s_lo)), e4m3x2_f16x2(__byte_perm(x0, x1, s_hi)),
                        e4m3x2_f16x2(__byte_perm(x2, x3, s_lo)), e4m3x2_f16x2(__byte_perm(x2, x3, s_hi)), b0, b1);
            }
        } else {
            float zh[4];
            uint32_t zlo[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                zh[u] = 0.0f;
                float z = bf16_to_f32(vcur.z[u]);
                if (!(z >= 0.0f && z <= 15.0f)) z = zp_split(z, zh[u]);
                zlo[u] = __float_as_uint(128.0f + z) >> 16;  // bf16 of 128 + z_lo (exact)
                pv[u] *= bf16_to_f32(vcur.s[u]);
            }
            const uint32_t zz0 = zlo[0] | (zlo[1] << 16), zz1 = zlo[2] | (zlo[3] << 16);
            const uint32_t b0 = pack_bf16x2(pv[0], pv[1]), b1 = pack_bf16x2(pv[2], pv[3]);
            // the rounded p' multiply the operands, so the z_hi correction uses the same rounded values
            zcorr += __uint_as_float(b0 << 16) * zh[0] + __uint_as_float(b0 & 0xffff0000u) * zh[1] +
                     __uint_as_float(b1 << 16) * zh[2] + __uint_as_float(b1 & 0xffff0000u) * zh[3];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                // byte i: low nibble d = 16 g + 2 i (row g), high nibble d + 1 (row g + 8)
                const int wi = i >> 2, bi = i & 3;
                // byte bi of the first token to bits 0-7, of the second to bits 16-23 (bytes 1 and 3 take a copy
                // of byte 0 of the first word, which the nibble masks below discard)
                const uint32_t sel = (uint32_t)(bi | ((4 + bi) << 8));
                const uint32_t x0 = wi ? vcur.c[0].y : vcur.c[0].x, x1 = wi ? vcur.c[1].y : vcur.c[1].x;
                const uint32_t x2 = wi ? vcur.c[2].y : vcur.c[2].x, x3 = wi ? vcur.c[3].y : vcur.c[3].x;
                const uint32_t pa = __byte_perm(x0, x1, sel);
                const uint32_t pb = __byte_perm(x2, x3, sel);
                mma_bf16(o[i], sub_bf16x2(lop_nib(pa), zz0), sub_bf16x2(lop_nib(pa >> 4), zz0),
                         sub_bf16x2(lop_nib(pb), zz1), sub_bf16x2(lop_nib(pb >> 4), zz1), b0, b1);
            }
        }
    }
    // l and the far-zero-point correction of head g: sum over the four tq lanes
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
    zcorr += __shfl_xor_sync(0xffffffffu, zcorr, 1);
    zcorr += __shfl_xor_sync(0xffffffffu, zcorr, 2);
    __syncthreads();  // every warp is done with the scores: reuse sc for the reduction of o over warps
    float *accum = &sc[0][0];  // [kR][kD]
    for (int i = tid; i < kR * kD; i += kThreads) accum[i] = 0.0f;
    if (tq == 0) {
        red[wid][g] = lsum;
        red[wid][kR + g] = zcorr;
    }
    __syncthreads();
    // this thread's outputs: heads 2 tq, 2 tq + 1; d = 16 g + 2 i (c0, c1) and 16 g + 2 i + 1 (c2, c3)
    for (int w = 0; w < kWarps; ++w) {
        if (wid == w) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int d0 = 16 * g + 2 * i;
                accum[(2 * tq) * kD + d0] += o[i][0];
                accum[(2 * tq + 1) * kD + d0] += o[i][1];
                accum[(2 * tq) * kD + d0 + 1] += o[i][2];
                accum[(2 * tq + 1) * kD + d0 + 1] += o[i][3];
            }
        }
        __syncthreads();
    }
    for (int i = tid; i < kR * kD; i += kThreads) {
        const int j = i / kD, d = i - j * kD;
        float zc = 0.0f;
        if (!FP8)
            for (int w = 0; w < kWarps; ++w) zc += red[w][kR + j];
        // o_j[d] = sum_t p'_t (q - z_lo) - sum_t p'_t z_hi   (int4);  v8 * sum_t p_t e4m3 (fp8)
        out[j * (kD + 2) + d] = FP8 ? accum[i] * v8 : accum[i] - zc;
    }
    if (tid < kR) {
        float l = 0.0f;
        for (int w = 0; w < kWarps; ++w) l += red[w][tid];
        out[tid * (kD + 2) + kD] = tid < a.r ? hmax[tid] : -INFINITY;
        out[tid * (kD + 2) + kD + 1] = l;
    }
}

// Merge the chunks of each (sequence, query head): o = sum_c e^(m_c - m) o_c / sum_c e^(m_c - m) l_c.
__global__ void __launch_bounds__(kD)
kv_attn_combine_kernel(const float *__restrict__ part, int H, int Hq, int r, int nchunk, float *__restrict__ o)
{
    const int j = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
    const int h = j / r, jj = j - h * r;
    const float *p = part + (((size_t)b * H + h) * nchunk * kR + jj) * (kD + 2);
    const size_t cstride = (size_t)kR * (kD + 2);
    float m = -INFINITY;
    for (int c = 0; c < nchunk; ++c) m = fmaxf(m, p[c * cstride + kD]);
    float num = 0.0f, den = 0.0f;
    if (m != -INFINITY) {
        for (int c = 0; c < nchunk; ++c) {
            const float mc = p[c * cstride + kD];
            if (mc == -INFINITY) continue;
            const float e = __expf(mc - m);
            num += e * p[c * cstride + d];
            den += e * p[c * cstride + kD + 1];
        }
    }
    o[((size_t)b * Hq + j) * kD + d] = den > 0.0f ? num / den : 0.0f;
}

}  // namespace

size_t kv_attn_workspace_bytes(int64_t B, int64_t T, int64_t H)
{
    const int64_t nchunk = (T + kChunk - 1) / kChunk;
    return (size_t)B * H * nchunk * kR * (kD + 2) * sizeof(float);
}

int launch_kv_attn(bool fp8, const uint16_t *q, const uint8_t *kc, const uint16_t *ks, const uint16_t *kz,
                   const float *k8s, const uint8_t *vc, const uint16_t *vs, const uint16_t *vz, const float *v8s,
                   const int *lengths, int64_t B, int64_t T, int64_t H, int64_t Hq, float *o, void *workspace,
                   cudaStream_t st)
{
    KvArgs a{};
    a.q = q; a.kc = kc; a.vc = vc; a.ks = ks; a.kz = kz; a.vs = vs; a.vz = vz; a.k8s = k8s; a.v8s = v8s;
    a.lengths = lengths;
    a.B = (int)B; a.T = (int)T; a.H = (int)H; a.Hq = (int)Hq; a.r = (int)(Hq / H);
    a.nchunk = (int)((T + kChunk - 1) / kChunk);
    a.part = static_cast<float *>(workspace);
    const dim3 grid((unsigned)H, (unsigned)a.nchunk, (unsigned)B);
    if (fp8) kv_attn_chunk_kernel<true><<<grid, kThreads, 0, st>>>(a);
    else kv_attn_chunk_kernel<false><<<grid, kThreads, 0, st>>>(a);
    kv_attn_combine_kernel<<<dim3((unsigned)Hq, (unsigned)B), kD, 0, st>>>(a.part, a.H, a.Hq, a.r, a.nchunk, o);
    return 0;
}

}  // namespace wq

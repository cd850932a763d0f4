"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Quantisation outputs (packed codes, bf16 scales, bf16 zero-points) must be
bit-exact.  Matmul outputs must satisfy, element by element,
    |y - y_ref| <= 4e-3 * sum_k |x[m][k] * w_hat[n][k]|
with y_ref and the sum computed by the oracle in binary64.  Inputs come from
the seeded generators in wq_inputs; small cases are compared in full, the
full-size workloads on sampled output rows the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import group_wise_weight_b200 as wq
import oracle
import wq_inputs
from group_wise_weight_b200 import build as wqbuild

pytestmark = pytest.mark.gpu
TOL = 4e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    wqbuild.build()
    wq.lib()
    torch.cuda.init()


@pytest.fixture(autouse=True)
def _no_device_timeouts():
    """Every test must leave the device status word clean (no bounded wait ran out)."""
    yield
    assert wq.wq_device_status() == wq.WQ_OK, "a kernel recorded a bounded-wait timeout"


def bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def w_f32(w: torch.Tensor) -> np.ndarray:
    return w.float().numpy()


def oracle_q4(w: torch.Tensor, g: int):
    codes, s, z = oracle.quantize_int4(w_f32(w), g)
    return codes, s, z, oracle.pack_int4(codes), oracle.bf16_bits(s), oracle.bf16_bits(z)


def oracle_q8(w: torch.Tensor, g: int):
    codes, s = oracle.quantize_int8(w_f32(w), g)
    return codes, s, oracle.bf16_bits(s)


def check_q4(w: torch.Tensor, g: int, rows=None):
    wd = w.cuda()
    q, s, z = wq.wq_quantize_int4(wd, g)
    torch.cuda.synchronize()
    sel = slice(None) if rows is None else rows
    codes, so, zo, packed, sb, zb = oracle_q4(w[sel], g)
    assert np.array_equal(q.cpu().numpy()[sel], packed), "packed codes differ"
    assert np.array_equal(bits(s)[sel], sb), "scales differ"
    assert np.array_equal(bits(z)[sel], zb), "zero-points differ"
    return q, s, z, (codes, so, zo)


def check_y(y: torch.Tensor, y_ref: np.ndarray, a_ref: np.ndarray) -> float:
    yg = y.double().cpu().numpy()
    err = np.abs(yg - y_ref)
    bound = TOL * a_ref
    bad = err > bound
    ratio = float(np.max(err / np.where(a_ref > 0, a_ref, 1.0)))
    assert not bad.any(), f"{bad.sum()} outputs outside 4e-3*sum|x*w_hat|; max ratio {ratio:.3e}"
    return ratio


def sample_rows(N: int, n: int, seed: int) -> np.ndarray:
    g = torch.Generator().manual_seed(seed)
    r = torch.randperm(N, generator=g)[:n].numpy()
    return np.unique(np.concatenate([r, [0, N - 1]]))


# ---------------------------------------------------------------------------
# Quantisation, bit-exact
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("g", [32, 64, 128])
def test_quantize_int4_tiny(g):
    check_q4(wq_inputs.tiny_weight(), g)


def test_quantize_int4_tiny_bf16_input():
    check_q4(wq_inputs.tiny_weight().to(torch.bfloat16), 128)


def test_quantize_int4_decode_up():
    w = wq_inputs.llm_weight(14336, 4096, wq_inputs.SEEDS["decode_up"])
    check_q4(w, 128)


def test_quantize_int4_gran_g32():
    w = wq_inputs.block_outlier_weight(8192, 8192, wq_inputs.SEEDS["gran"])
    check_q4(w, 32)


def test_quantize_int4_sweep_sampled_rows():
    w = wq_inputs.llm_weight(28672, 8192, wq_inputs.SEEDS["sweep"])
    check_q4(w, 128, rows=sample_rows(28672, 512, 1))


@pytest.mark.parametrize("g", [32, 128, None])
def test_quantize_int8(g):
    w = wq_inputs.block_outlier_weight(1024, 2048, 40)
    gg = 2048 if g is None else g
    wd = w.cuda()
    q, s = wq.wq_quantize_int8(wd, g)
    torch.cuda.synchronize()
    codes, so, sb = oracle_q8(w, gg)
    assert np.array_equal(q.cpu().numpy(), codes)
    assert np.array_equal(bits(s), sb)


def test_quantize_int8_gran_per_channel_fp32():
    w = wq_inputs.block_outlier_weight(8192, 8192, wq_inputs.SEEDS["gran"], dtype=torch.float32)
    q, s = wq.wq_quantize_int8(w.cuda())
    torch.cuda.synchronize()
    codes, so, sb = oracle_q8(w, 8192)
    assert np.array_equal(q.cpu().numpy(), codes)
    assert np.array_equal(bits(s), sb)


@pytest.mark.parametrize("N,K,ldw,dtype", [(64, 28672, 28672, torch.bfloat16), (32, 16384, 16384, torch.float32),
                                            (16, 65536, 65536, torch.bfloat16), (5, 8224, 8232, torch.bfloat16),
                                            (3, 96, 104, torch.float32)])
def test_quantize_int8_per_channel_row_lengths(N, K, ldw, dtype):
    """Per output channel: rows held in registers (4 or 8 chunks of 8 per thread), rows too long for that
    (two passes), a ragged last chunk row and a padded leading dimension."""
    base = wq_inputs.block_outlier_weight(N, ldw, 41 + N, dtype=dtype)
    q, s = wq.wq_quantize_int8(base.cuda()[:, :K])  # a column slice: leading dimension ldw
    torch.cuda.synchronize()
    codes, so, sb = oracle_q8(base[:, :K].contiguous(), K)
    assert np.array_equal(q.cpu().numpy(), codes)
    assert np.array_equal(bits(s), sb)


def test_quantize_padded_rows_and_odd_sizes():
    # ldw > K (a column slice of a wider matrix), N = 1 and N not a multiple of anything
    for N, K, ldw in ((1, 32, 32), (7, 96, 104), (129, 4096 + 128, 4352), (3, 288, 296)):
        base = wq_inputs.llm_weight(N, ldw, 70 + N, dtype=torch.float32)
        wd = base.cuda()[:, :K]
        g = 32
        q, s, z = wq.wq_quantize_int4(wd, g)
        q8, s8 = wq.wq_quantize_int8(wd, g)
        torch.cuda.synchronize()
        _, _, _, packed, sb, zb = oracle_q4(base[:, :K].contiguous(), g)
        assert np.array_equal(q.cpu().numpy(), packed) and np.array_equal(bits(s), sb) and np.array_equal(bits(z), zb)
        c8, _, s8b = oracle_q8(base[:, :K].contiguous(), g)
        assert np.array_equal(q8.cpu().numpy(), c8) and np.array_equal(bits(s8), s8b)


def test_quantize_degenerate_and_one_signed_groups():
    w = wq_inputs.llm_weight(64, 512, 81, dtype=torch.float32)
    w[0] = 0.0                    # all-zero row
    w[1, :128] = 0.25             # constant group
    w[2, 128:256] = -3.0
    w[3] = w[3].abs() + 0.01      # one-signed row
    w[4, :128] = 1e-30            # tiny constant group
    w[5, :32] = torch.tensor([0.0, 15.0, 2.5, 3.5, 0.5, 1.5, 14.5, 7.5] * 4)  # exact ties
    w[6] = -w[6].abs() - 5.0      # one-signed, far from zero
    for g in (32, 128):
        check_q4(w, g)
        q8, s8 = wq.wq_quantize_int8(w.cuda(), g)
        torch.cuda.synchronize()
        c8, _, s8b = oracle_q8(w, g)
        assert np.array_equal(q8.cpu().numpy(), c8) and np.array_equal(bits(s8), s8b)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_quantize_extreme_magnitudes(dtype):
    """Rows scaled towards the ends of the binary32 range, subnormal groups and a group mixing a huge and
    tiny values: the quantisers' reciprocal quotients hand these to the IEEE division (scales or
    quotients outside [2^-100, 2^100], ranges outside [2^-90, 2^100]); codes and parameters stay
    bit-exact either way."""
    w = wq_inputs.llm_weight(48, 512, 83, dtype=torch.float32)
    for i, e in enumerate((-140, -130, -120, -110, -100, -92, -88, 88, 96, 100, 104, 110, 120, 124)):
        w[i] *= 2.0 ** e
    w[16, :128] = 1e-40                       # subnormal constant group
    w[17, :64] = 2.0 ** -135                  # smallest subnormals
    w[17, 64:128] = -(2.0 ** -140)
    w[18, :128] = w[18, :128] * 1e-38         # a group of subnormals and tiny normals
    w[19, :128] = 1e-3
    w[19, 5] = 1e30                           # one huge value in a small group
    w[20, 128:256] = -1e30
    w[20, 130] = 3e30
    w[21] = w[21].abs() * 2.0 ** 100 + 2.0 ** 110   # one-signed, huge offset
    w = w.to(dtype)
    for g in (32, 128):
        check_q4(w, g)
        q8, s8 = wq.wq_quantize_int8(w.cuda(), g)
        torch.cuda.synchronize()
        c8, _, s8b = oracle_q8(w, g)
        assert np.array_equal(q8.cpu().numpy(), c8) and np.array_equal(bits(s8), s8b)
    q8, s8 = wq.wq_quantize_int8(w.cuda(), None)  # per output channel
    torch.cuda.synchronize()
    c8, _, s8b = oracle_q8(w, 512)
    assert np.array_equal(q8.cpu().numpy(), c8) and np.array_equal(bits(s8), s8b)


@pytest.mark.parametrize("g", [32, 128])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_quantize_int4_column_scaled(g, dtype):
    """The weight side of activation-aware scaling: the codes of w[n][k] * s_k are those the oracle gets
    for the same binary32 products, bit for bit; scales from activations with salient channels."""
    from oracle import awq
    N, K = 200, 1024
    w = wq_inputs.llm_weight(N, K, 150 + g, dtype=torch.float32).to(dtype)
    x_cal = wq_inputs.activations(32, K, 151, channel_seed=150 + g).double().numpy()
    sc = awq.channel_scales(awq.channel_magnitude(x_cal), 0.5)
    q, s, z = wq.wq_quantize_int4_scaled(w.cuda(), torch.from_numpy(sc).cuda(), g)
    torch.cuda.synchronize()
    codes, so, zo = oracle.quantize_int4(awq.scaled_weights(w_f32(w), sc), g)
    assert np.array_equal(q.cpu().numpy(), oracle.pack_int4(codes))
    assert np.array_equal(bits(s), oracle.bf16_bits(so)) and np.array_equal(bits(z), oracle.bf16_bits(zo))


def check_q4_sym(w: torch.Tensor, g: int):
    q, s, z = wq.wq_quantize_int4_sym(w.cuda(), g)
    torch.cuda.synchronize()
    codes, so = oracle.quantize_int4_sym(w_f32(w), g)
    assert np.array_equal(q.cpu().numpy(), oracle.pack_int4(codes)), "packed symmetric codes differ"
    assert np.array_equal(bits(s), oracle.bf16_bits(so)), "symmetric scales differ"
    assert np.all(bits(z) == oracle.bf16_bits(np.float32(8.0))), "zero-points are not all 8"
    return q, s, z, (codes, so)


def _sym_weights(N, K, seed, dtype=torch.float32):
    w = wq_inputs.llm_weight(N, K, seed, dtype=torch.float32)
    w[0] = 0.0                                            # all-zero row: s = 1, codes 8
    w[1, :128] = -0.25                                    # constant group: -7
    w[2, :8] = torch.tensor([7.0, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.5])  # s = 1 with g = 8 .. ties
    w[3, 5] = -30.0                                       # one 30x outlier channel
    w[4] = w[4].abs() + 0.5                               # one-signed row
    return w.to(dtype)


@pytest.mark.parametrize("g", [32, 64, 128])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_quantize_int4_sym(g, dtype):
    check_q4_sym(_sym_weights(300, 1024, 120 + g, dtype), g)


def test_quantize_int4_sym_padded_and_extreme():
    base = wq_inputs.llm_weight(40, 520, 131, dtype=torch.float32)
    for i, e in enumerate((-140, -120, -100, -90, 90, 100, 110, 124)):
        base[i] *= 2.0 ** e
    base[9, :64] = 1e-40
    base[10, 3] = 1e30
    # a column slice of a wider matrix (ldw = 520 > K = 512)
    q, s, z = wq.wq_quantize_int4_sym(base.cuda()[:, :512], 64)
    torch.cuda.synchronize()
    codes, so = oracle.quantize_int4_sym(base[:, :512].contiguous().numpy(), 64)
    assert np.array_equal(q.cpu().numpy(), oracle.pack_int4(codes)) and np.array_equal(bits(s), oracle.bf16_bits(so))


@pytest.mark.parametrize("M", [1, 2, 8, 40, 128])
def test_gemm_w4a16_on_symmetric_codes(M):
    """Symmetric codes go through the W4A16 matmul unchanged (zero-point 8): within the bound of the
    oracle's s * q decode."""
    N, K, g = 640, 2048, 128
    w = _sym_weights(N, K, 140)
    x = wq_inputs.activations(M, K, 141 + M)
    q, s, z, (codes, so) = check_q4_sym(w, g)
    y = wq.wq_gemm_w4a16(x.cuda(), q, s, z, g)
    torch.cuda.synchronize()
    y_ref, a_ref = oracle.gemm_w4a16(x.double().numpy(), codes, so, np.full(so.shape, 8.0, np.float32), g)
    check_y(y.cpu(), y_ref, a_ref)


def test_quantize_worked_example_on_gpu():
    # the page's 8-weight group, replicated into one 32-wide group of a row
    v = torch.tensor([0.31, -0.12, 0.78, -0.05, 1.42, -0.91, 0.23, 0.66], dtype=torch.float32)
    w = v.repeat(1, 4)
    q, s, z = wq.wq_quantize_int4(w.cuda(), 32)
    torch.cuda.synchronize()
    codes = oracle.unpack_int4(q.cpu().numpy(), 32)[0]
    assert codes[:8].tolist() == [8, 5, 11, 6, 15, 0, 7, 10]
    assert bits(z)[0, 0] == oracle.bf16_bits(np.float32(6.0))


def test_quantize_does_not_write_outside_outputs():
    N, K, g = 37, 256, 64
    w = wq_inputs.llm_weight(N, K, 91).cuda()
    pad = 4096
    canary = 0x5A
    qb = torch.full((N * K // 2 + 2 * pad,), canary, dtype=torch.uint8, device="cuda")
    sb = torch.full((N * K // g + 2 * pad,), 12345, dtype=torch.int16, device="cuda")
    zb = torch.full((N * K // g + 2 * pad,), 12345, dtype=torch.int16, device="cuda")
    q = qb[pad:pad + N * K // 2].view(N, K // 2)
    s = sb[pad:pad + N * K // g].view(torch.bfloat16).view(N, K // g)
    z = zb[pad:pad + N * K // g].view(torch.bfloat16).view(N, K // g)
    wq.wq_quantize_int4(w, g, q, s, z)
    torch.cuda.synchronize()
    assert bool((qb[:pad] == canary).all()) and bool((qb[-pad:] == canary).all())
    assert bool((sb[:pad] == 12345).all()) and bool((sb[-pad:] == 12345).all())
    assert bool((zb[:pad] == 12345).all()) and bool((zb[-pad:] == 12345).all())


def test_errors_with_real_tensors():
    w = torch.zeros(4, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(wq.WQError) as e:
        wq.wq_quantize_int4(w, 48)
    assert e.value.status == wq.WQ_ERR_UNSUPPORTED
    buf = torch.zeros(4 * 256 + 8, dtype=torch.bfloat16, device="cuda")
    wmis = buf[1:1 + 4 * 256].view(4, 256)  # 2-byte offset
    with pytest.raises(wq.WQError) as e:
        wq.wq_quantize_int4(wmis, 128)
    assert e.value.status == wq.WQ_ERR_ALIGN


# ---------------------------------------------------------------------------
# Matmul, within 4e-3 * sum|x * w_hat|
# ---------------------------------------------------------------------------

def _w4_case(N, K, g, M, seed, wgen=None, xgen=None):
    w = wq_inputs.llm_weight(N, K, seed) if wgen is None else wgen
    x = wq_inputs.activations(M, K, seed) if xgen is None else xgen
    q, s, z, (codes, so, zo) = check_q4(w, g)
    y = wq.wq_gemm_w4a16(x.cuda(), q, s, z, g)
    torch.cuda.synchronize()
    y_ref, a_ref = oracle.gemm_w4a16(x.double().numpy(), codes, so, zo, g)
    return check_y(y.cpu(), y_ref, a_ref)


def test_gemm_w4a16_tiny():
    w = wq_inputs.tiny_weight()
    x = wq_inputs.plain_activations(1, 256, 0)
    _w4_case(512, 256, 128, 1, 0, wgen=w, xgen=x)


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 7, 8, 9, 15, 16, 17, 31, 32, 33, 64, 127, 128, 129])
def test_gemm_w4a16_batch_sizes(M):
    _w4_case(1000, 512, 128, M, 100 + M)


@pytest.mark.parametrize("M,N,K,g", [(32, 128, 128, 128), (17, 256, 256, 64), (64, 384, 1024, 32),
                                     (128, 130, 384, 128), (200, 512, 640, 128), (256, 128, 128, 32),
                                     (255, 384, 512, 64)])
def test_gemm_w4a16_tensor_core_tiles(M, N, K, g):
    """Shapes around the tcgen05 kernel's tile edges: one tile, ragged N, several M tiles, split K."""
    _w4_case(N, K, g, M, 17 * M + N)


@pytest.mark.parametrize("M,N,K", [(17, 384, 2048), (32, 1000, 1024), (40, 128, 3072), (64, 700, 1024),
                                   (65, 1000, 1024), (127, 300, 2048), (128, 128, 1024), (129, 640, 3072),
                                   (200, 1000, 8192), (256, 257, 1024), (384, 384, 2048)])
def test_gemm_w4a16_tensor_core_split_roles(M, N, K):
    """The 128 x 128-tile form (g = 128, K a multiple of 1024, every M > 16) with dequantisation and
    promotion in separate warps and the scales and zero-points in shared-memory windows: one and several M
    tiles, M well below the tile, ragged N and M, K ranges whose windows start mid-way through a CTA's
    share."""
    _w4_case(N, K, 128, M, 31 * M + N + K)


@pytest.mark.parametrize("M", [65, 128, 200])
def test_gemm_w4a16_split_roles_zero_rows_and_far_zero_points(M):
    N, K = 640, 2048
    w = wq_inputs.llm_weight(N, K, 96, dtype=torch.float32)
    w[::7] = 0.0
    _w4_case(N, K, 128, M, 0, wgen=w, xgen=wq_inputs.wide_range_activations(M, K, 97 + M))
    _w4_case(N, K, 128, M, 0, wgen=wq_inputs.offset_group_weight(N, K, 98),
             xgen=wq_inputs.positive_activations(M, K, 99 + M))


@pytest.mark.parametrize("N,K,g", [(1, 32, 32), (7, 64, 32), (129, 128, 64), (300, 1024, 128), (33, 4096, 32)])
@pytest.mark.parametrize("M", [1, 4, 16, 40])
def test_gemm_w4a16_shapes(N, K, g, M):
    _w4_case(N, K, g, M, 7 * N + K + M)


@pytest.mark.parametrize("N,K", [(1, 1024), (33, 1024), (31, 3072), (64, 32768), (4097, 2048), (8192, 8192),
                                 (100, 65536), (4097, 1152), (65536, 1024), (40000, 2048)])
def test_gemm_w4a16_m1_stream_k_edges(N, K):
    """M = 1, group 128: a single row, ragged row blocks, the largest K of the TMA kernel, more warps than
    units, CTAs whose range holds whole tiles between two split ones (the last two); and two shapes it does
    not take (K > 32768, K not a multiple of 1024)."""
    _w4_case(N, K, 128, 1, 11 * N + K)


@pytest.mark.parametrize("g", [32, 64])
@pytest.mark.parametrize("N,K", [(1, 1024), (33, 1024), (31, 3072), (4097, 2048), (3000, 4096), (65536, 1024),
                                 (40000, 2048), (64, 31744), (64, 32768)])
def test_gemm_w4a16_m1_small_groups(N, K, g):
    """M = 1 with groups of 32 and 64 on the decode kernel: each 128-input block holds 4 or 2 groups, whose
    digit sums the MMA keeps in separate columns; ragged row blocks, tiles split over CTAs, CTAs with whole
    tiles between split ones, the longest K each group size takes (groups of 32 at K = 32768 do not fit
    shared memory and go to the CUDA-core kernel)."""
    _w4_case(N, K, g, 1, 19 * N + K + g)


@pytest.mark.parametrize("g", [32, 64])
def test_gemm_w4a16_m1_small_groups_exact_zeros_far_zero_points_nonfinite(g):
    """Groups of 32 and 64 at M = 1: all-zero rows and a single all-zero group give exactly 0 under
    activations spanning many binades; zero-points far outside [0, 15] with one-signed activations meet the
    bound; an infinite activation makes every output non-finite."""
    N, K = 640, 2048
    w = wq_inputs.llm_weight(N, K, 191, dtype=torch.float32)
    w[::5] = 0.0
    w[3, 256:256 + g] = 0.0
    _w4_case(N, K, g, 1, 0, wgen=w, xgen=wq_inputs.wide_range_activations(1, K, 192 + g))
    _w4_case(N, K, g, 1, 0, wgen=wq_inputs.offset_group_weight(N, K, 193, group=g),
             xgen=wq_inputs.positive_activations(1, K, 194 + g))
    x = wq_inputs.activations(1, K, 195)
    x[:, 300] = float("inf")
    q, s, z = wq.wq_quantize_int4(w.cuda(), g)
    y = wq.wq_gemm_w4a16(x.cuda(), q, s, z, g)
    torch.cuda.synchronize()
    assert not torch.isfinite(y.float()).any()


@pytest.mark.parametrize("M,N,K", [(1, 3000, 4096), (2, 3000, 4096), (8, 3000, 4096), (16, 1000, 8192),
                                   (128, 256, 16384), (40, 384, 8192)])
def test_gemm_w4a16_workspace_reuse_deterministic(M, N, K):
    """Calls that share one workspace find it ready (its counters re-zeroed by the previous call) and the
    split-K combine runs in a fixed order: the same inputs give the same bytes every time.  M = 1 runs the
    persistent decode kernel, M = 2 and 8 its small-batch forms, M = 16, 40 and 128 the tensor-core kernel
    with K split over many CTAs per tile."""
    w = wq_inputs.llm_weight(N, K, 77)
    q, s, z = wq.wq_quantize_int4(w.cuda(), 128)
    ws = torch.zeros(wq.wq_gemm_workspace_bytes(M, N, K, 128, 4) + 16, dtype=torch.uint8, device="cuda")
    outs = []
    for seed in (1, 2, 1, 2, 1):
        x = wq_inputs.activations(M, K, seed).cuda()
        outs.append(wq.wq_gemm_w4a16(x, q, s, z, 128, workspace=ws).clone())
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[2]) and torch.equal(outs[0], outs[4])
    assert torch.equal(outs[1], outs[3])
    assert not torch.equal(outs[0], outs[1])


@pytest.mark.parametrize("M,N,K", [(2, 1, 1024), (3, 300, 1024), (8, 4097, 2048), (16, 4097, 2048),
                                   (9, 40000, 2048), (12, 256, 32768), (5, 8192, 8192), (7, 33, 3072)])
def test_gemm_w4a16_small_batch_persistent(M, N, K):
    """2 <= M <= 16, group 128, K % 1024 = 0: the persistent small-batch kernel with the M rows as the
    MMA's columns (8 or 16), a single row, ragged row blocks, tiles split over several CTAs, CTAs holding
    whole tiles, the longest K, a 2-row-short column tile."""
    _w4_case(N, K, 128, M, 13 * N + K + M)


@pytest.mark.parametrize("M,N,K", [(13, 1000, 8192), (16, 4097, 2048), (9, 2000, 28672), (12, 3000, 4096),
                                   (16, 128, 1024), (14, 300, 32768)])
def test_gemm_w4a16_small_batch_on_tensor_cores(M, N, K):
    """9 to 16 rows, g = 128, K % 1024 = 0: the 128 x 128-tile tensor-core kernel takes the shapes where the
    persistent small-batch kernel would run with fewer than three stages or more than 12 rows; its tile holds
    the M rows and zeros (the activation copies fill rows past M)."""
    _w4_case(N, K, 128, M, 23 * M + N + K)


@pytest.mark.parametrize("M", [8, 16])
def test_gemm_w4a16_small_batch_large_shape(M):
    """The gate+up shape at M = 8 (the persistent kernel with two weight stages, its activations filling
    shared memory) and M = 16 (too many activations for it: the tensor-core kernel); rows sampled."""
    N, K = 57344, 8192
    w = wq_inputs.llm_weight(N, K, 333)
    rows = np.r_[0:64, 20000:20064, N - 64:N]
    _sampled_w4(N, K, 128, (M,), 334, w, rows)  # asserts the bound on every sampled output


@pytest.mark.parametrize("M", [1, 2, 4, 128])
def test_gemm_nonfinite_activation_propagates(M):
    """An infinite activation makes every output non-finite (x_k * w_hat_nk is +-inf, or NaN where
    w_hat_nk = 0), on every kernel; the M = 1 kernels carry it through their digit planes as a NaN factor."""
    N, K = 512, 2048
    w = wq_inputs.llm_weight(N, K, 51)
    x = wq_inputs.activations(M, K, 52)
    x[:, 300] = float("inf")
    q, s, z = wq.wq_quantize_int4(w.cuda(), 128)
    y = wq.wq_gemm_w4a16(x.cuda(), q, s, z, 128)
    q8, s8 = wq.wq_quantize_int8(w.cuda(), None)
    y8 = wq.wq_gemm_w8a16(x.cuda(), q8, s8, None)
    torch.cuda.synchronize()
    assert not torch.isfinite(y.float()).any()
    assert not torch.isfinite(y8.float()).any()


@pytest.mark.parametrize("M", [1, 2, 5, 8, 16, 17, 40])
def test_gemm_w4a16_zero_rows_exact(M):
    """Rows (and groups) whose weights are all zero have w_hat = 0, so the bound is 0: y must be exactly 0,
    even when the activations of a group span so many binades that their binary32 sums round."""
    N, K = 640, 2048
    w = wq_inputs.llm_weight(N, K, 91, dtype=torch.float32)
    w[::5] = 0.0
    w[3, 256:384] = 0.0  # one all-zero group inside a non-zero row
    x = wq_inputs.wide_range_activations(M, K, 92 + M)
    _w4_case(N, K, 128, M, 0, wgen=w, xgen=x)


@pytest.mark.parametrize("M", [1, 2, 5, 8, 16, 17, 40, 128])
def test_gemm_w4a16_far_zero_points(M):
    """Groups on one side of zero, far from it compared with their width, get zero-points far outside
    [0, 15] (z = round(-min / s) is not clamped), where neither 128 + z nor q - z need fit bf16's 8
    significant bits.  With activations of one sign no rounding error cancels: every kernel must still
    meet the bound (M = 1, 2..16 and > 16 each take their own kernel)."""
    N, K = 640, 2048
    w = wq_inputs.offset_group_weight(N, K, 93)
    x = wq_inputs.positive_activations(M, K, 94 + M)
    _w4_case(N, K, 128, M, 0, wgen=w, xgen=x)


@pytest.mark.parametrize("g,M,K", [(32, 1, 1024), (64, 4, 1024), (128, 1, 1152), (32, 40, 1024), (64, 64, 1024)])
def test_gemm_w4a16_far_zero_points_other_kernels(g, M, K):
    """The same for the decode kernel with groups of 32, the small-batch CUDA-core kernel (groups of 64), the
    M = 1 CUDA-core kernel (K that the TMA kernels do not take) and the tensor-core kernel with several groups
    per stage."""
    N = 384
    w = wq_inputs.offset_group_weight(N, K, 95 + g, group=g)
    x = wq_inputs.positive_activations(M, K, 96 + M)
    _w4_case(N, K, g, M, 0, wgen=w, xgen=x)


def test_gemm_w4a16_degenerate_groups():
    w = wq_inputs.llm_weight(64, 512, 81, dtype=torch.float32)
    w[0] = 0.0
    w[1, :128] = 0.25
    w[3] = w[3].abs() + 0.01
    w[6] = -w[6].abs() - 5.0
    for M in (1, 8, 48):
        _w4_case(64, 512, 128, M, 5, wgen=w)


def _sampled_w4(N, K, g, Ms, seed, wgen, rows):
    q, s, z, (codes, so, zo) = check_q4(wgen, g, rows=rows)
    ratios = []
    for M in Ms:
        x = wq_inputs.activations(M, K, seed + M)
        y = wq.wq_gemm_w4a16(x.cuda(), q, s, z, g)
        torch.cuda.synchronize()
        y_ref, a_ref = oracle.gemm_w4a16(x.double().numpy(), codes, so, zo, g)
        ratios.append(check_y(y.cpu()[:, rows], y_ref, a_ref))
    return ratios


def test_gemm_w4a16_decode_up_m1():
    w = wq_inputs.llm_weight(14336, 4096, wq_inputs.SEEDS["decode_up"])
    _sampled_w4(14336, 4096, 128, [1], 2, w, sample_rows(14336, 256, 2))


def test_gemm_w4a16_sweep_sampled():
    w = wq_inputs.llm_weight(28672, 8192, wq_inputs.SEEDS["sweep"])
    _sampled_w4(28672, 8192, 128, [1, 8, 16, 32, 128], 3, w, sample_rows(28672, 192, 3))


def test_gemm_w4a16_gran_g32():
    w = wq_inputs.block_outlier_weight(8192, 8192, wq_inputs.SEEDS["gran"])
    _sampled_w4(8192, 8192, 32, [1, 16], 4, w, sample_rows(8192, 192, 4))


def _w8_case(w, x, g, rows=None):
    K = w.shape[1]
    gg = K if g is None else g
    q, s = wq.wq_quantize_int8(w.cuda(), g)
    y = wq.wq_gemm_w8a16(x.cuda(), q, s, g)
    torch.cuda.synchronize()
    sel = slice(None) if rows is None else rows
    codes, so, sb = oracle_q8(w[sel], gg)
    assert np.array_equal(q.cpu().numpy()[sel], codes) and np.array_equal(bits(s)[sel], sb)
    y_ref, a_ref = oracle.gemm_w8a16(x.double().numpy(), codes, so, gg)
    return check_y(y.cpu()[:, sel], y_ref, a_ref)


@pytest.mark.parametrize("M", [1, 2, 5, 16, 17, 64, 128])
@pytest.mark.parametrize("g", [None, 32, 64, 128])
def test_gemm_w8a16(M, g):
    w = wq_inputs.block_outlier_weight(600, 1024, 200 + M)
    x = wq_inputs.activations(M, 1024, 300 + M)
    _w8_case(w, x, g)


@pytest.mark.parametrize("M,N,K,g", [
    (4, 100, 1024, 32),     # N < 128: CUDA-core kernel
    (4, 256, 1056, 32),     # K % 128 != 0: CUDA-core kernel
    (130, 300, 384, None),  # two 128-row activation tiles, the second of 2 rows; ragged N
    (40, 128, 128, 128),    # one stage, one weight tile
    (3, 1000, 2048, 64),    # many K-splits of a few tiles
])
def test_gemm_w8a16_kernel_boundaries(M, N, K, g):
    w = wq_inputs.block_outlier_weight(N, K, 17 * M + N)
    x = wq_inputs.activations(M, K, 19 * M + K)
    _w8_case(w, x, g)


def test_gemm_w8a16_repeatable_and_zero_rows():
    """The tensor-core W8A16 path combines K-splits in a fixed order (identical bytes on repeat); rows of
    zero weights give exactly zero."""
    w = wq_inputs.block_outlier_weight(512, 4096, 23)
    w[7] = 0.0
    w[300] = 0.0
    x = wq_inputs.activations(16, 4096, 29).cuda()
    q, s = wq.wq_quantize_int8(w.cuda(), 128)
    y1 = wq.wq_gemm_w8a16(x, q, s, 128)
    y2 = wq.wq_gemm_w8a16(x, q, s, 128)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    assert not y1[:, 7].any() and not y1[:, 300].any()


@pytest.mark.parametrize("N,K", [(1, 128), (33, 256), (4097, 1152), (300, 28672), (65536, 1024), (100, 65536),
                                 (1000, 8192)])
def test_gemm_w8a16_m1_per_channel_shapes(N, K):
    """M = 1, per output channel: the persistent integer kernel (one row, ragged row blocks, K not a multiple
    of 1024, CTAs holding whole tiles, the longest K)."""
    w = wq_inputs.block_outlier_weight(N, K, 31 * N + K)
    x = wq_inputs.activations(1, K, 37 * N + K)
    _w8_case(w, x, None)


@pytest.mark.parametrize("M,N,K", [(2, 1, 128), (3, 300, 1152), (4, 4097, 2048), (8, 1000, 8192), (9, 257, 4096),
                                   (16, 8192, 8192), (16, 40000, 1024)])
def test_gemm_w8a16_small_batch_per_channel(M, N, K):
    """2 <= M <= 16, per output channel: the persistent integer kernel with M rows x 4 digits in the MMA's
    B columns (1, 2 or 4 column tiles, M <= 8), or, at M > 8 and where its digit planes do not fit, the
    tensor-core kernel."""
    w = wq_inputs.block_outlier_weight(N, K, 53 * N + K + M)
    x = wq_inputs.activations(M, K, 59 * N + K + M)
    _w8_case(w, x, None, rows=None if N * K <= 8192 * 1024 else sample_rows(N, 256, M))


def test_gemm_w8a16_m1_exact_zero_rows_and_repeatable():
    """M = 1, per output channel: rows of zero weights give exactly zero even for activations spanning many
    binades, and the split-K combine runs in a fixed order (identical bytes on repeat)."""
    N, K = 640, 2048
    w = wq_inputs.block_outlier_weight(N, K, 43)
    w[::5] = 0.0
    x = wq_inputs.wide_range_activations(1, K, 47)
    _w8_case(w, x, None)
    q, s = wq.wq_quantize_int8(w.cuda(), None)
    xd = x.cuda()
    y1 = wq.wq_gemm_w8a16(xd, q, s, None)
    y2 = wq.wq_gemm_w8a16(xd, q, s, None)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    assert not y1[:, ::5].any()


def test_gemm_w8a16_gran_per_channel():
    w = wq_inputs.block_outlier_weight(8192, 8192, wq_inputs.SEEDS["gran"])
    rows = sample_rows(8192, 192, 5)
    for M in (1, 16):
        _w8_case(w, wq_inputs.activations(M, 8192, 4 + M), None, rows=rows)


def test_full70b_layer_shapes_sampled():
    """One layer of the 70B-shaped step, generated on the GPU like the benchmark, sampled rows checked."""
    layer = 0
    for j, (name, K, N) in enumerate(wq_inputs.FULL70B_LINEARS):
        seed = wq_inputs.full70b_seed(layer, j)
        wd = wq_inputs.llm_weight(N, K, seed, outlier_frac=0.0, device="cuda")
        rows = sample_rows(N, 64, seed)
        q, s, z = wq.wq_quantize_int4(wd, 128)
        wrows = wd[torch.as_tensor(rows, device="cuda")].cpu()
        codes, so, zo, packed, sb, zb = oracle_q4(wrows, 128)
        assert np.array_equal(q.cpu().numpy()[rows], packed)
        assert np.array_equal(bits(s)[rows], sb) and np.array_equal(bits(z)[rows], zb)
        for M in (1, 128):
            x = wq_inputs.plain_activations(M, K, seed, device="cuda")
            y = wq.wq_gemm_w4a16(x, q, s, z, 128)
            torch.cuda.synchronize()
            y_ref, a_ref = oracle.gemm_w4a16(x.double().cpu().numpy(), codes, so, zo, 128)
            check_y(y.cpu()[:, rows], y_ref, a_ref)
        del wd, q, s, z
        torch.cuda.empty_cache()


def test_gemm_output_offsets_and_canaries():
    N, K, M = 100, 256, 3
    w = wq_inputs.llm_weight(N, K, 11)
    q, s, z, (codes, so, zo) = check_q4(w, 64)
    x = wq_inputs.activations(M, K, 12).cuda()
    pad = 2048
    yb = torch.full((M * N + 2 * pad,), -7, dtype=torch.int16, device="cuda")
    y = yb[pad:pad + M * N].view(torch.bfloat16).view(M, N)
    wq.wq_gemm_w4a16(x, q, s, z, 64, y=y)
    torch.cuda.synchronize()
    assert bool((yb[:pad] == -7).all()) and bool((yb[-pad:] == -7).all())
    y_ref, a_ref = oracle.gemm_w4a16(x.double().cpu().numpy(), codes, so, zo, 64)
    check_y(y.cpu(), y_ref, a_ref)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_quantize_ragged_last_chunk(dtype):
    """K not a multiple of 256: a warp's last 256-weight chunk of a row runs past K, and the lanes beyond K
    must sit out of the group reductions (for bf16 input the asymmetric quantiser carries min and -max as
    one packed pair).  Every quantiser, both input types; K = 128 with g = 128 is one group per row, the
    layout of a KV cache quantised in blocks of 128."""
    for N, K, g in ((7, 96, 32), (5, 128, 128), (9, 128, 64), (3, 288, 32), (4, 640, 128)):
        w = wq_inputs.llm_weight(N, K, 90 + K + g, dtype=torch.float32).to(dtype)
        check_q4(w, g)
        check_q4_sym(w, g)
        q8, s8 = wq.wq_quantize_int8(w.cuda(), g)
        torch.cuda.synchronize()
        c8, _, s8b = oracle_q8(w, g)
        assert np.array_equal(q8.cpu().numpy(), c8) and np.array_equal(bits(s8), s8b)

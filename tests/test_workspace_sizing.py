"""The workspace size the library asks for covers every slot its split-K kernels index (CPU only).

The persistent decode kernel (M = 1) and the tensor-core kernel (M > 16) split tiles between CTAs with
equal contiguous ranges of units (stream-K); each segment of a split tile writes a binary32 partial into
slot (CTA - first CTA of the tile), and each tile has an arrival counter.  This test models those ranges
for many shapes, finds the largest number of segments any tile really has, and checks that
wq_gemm_workspace_bytes (queried without a GPU; the library then assumes a B200's 148 SMs) leaves room for
all of them.
"""
import math

import pytest

import group_wise_weight_b200 as wq

SMS = 148


def _m1_needed(N, K):
    P = K // 256                      # group pairs per 256-row tile
    ntiles = math.ceil(N / 256)
    units = ntiles * P
    B = min(units, SMS)
    cta_of = lambda u: ((u + 1) * B - 1) // units  # noqa: E731
    for b in (0, B // 2, B - 1):      # the formula agrees with the ranges [units b / B, units (b+1) / B)
        lo, hi = units * b // B, units * (b + 1) // B
        assert all(cta_of(u) == b for u in range(lo, hi))
    max_seg = max(cta_of(t * P + P - 1) - cta_of(t * P) + 1 for t in range(ntiles))
    return ntiles * max_seg * 256 * 4 + ntiles * 4


def _mt_stages(M, N, K):
    """Weight stages of the persistent small-batch kernel (2 <= M <= 16, g = 128) as the library decides it
    for a B200: 3 or 2 when the CTA's activation pairs fit shared memory beside them, else 0."""
    P = K // 256
    units = math.ceil(N / 256) * P
    npairs = min(-(-units // min(units, SMS)), P)

    def total(stages):
        return stages * 32768 + 16384 + 2 * M * 256 * 4 + npairs * 2 * M * 256 + 16 * 8 + 1024

    return 3 if total(3) <= 232448 else 2 if total(2) <= 232448 else 0


def _tc_takes_small_batch(M, N, K):
    """9 <= M <= 16, g = 128, K % 1024 == 0, N >= 128: the 128 x 128-tile tensor-core kernel, unless M <= 12 and
    the persistent small-batch kernel runs with three stages."""
    return 9 <= M <= 16 and N >= 128 and K % 1024 == 0 and not (M <= 12 and _mt_stages(M, N, K) == 3)


def _mt_needed(M, N, K):
    """2 <= M <= 16, g = 128: the persistent kernel's [segment][m][256] slots when the CTA's activation pairs
    fit shared memory (as the library decides it for a B200), else the older kernel's M x N binary32 buffer."""
    P = K // 256
    ntiles = math.ceil(N / 256)
    units = ntiles * P
    B = min(units, SMS)
    if _mt_stages(M, N, K) == 0:
        return M * N * 4
    cta_of = lambda u: ((u + 1) * B - 1) // units  # noqa: E731
    max_seg = max(cta_of(t * P + P - 1) - cta_of(t * P) + 1 for t in range(ntiles))
    return ntiles * max_seg * M * 256 * 4 + ntiles * 4


def _tc_needed(M, N, K, g):
    # g = 128 with K a multiple of 1024 runs the split-role kernel: 128-row activation tiles for every M
    BN = 128 if (g == 128 and K % 1024 == 0) else min(32 if M <= 32 else (64 if M <= 64 else 128), g)
    tiles = math.ceil(N / 128) * math.ceil(M / BN)
    spt = K // 128
    total = tiles * spt
    grid = max(1, min(total, SMS))
    per, extra = total // grid, total % grid
    big = extra * (per + 1)
    cta_of = lambda u: u // (per + 1) if u < big else extra + (u - big) // per  # noqa: E731
    max_seg = max(cta_of(t * spt + spt - 1) - cta_of(t * spt) + 1 for t in range(tiles))
    return tiles * max_seg * BN * 128 * 4 + tiles * 4


@pytest.fixture(scope="module", autouse=True)
def _lib():
    wq.lib()


@pytest.mark.parametrize("N,K", [(1, 1024), (33, 1024), (31, 3072), (64, 32768), (4097, 2048), (3000, 4096),
                                 (8192, 8192), (10240, 8192), (57344, 8192), (8192, 28672), (14336, 4096),
                                 (256 * 148, 1024), (256 * 149 + 1, 2048), (300000, 1024)])
@pytest.mark.parametrize("g", [128, 64, 32])
def test_m1_workspace_covers_every_segment(N, K, g):
    if g == 32 and K > 31744:
        pytest.skip("groups of 32 at K = 32768 do not fit the decode kernel's shared memory")
    assert wq.wq_gemm_workspace_bytes(1, N, K, g, 4) >= _m1_needed(N, K)


@pytest.mark.parametrize("M,N,K,g", [(17, 128, 128, 32), (32, 256, 256, 64), (40, 384, 8192, 128),
                                     (64, 384, 1024, 32), (128, 130, 384, 128), (128, 256, 16384, 128),
                                     (128, 10240, 8192, 128), (128, 57344, 8192, 128), (128, 8192, 28672, 128),
                                     (200, 512, 640, 128), (256, 128, 128, 32), (129, 4097, 4096, 64),
                                     (17, 8192, 8192, 128), (32, 28672, 8192, 128), (64, 57344, 8192, 128),
                                     (24, 1000, 3072, 128)])
def test_tc_workspace_covers_every_segment(M, N, K, g):
    assert wq.wq_gemm_workspace_bytes(M, N, K, g, 4) >= _tc_needed(M, N, K, g)


@pytest.mark.parametrize("M,N,K", [(2, 1, 1024), (3, 4097, 2048), (8, 28672, 8192), (8, 57344, 8192),
                                   (8, 8192, 28672), (16, 10240, 8192), (16, 57344, 8192), (5, 300000, 1024),
                                   (9, 33, 32768), (16, 256 * 149 + 1, 2048), (12, 10240, 8192), (12, 8192, 28672),
                                   (9, 57344, 8192), (13, 8192, 8192), (16, 100, 8192)])
def test_mt_workspace_covers_every_segment(M, N, K):
    """2 <= M <= 16, g = 128: the small-batch kernels' slots, or the tensor-core kernel's where it takes the
    shape (9 to 16 rows)."""
    need = _tc_needed(M, N, K, 128) if _tc_takes_small_batch(M, N, K) else _mt_needed(M, N, K)
    assert wq.wq_gemm_workspace_bytes(M, N, K, 128, 4) >= need


def _w8int_needed(M, N, K):
    """W8A16 per channel, 1 <= M <= 8: the persistent integer kernel's [segment][m][256] slots when a CTA's
    digit planes fit shared memory with two or three stages (as the library decides for a B200); 0 when
    another kernel takes the shape."""
    G = K // 128                      # groups of 128 inputs (units) per 256-row tile
    ntiles = math.ceil(N / 256)
    units = ntiles * G
    B = min(units, SMS)
    nslots = min(-(-units // B), G)
    if M > 8:
        return 0
    NT = 1 if M <= 2 else 2 if M <= 4 else 4

    def total(stages):
        return stages * 32768 + 2 * M * 1024 + nslots * 1024 * NT + nslots * 64 + 14 * 8 + 1024

    if total(3) > 232448 and total(2) > 232448:
        return 0
    cta_of = lambda u: ((u + 1) * B - 1) // units  # noqa: E731
    max_seg = max(cta_of(t * G + G - 1) - cta_of(t * G) + 1 for t in range(ntiles))
    return ntiles * max_seg * M * 256 * 4 + ntiles * 4


@pytest.mark.parametrize("M,N,K", [(1, 1, 128), (1, 33, 256), (1, 4097, 1152), (1, 300, 28672), (1, 65536, 1024),
                                   (1, 100, 65536), (1, 8192, 8192), (1, 57344, 8192), (2, 4097, 2048),
                                   (5, 8192, 8192), (8, 10240, 8192), (16, 8192, 8192), (16, 57344, 8192)])
def test_w8int_workspace_covers_every_segment(M, N, K):
    assert wq.wq_gemm_workspace_bytes(M, N, K, K, 8) >= _w8int_needed(M, N, K)


COUNTER_REGION = 65536


@pytest.mark.parametrize("N,K", [(10240, 8192), (8192, 8192), (57344, 8192), (8192, 28672), (300000, 1024),
                                 (4200000, 1024)])
def test_tile_counters_sit_below_the_partial_sums(N, K):
    """Every kernel that splits tiles keeps its arrival counters in the workspace's first 64 KB (more for a
    shape of over 16,384 tiles) and its partial sums above them, so that one workspace can serve calls of any
    shapes in turn (a call leaves its partial sums behind but re-zeroes its counters).  The size asked for is
    therefore the counter region plus the partial sums: M = 1 INT4, M = 128 INT4 (128 x 128 tiles) and M = 1
    W8A16 per channel."""
    nt256 = math.ceil(N / 256)
    region = max(COUNTER_REGION, math.ceil(nt256 * 4 / COUNTER_REGION) * COUNTER_REGION)
    assert wq.wq_gemm_workspace_bytes(1, N, K, 128, 4) >= region + _m1_needed(N, K) - nt256 * 4
    tiles128 = math.ceil(N / 128)
    region128 = max(COUNTER_REGION, math.ceil(tiles128 * 4 / COUNTER_REGION) * COUNTER_REGION)
    assert wq.wq_gemm_workspace_bytes(128, N, K, 128, 4) >= region128 + _tc_needed(128, N, K, 128) - tiles128 * 4
    w8 = _w8int_needed(1, N, K)
    if w8:
        assert wq.wq_gemm_workspace_bytes(1, N, K, K, 8) >= region + w8 - nt256 * 4

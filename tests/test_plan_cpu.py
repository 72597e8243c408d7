"""The path and tiling policy, through vq_plan_for_device (host arithmetic, no GPU).

These pin what a forward would launch on a B200 (148 SMs, 227 KiB of opt-in shared
memory per block) for the benchmark shapes, the fallbacks on smaller devices and the
argument checks.  The expected plans are the ones vq_linear_plan reports for the same
layers on a B200 (the GPU tests check that query against the launches)."""

import pytest

import compressed_index_matmul_b200 as vq
from synth import DT_BF16, DT_F16, FMT_RVQ12, FMT_RVQ12_4, FMT_VQ16, FMT_VQ16_RVQ

LUT, GEMV, TC, GATHER = vq.VQ_PATH_LUT, vq.VQ_PATH_GEMV, vq.VQ_PATH_TC, vq.VQ_PATH_GATHER
VQ_ERR_INVALID_ARG, VQ_ERR_UNSUPPORTED = 1, 2


@pytest.fixture(scope="module", autouse=True)
def lib():
    vq.load()


def plan(N, K, fmt, M, sg=64, path=0, max_M=1024, act=DT_BF16, **kw):
    return vq.vq_plan_for_device(N, K, fmt, sg, act, max_M, M, path=path, **kw)


def as_tuple(p):
    return (p["path"], p["launches"], p["ctas"], p["splits"])


@pytest.mark.parametrize("N, K, fmt, sg, M, want", [
    # batch 1, 12-bit: the table kernel, one CTA per SM, one K split per 128-input slice
    (14336, 4096, FMT_RVQ12_4, 64, 1, (LUT, 1, 148, 32)),
    (4096, 14336, FMT_RVQ12_4, 64, 1, (LUT, 1, 148, 112)),
    # 12-bit, 16 tokens: two CTAs per SM (296 slots); 112 row tiles -> a K-split pair each
    (14336, 4096, FMT_RVQ12_4, 64, 16, (TC, 1, 224, 2)),
    (14336, 4096, FMT_RVQ12_4, 64, 4, (TC, 1, 224, 2)),
    # 32 row tiles -> 9 slots each, capped at 8 splits of 14 slices
    (4096, 14336, FMT_RVQ12_4, 64, 16, (TC, 1, 256, 8)),
    # 64-token tiles: two CTAs per SM only while the split stays a pair
    (14336, 4096, FMT_RVQ12_4, 64, 64, (TC, 1, 224, 2)),
    (8192, 8192, FMT_RVQ12_4, 64, 64, (TC, 1, 128, 2)),
    # 32-token tiles of 8192 x 8192: 64 tiles, 4 splits over two slots per SM
    (8192, 8192, FMT_RVQ12_4, 64, 32, (TC, 1, 256, 4)),
    # wide tiles: one CTA per SM, 148 / 64 tiles -> 2 splits
    (8192, 8192, FMT_RVQ12_4, 64, 256, (TC, 1, 128, 2)),
    # 1024 tokens: 4 token tiles x 64 row tiles fill the SMs without a split
    (8192, 8192, FMT_RVQ12_4, 64, 1024, (TC, 1, 256, 1)),
    # 16-bit indices: the gather kernel up to 4 tokens (74 clusters of 2), then one
    # tensor-core CTA per SM (148 / 32 tiles -> 4 splits)
    (4096, 4096, FMT_VQ16, 4096, 1, (GATHER, 1, 148, 32)),
    (4096, 4096, FMT_VQ16, 4096, 4, (GATHER, 1, 148, 32)),
    (4096, 4096, FMT_VQ16, 4096, 8, (TC, 1, 128, 4)),
    # small layers (N K < 2^22): the warp-MMA GEMV for 2..16 tokens
    (576, 576, FMT_RVQ12_4, 64, 16, (GEMV, 1, 15, 3)),
    (1536, 576, FMT_RVQ12, 64, 4, (GEMV, 1, 0, 0)),
])
def test_plan_on_b200(N, K, fmt, sg, M, want):
    got = as_tuple(plan(N, K, fmt, M, sg=sg))
    if want[2] == 0:  # only the path is pinned
        assert got[0] == want[0] and got[1] == want[1], got
    else:
        assert got == want, got


def test_ladder_plans_like_the_16_bit_format():
    kw = dict(n16=1, n8=1, mult=(0.25,))
    assert plan(4096, 4096, FMT_VQ16_RVQ, 1, sg=4096, **kw)["path"] == GATHER
    assert as_tuple(plan(4096, 4096, FMT_VQ16_RVQ, 8, sg=4096, **kw)) == (TC, 1, 128, 4)


def test_forced_paths():
    assert plan(14336, 4096, FMT_RVQ12_4, 1, path=TC)["path"] == TC
    assert plan(14336, 4096, FMT_RVQ12_4, 16, path=GEMV)["path"] == GEMV
    with pytest.raises(vq.VQError) as ei:
        plan(14336, 4096, FMT_RVQ12_4, 1, path=GATHER)  # 12-bit indices: no gather kernel
    assert ei.value.status == VQ_ERR_UNSUPPORTED
    with pytest.raises(vq.VQError) as ei:
        plan(14336, 4096, FMT_RVQ12_4, 2, path=LUT)  # the table kernel is batch 1 only
    assert ei.value.status == VQ_ERR_UNSUPPORTED
    with pytest.raises(vq.VQError) as ei:
        plan(14336, 4096, FMT_RVQ12_4, 17, path=GEMV)  # the GEMV takes at most 16 tokens
    assert ei.value.status == VQ_ERR_UNSUPPORTED
    # the gather kernel forced up to 8 tokens, not beyond
    assert plan(4096, 4096, FMT_VQ16, 8, sg=4096, path=GATHER)["path"] == GATHER
    with pytest.raises(vq.VQError):
        plan(4096, 4096, FMT_VQ16, 9, sg=4096, path=GATHER)


def test_correction_adds_a_launch():
    assert plan(14336, 4096, FMT_RVQ12_4, 1, corr=1)["launches"] == 2
    assert plan(14336, 4096, FMT_RVQ12_4, 16, corr=1)["launches"] == 2


def test_smaller_devices():
    # half the SMs: the table kernel follows the SM count; the 16-token gate gets one
    # slot per row tile (148 slots / 112 tiles) and no split
    assert as_tuple(plan(14336, 4096, FMT_RVQ12_4, 1, num_sms=74)) == (LUT, 1, 74, 32)
    assert as_tuple(plan(14336, 4096, FMT_RVQ12_4, 16, num_sms=74)) == (TC, 1, 112, 1)
    # too little shared memory for the table and tensor-core kernels: the GEMV takes
    # batches up to 16, larger ones cannot run
    small = dict(smem_optin=100 * 1024)
    assert plan(14336, 4096, FMT_RVQ12_4, 1, **small)["path"] == GEMV
    assert plan(14336, 4096, FMT_RVQ12_4, 16, **small)["path"] == GEMV
    with pytest.raises(vq.VQError) as ei:
        plan(14336, 4096, FMT_RVQ12_4, 64, **small)
    assert ei.value.status == VQ_ERR_UNSUPPORTED


def test_plan_is_deterministic_and_independent_of_the_activation_type():
    a = [as_tuple(plan(14336, 4096, FMT_RVQ12_4, M)) for M in (1, 2, 16, 17, 64, 256)]
    b = [as_tuple(plan(14336, 4096, FMT_RVQ12_4, M, act=DT_F16)) for M in (1, 2, 16, 17, 64, 256)]
    assert a == b == [as_tuple(plan(14336, 4096, FMT_RVQ12_4, M)) for M in (1, 2, 16, 17, 64, 256)]


@pytest.mark.parametrize("kw, M", [
    (dict(num_sms=0), 1),
    (dict(smem_optin=-1), 1),
    (dict(path=9), 1),
    ({}, 0),
    ({}, 1025),
])
def test_argument_errors(kw, M):
    with pytest.raises(vq.VQError) as ei:
        plan(14336, 4096, FMT_RVQ12_4, M, **kw)
    assert ei.value.status == VQ_ERR_INVALID_ARG


def test_invalid_desc_is_refused():
    with pytest.raises(vq.VQError) as ei:
        plan(4096, 4100, FMT_RVQ12_4, 1)  # K not a multiple of 16
    assert ei.value.status == VQ_ERR_INVALID_ARG

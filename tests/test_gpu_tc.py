"""GPU parity of the tensor-core path (decode to shared memory + tcgen05 MMA) against the oracle."""

import numpy as np
import pytest
import torch

import compressed_index_matmul_b200 as vq
from synth import DT_BF16, DT_F16, FMT_RVQ12, FMT_RVQ12_4, FMT_VQ16, CONFIGS, LayerSpec, make_layer, make_x
from tests.gpu_util import assert_y_within, layer_on_gpu, require_gpu, run_forward, widen

pytestmark = pytest.mark.gpu
TOL = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _check(oracle, layer, act, M, seed=0):
    L = layer_on_gpu(layer, act, M)
    x = make_x(M, layer["spec"].K, act, cfg_id=80, seed=seed)
    y = run_forward(L, x, act, vq.VQ_PATH_TC)
    vq.vq_linear_check(L.handle)
    y_ref = oracle.forward(layer, x, act)
    w, _ = oracle.dequant(layer)
    r = assert_y_within(y, act, y_ref, oracle.tolerance(x, act, w, TOL), what=f"tc M={M}")
    y2 = run_forward(L, x, act, vq.VQ_PATH_TC)
    assert np.array_equal(y, y2), "not bit-identical run to run"
    return r


TC_CASES = [
    # (N, K, fmt, scale_group, act, M): ragged rows (N % 128), ragged tokens (M % 16), few/many k blocks
    (256, 512, FMT_RVQ12_4, 64, DT_BF16, 64),
    (200, 576, FMT_RVQ12_4, 64, DT_F16, 17),
    (130, 4096, FMT_VQ16, 4096, DT_F16, 40),
    (384, 1024, FMT_RVQ12, 64, DT_BF16, 256),
    (128, 2048, FMT_RVQ12_4, 64, DT_BF16, 300),   # two token tiles, the second ragged
    (96, 1536, FMT_RVQ12_4, 64, DT_F16, 1),
    (136, 1024, FMT_VQ16, 64, DT_BF16, 24),       # 16-bit indices with block scales, staged slices
    (256, 640, FMT_RVQ12, 640, DT_F16, 33),       # one scale per row, 64-wide last slice, staged
    (132, 576, FMT_RVQ12_4, 64, DT_F16, 20),      # N % 8 != 0: indices read from global memory
    (256, 8192, FMT_RVQ12_4, 64, DT_BF16, 32),    # 8 slices per split: the index ring refills
    (2040, 512, FMT_RVQ12_4, 64, DT_BF16, 900),   # 64 tiles: K-split pair (2-CTA cluster), ragged rows/tokens
    (2040, 256, FMT_RVQ12, 64, DT_F16, 1200),     # 80 tiles: one split, y by TMA stores, ragged edges
]


@pytest.mark.parametrize("case", TC_CASES, ids=lambda c: f"{c[0]}x{c[1]}f{c[2]}a{c[4]}M{c[5]}")
def test_tc_forward_matches_oracle(oracle, case):
    N, K, fmt, sg, act, M = case
    layer = make_layer(LayerSpec(N, K, fmt, sg), cfg_id=81, tensor_id=N + M)
    _check(oracle, layer, act, M)


@pytest.mark.parametrize("M", [64, 256, 1024])
def test_prefill_8192_sampled(oracle, M):
    spec = CONFIGS[5]["tensors"][0][1]
    layer = make_layer(spec, cfg_id=5)
    L = layer_on_gpu(layer, DT_BF16, M)
    x = make_x(M, spec.K, DT_BF16, cfg_id=5)
    y = run_forward(L, x, DT_BF16, vq.VQ_PATH_AUTO)
    vq.vq_linear_check(L.handle)
    rows = np.sort(np.random.default_rng(M).choice(spec.N, size=96, replace=False))
    y_ref = oracle.forward(layer, x, DT_BF16, rows=rows)
    w, _ = oracle.dequant(layer, rows=rows)
    assert_y_within(y[:, rows], DT_BF16, y_ref, oracle.tolerance(x, DT_BF16, w, TOL), what=f"prefill M={M}")


def test_single_split_many_slices(oracle):
    """Enough tiles that K is not split: one CTA walks all 16 slices (ring refills,
    no partial sums); checked on sampled rows of a ragged last token tile."""
    N, K, M = 2560, 2048, 1000
    layer = make_layer(LayerSpec(N, K, FMT_RVQ12_4, 64), cfg_id=82)
    L = layer_on_gpu(layer, DT_F16, M)
    x = make_x(M, K, DT_F16, cfg_id=82)
    y = run_forward(L, x, DT_F16, vq.VQ_PATH_TC)
    vq.vq_linear_check(L.handle)
    rows = np.sort(np.random.default_rng(3).choice(N, size=64, replace=False))
    y_ref = oracle.forward(layer, x, DT_F16, rows=rows)
    w, _ = oracle.dequant(layer, rows=rows)
    assert_y_within(y[:, rows], DT_F16, y_ref, oracle.tolerance(x, DT_F16, w, TOL), what="tc single split")


# Layer-sized cases, checked element by element (or on sampled rows): up to eight
# K splits with the last-CTA reduction, ragged rows and tokens, both index widths.
LARGE_CASES = [
    # (N, K, fmt, scale_group, act, M, rows sampled or None)
    (2048, 4096, FMT_RVQ12_4, 64, DT_BF16, 16, None),    # 16 row tiles x 8 K splits
    (2040, 4096, FMT_RVQ12_4, 64, DT_F16, 20, None),     # N % 8 != 0 (indices from global), ragged tokens
    (2048, 4096, FMT_RVQ12, 4096, DT_BF16, 16, None),    # one stage, one scale per row
    (1024, 8192, FMT_VQ16, 8192, DT_F16, 48, None),      # 16-bit indices, 8 splits of 8 slices
    (5120, 512, FMT_RVQ12_4, 64, DT_BF16, 1024, 160),    # 160 tiles in two waves, one split
    (8192, 1024, FMT_RVQ12_4, 64, DT_BF16, 300, 160),    # two token tiles, the second ragged
    (14336, 1024, FMT_RVQ12_4, 64, DT_BF16, 16, 160),    # two CTAs per SM, K-split cluster pairs
    (14336, 1024, FMT_RVQ12_4, 64, DT_F16, 64, 160),     # the same with 64-token tiles (three x stages)
]


@pytest.mark.parametrize("case", LARGE_CASES, ids=lambda c: f"{c[0]}x{c[1]}f{c[2]}a{c[4]}M{c[5]}")
def test_tc_layer_sized_match_oracle(oracle, case):
    N, K, fmt, sg, act, M, nrows = case
    layer = make_layer(LayerSpec(N, K, fmt, sg), cfg_id=84, tensor_id=N + M)
    L = layer_on_gpu(layer, act, M)
    L.set_path(vq.VQ_PATH_TC)
    plan = L.plan(M)
    assert plan["path"] == vq.VQ_PATH_TC and plan["launches"] == 1 and plan["ctas"] >= 1, plan
    x = make_x(M, K, act, cfg_id=84, seed=M)
    y = run_forward(L, x, act, vq.VQ_PATH_TC)
    vq.vq_linear_check(L.handle)
    y2 = run_forward(L, x, act, vq.VQ_PATH_TC)
    assert np.array_equal(y, y2), "not bit-identical run to run"
    rows = None if nrows is None else np.sort(np.random.default_rng(N).choice(N, size=nrows, replace=False))
    y_ref = oracle.forward(layer, x, act, rows=rows)
    w, _ = oracle.dequant(layer, rows=rows)
    got = y if rows is None else y[:, rows]
    assert_y_within(got, act, y_ref, oracle.tolerance(x, act, w, TOL), what=f"layer-sized M={M}")


def test_plan_reports_the_kernel():
    """vq_linear_plan: the kernel family, launches, CTAs and K splits of a forward."""
    handles = []

    def plan_of(spec, M, max_M=1024, corr=0):
        h = vq.vq_linear_create(spec.N, spec.K, spec.fmt, spec.scale_group, DT_BF16, max_M, corr=corr)
        handles.append(h)
        return vq.vq_linear_plan(h, M)

    try:
        gate = CONFIGS[4]["tensors"][0][1]
        p1 = plan_of(gate, 1)
        assert p1["path"] == vq.VQ_PATH_LUT and p1["launches"] == 1 and p1["splits"] == gate.K // 128
        assert p1["ctas"] == torch.cuda.get_device_properties(0).multi_processor_count
        p16 = plan_of(gate, 16)
        assert p16["path"] == vq.VQ_PATH_TC and p16["launches"] == 1
        assert p16["ctas"] == (gate.N // 128) * p16["splits"]
        assert plan_of(gate, 16, corr=1)["launches"] == 2  # the correction's kernel first
        ps = plan_of(LayerSpec(256, 512, FMT_RVQ12_4, 64), 64)
        assert ps["path"] == vq.VQ_PATH_TC and ps["ctas"] == 2 * ps["splits"]
        pg = plan_of(LayerSpec(256, 512, FMT_RVQ12_4, 64), 4)
        assert pg["path"] == vq.VQ_PATH_GEMV
        with pytest.raises(vq.VQError):
            vq.vq_linear_plan(handles[0], 0)
    finally:
        for h in handles:
            vq.vq_linear_destroy(h)


ONE_HOT_CASES = [
    (200, 576, FMT_RVQ12_4, 64, DT_F16),    # staged slices, 64-wide last slice
    (200, 576, FMT_RVQ12_4, 64, DT_BF16),
    (132, 576, FMT_RVQ12, 64, DT_BF16),     # N % 8 != 0: indices from global memory
    (136, 1024, FMT_VQ16, 1024, DT_F16),    # 16-bit indices, one scale per row
    (136, 1024, FMT_VQ16, 64, DT_BF16),
    (8192, 256, FMT_RVQ12_4, 64, DT_BF16),  # 64 row tiles: K-split pair over a 2-CTA cluster
    (9600, 256, FMT_RVQ12, 256, DT_F16),    # 75 row tiles: one split, TMA-stored y
    (2048, 4096, FMT_RVQ12_4, 64, DT_BF16), # 8 K splits: the last CTA of a tile adds the partial sums
]


@pytest.mark.parametrize("case", ONE_HOT_CASES, ids=lambda c: f"{c[0]}x{c[1]}f{c[2]}s{c[3]}a{c[4]}")
def test_tc_one_hot_rows_return_decoded_weights(oracle, case):
    """x = one-hot rows: every y[m][n] is one decoded weight w[n][k_m] (a single
    nonzero product, fp32 accumulation, no rounding), so the tensor-core decode
    must reproduce the oracle's materialised weights bit for bit."""
    N, K, fmt, sg, act = case
    layer = make_layer(LayerSpec(N, K, fmt, sg), cfg_id=83, tensor_id=N + fmt)
    rng = np.random.default_rng(N * 7 + K)
    ks = np.unique(np.concatenate([[0, 7, 8, 63, 64, 127, 128, K - 64, K - 1], rng.integers(0, K, 31)]))
    M = len(ks)
    assert M >= 17
    one = 0x3C00 if act == DT_F16 else 0x3F80
    x = np.zeros((M, K), np.uint16)
    x[np.arange(M), ks] = one
    L = layer_on_gpu(layer, act, M)
    y = run_forward(L, x, act, vq.VQ_PATH_TC)
    vq.vq_linear_check(L.handle)
    _, wb = oracle.dequant(layer, act)
    got = widen(y, act)
    want = widen(wb[:, ks].T, act)
    bad = got != want  # compares values (+0 == -0)
    assert not bad.any(), f"{bad.sum()} decoded weights differ; first at {np.argwhere(bad)[0]}"

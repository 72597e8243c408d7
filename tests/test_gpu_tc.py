"""GPU parity of the tensor-core path (decode to shared memory + tcgen05 MMA) against the oracle."""

import numpy as np
import pytest

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


ONE_HOT_CASES = [
    (200, 576, FMT_RVQ12_4, 64, DT_F16),    # staged slices, 64-wide last slice
    (200, 576, FMT_RVQ12_4, 64, DT_BF16),
    (132, 576, FMT_RVQ12, 64, DT_BF16),     # N % 8 != 0: indices from global memory
    (136, 1024, FMT_VQ16, 1024, DT_F16),    # 16-bit indices, one scale per row
    (136, 1024, FMT_VQ16, 64, DT_BF16),
    (8192, 256, FMT_RVQ12_4, 64, DT_BF16),  # 64 row tiles: K-split pair over a 2-CTA cluster
    (9600, 256, FMT_RVQ12, 256, DT_F16),    # 75 row tiles: one split, TMA-stored y
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

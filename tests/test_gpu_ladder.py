"""GPU parity of the residual bit-width ladder (VQ_FMT_VQ16_RVQ; GLQ README, "Bit widths":
a 16-bit primary stage, 16-bit residual stages and, for odd bit widths, one final 8-bit
stage) on every path that takes it: the gather kernel (M <= 8), the warp-MMA GEMV
(M <= 16) and the tensor-core kernel (any M), plus the debug dequant.

Materialised weights (debug dequant, and the one-hot columns of the two paths that
materialise them) must equal the oracle's bit for bit; forwards must satisfy
max|y_gpu - y_oracle| <= 2e-3 * ||x_m||_2 * max|w| per element and be bit-identical from
run to run."""

import numpy as np
import pytest
import torch

import compressed_index_matmul_b200 as vq
from synth import DT_BF16, DT_F16, FMT_VQ16_RVQ, LayerSpec, make_layer, make_signs, make_x
from tests.gpu_util import assert_y_within, dev, host_bits, layer_on_gpu, require_gpu, run_forward, widen

pytestmark = pytest.mark.gpu

TOL = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _tdt(act):
    return torch.bfloat16 if act == DT_BF16 else torch.float16


@pytest.mark.parametrize("bpw", [3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("wdt", [DT_F16, DT_BF16])
def test_ladder_debug_dequant_is_bit_exact(oracle, bpw, wdt):
    N, K = 72, 448  # 3 full slices and a 64-wide tail
    layer = make_layer(LayerSpec(N, K, FMT_VQ16_RVQ, 64, bpw=bpw), cfg_id=80, tensor_id=bpw)
    L = layer_on_gpu(layer, DT_F16, 1)
    w = torch.empty((N, K), dtype=torch.int16, device="cuda")
    vq.vq_debug_dequant(L.handle, L.planes, L.codebooks, L.t["scales"], w, wdt)
    torch.cuda.synchronize()
    _, ref = oracle.dequant(layer, wdt)
    got = w.cpu().numpy().view(np.uint16)
    assert np.array_equal(got, ref), f"{np.sum(got != ref)} weights differ"


def _check(oracle, layer, act, M, path, what):
    L = layer_on_gpu(layer, act, max(M, 1))
    x = make_x(M, layer["spec"].K, act, cfg_id=81, seed=M)
    y = run_forward(L, x, act, path)
    y2 = run_forward(L, x, act, path)
    vq.vq_linear_check(L.handle)
    w, _ = oracle.dequant(layer)
    assert_y_within(y, act, oracle.forward(layer, x, act), oracle.tolerance(x, act, w, TOL), what=what)
    assert np.array_equal(y, y2), f"{what}: not bit-identical run to run"


LAYERS = [
    # (N, K, scale_group, act)
    (520, 2048, 64, DT_BF16),
    (200, 384, 384, DT_F16),
]


@pytest.mark.parametrize("shape", LAYERS, ids=lambda s: f"{s[0]}x{s[1]}sg{s[2]}a{s[3]}")
@pytest.mark.parametrize("bpw", [3, 4, 5, 7, 8])
@pytest.mark.parametrize("path,M", [(vq.VQ_PATH_GATHER, 1), (vq.VQ_PATH_GATHER, 3), (vq.VQ_PATH_GATHER, 8),
                                    (vq.VQ_PATH_GEMV, 1), (vq.VQ_PATH_GEMV, 9), (vq.VQ_PATH_GEMV, 16),
                                    (vq.VQ_PATH_TC, 2), (vq.VQ_PATH_TC, 40), (vq.VQ_PATH_AUTO, 1),
                                    (vq.VQ_PATH_AUTO, 4)],
                         ids=lambda v: str(v))
def test_ladder_forward_matches_oracle(oracle, shape, bpw, path, M):
    N, K, sg, act = shape
    layer = make_layer(LayerSpec(N, K, FMT_VQ16_RVQ, sg, bpw=bpw), cfg_id=82, tensor_id=N + bpw)
    _check(oracle, layer, act, M, path, f"ladder bpw={bpw} {shape} path {path} M={M}")


@pytest.mark.parametrize("path", [vq.VQ_PATH_GEMV, vq.VQ_PATH_TC])
def test_ladder_ragged_tail_and_rows(oracle, path):
    """K with a 64-wide last slice and N off every tile size: the two materialising paths
    (the gather kernel takes K % 128 == 0 only)."""
    layer = make_layer(LayerSpec(131, 1216, FMT_VQ16_RVQ, 64, bpw=7), cfg_id=83)
    for M in (5, 17):
        if path == vq.VQ_PATH_GEMV and M > 16:
            continue
        _check(oracle, layer, DT_F16, M, path, f"ragged path {path} M={M}")


@pytest.mark.parametrize("path", [vq.VQ_PATH_GEMV, vq.VQ_PATH_TC])
def test_ladder_one_hot_x_returns_materialised_column(oracle, path):
    N, K = 96, 512
    layer = make_layer(LayerSpec(N, K, FMT_VQ16_RVQ, 64, bpw=5), cfg_id=84)
    L = layer_on_gpu(layer, DT_F16, 16)
    ks = [0, 1, 63, 64, 255, 256, 511]
    x = np.zeros((len(ks), K), np.float16)
    for r, k in enumerate(ks):
        x[r, k] = 1.0
    y = run_forward(L, x.view(np.uint16), DT_F16, path)
    _, wb = oracle.dequant(layer, DT_F16)
    for r, k in enumerate(ks):
        assert np.array_equal(y[r], wb[:, k]), f"column {k}"


def _tie_layer():
    """The oracle pin's constructed tie (v = 1 + 2^-11 after stage 2, then mult * c =
    2^-24 + 2^-57): a single rounding of each stage sum makes the fp16 weight 0x3C01,
    rounding the fp64 sum instead would give 0x3C00.  Every group of the 8 x 128 layer
    uses entry 0 of every codebook."""
    N, K = 8, 128
    G = K // 8
    f16 = lambda v: np.asarray(v, np.float32).astype(np.float16).view(np.uint16)  # noqa: E731
    cb1 = np.zeros((65536, 8), np.uint16)
    cbr = np.zeros((2, 65536, 8), np.uint16)
    cb1[0] = f16([1.0] * 8)
    cbr[0][0] = f16([1.0] * 8)
    cbr[1][0] = f16([1206 / 1024] * 8)
    return {"spec": LayerSpec(N, K, FMT_VQ16_RVQ, K, bpw=6), "cb1": cb1, "cbr": cbr,
            "cb8": np.zeros((256, 8), np.uint16), "idx16": np.zeros(3 * N * G, np.uint16), "idx8": None,
            "mult": np.array([2.0 ** -11, 14245331 * 2.0 ** -48], np.float32), "scales": f16([1.0] * N)}


def test_ladder_stage_sum_rounds_once_on_the_gpu(oracle):
    layer = _tie_layer()
    _, wb = oracle.dequant(layer, DT_F16)
    assert np.all(wb == 0x3C01)
    L = layer_on_gpu(layer, DT_F16, 16)
    w = torch.empty((8, 128), dtype=torch.int16, device="cuda")
    vq.vq_debug_dequant(L.handle, L.planes, L.codebooks, L.t["scales"], w, DT_F16)
    torch.cuda.synchronize()
    assert np.all(w.cpu().numpy().view(np.uint16) == 0x3C01)
    x = np.zeros((2, 128), np.float16)
    x[0, 3] = x[1, 100] = 1.0
    for path in (vq.VQ_PATH_GEMV, vq.VQ_PATH_TC):
        y = run_forward(L, x.view(np.uint16), DT_F16, path)
        assert np.all(y == 0x3C01), (path, y)


def test_ladder_rotated_fused(oracle):
    """The batch-1 gather kernel rotates x itself for the ladder too (K = 2688, block-diagonal)."""
    N, K = 256, 2688
    layer = make_layer(LayerSpec(N, K, FMT_VQ16_RVQ, 64, bpw=5), cfg_id=85)
    L = layer_on_gpu(layer, DT_BF16, 1)
    assert L.launches(1) == 1
    x = make_x(1, K, DT_BF16, cfg_id=85)
    signs = make_signs(K, cfg_id=85)
    y = host_bits(L.forward_rotated(dev(x).view(torch.bfloat16), dev(signs)))
    torch.cuda.synchronize()
    xr = oracle.rht(x, DT_BF16, signs)
    w, _ = oracle.dequant(layer)
    tol = TOL * np.linalg.norm(xr) * np.abs(w).max()
    assert_y_within(y, DT_BF16, xr @ w.T, tol, what="ladder fused rotation")


@pytest.mark.parametrize("M", [1, 8])
def test_ladder_full_size_sampled(oracle, M):
    """4096 x 4096 at 5 bpw (16 + 16 + 8): the oracle recomputes 256 sampled rows."""
    spec = LayerSpec(4096, 4096, FMT_VQ16_RVQ, 64, bpw=5)
    layer = make_layer(spec, cfg_id=86)
    L = layer_on_gpu(layer, DT_F16, M)
    x = make_x(M, spec.K, DT_F16, cfg_id=86)
    y = run_forward(L, x, DT_F16)
    vq.vq_linear_check(L.handle)
    rows = np.sort(np.random.default_rng(M).choice(spec.N, size=256, replace=False))
    w, _ = oracle.dequant(layer, rows=rows)
    assert_y_within(y[:, rows], DT_F16, oracle.forward(layer, x, DT_F16, rows=rows),
                    oracle.tolerance(x, DT_F16, w, TOL), what=f"ladder 4096^2 M={M}")


def test_ladder_noalloc_forward(oracle):
    """The handle-free forward takes the ladder's descriptor fields too."""
    N, K, M = 136, 512, 3
    layer = make_layer(LayerSpec(N, K, FMT_VQ16_RVQ, 64, bpw=7), cfg_id=87)
    L = layer_on_gpu(layer, DT_F16, M)
    x = make_x(M, K, DT_F16, cfg_id=87)
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    vq.vq_linear_forward_noalloc(N, K, FMT_VQ16_RVQ, 64, DT_F16, dev(x).view(torch.float16), L.planes, L.codebooks,
                                 L.t["scales"], y, M, n16=L.n16, n8=L.n8, mult=L.mult)
    torch.cuda.synchronize()
    w, _ = oracle.dequant(layer)
    assert_y_within(host_bits(y), DT_F16, oracle.forward(layer, x, DT_F16), oracle.tolerance(x, DT_F16, w, TOL),
                    what="ladder noalloc")


def test_ladder_missing_stage_pointers_are_rejected():
    layer = make_layer(LayerSpec(64, 256, FMT_VQ16_RVQ, 64, bpw=5), cfg_id=88)
    L = layer_on_gpu(layer, DT_F16, 1)
    x = torch.zeros((1, 256), dtype=torch.float16, device="cuda")
    y = torch.empty((1, 64), dtype=torch.float16, device="cuda")
    no8 = vq.make_planes(idx16=L.t["idx16"])  # n8 == 1 needs idx8
    with pytest.raises(vq.VQError) as ei:
        vq.vq_linear_forward(L.handle, x, no8, L.codebooks, L.t["scales"], y, 1, 64, 256)
    assert ei.value.status == vq._binding.VQ_ERR_INVALID_ARG
    nocb = vq.make_codebooks(L.t["cb1"], None, (), L.t["cb8"])  # n16 == 2 needs cbr[0]
    with pytest.raises(vq.VQError) as ei:
        vq.vq_linear_forward(L.handle, x, L.planes, nocb, L.t["scales"], y, 1, 64, 256)
    assert ei.value.status == vq._binding.VQ_ERR_INVALID_ARG

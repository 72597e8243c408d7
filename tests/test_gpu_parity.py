"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Indices and materialised weights must match bit-exactly; y must satisfy
max|y_gpu - y_oracle| <= 2e-3 * ||x_m||_2 * max|w| per element (fp32 accumulate,
fp16/bf16 output), and repeated runs must be bit-identical.
"""

import numpy as np
import pytest
import torch

import compressed_index_matmul_b200 as vq
from synth import (DT_BF16, DT_F16, FMT_RVQ12, FMT_RVQ12_4, FMT_VQ16, CONFIGS, LayerSpec, make_layer, make_signs,
                   make_x)
from tests.gpu_util import assert_y_within, dev, host_bits, layer_on_gpu, require_gpu, run_forward, widen

pytestmark = pytest.mark.gpu

TOL = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


SHAPES = [
    # (N, K, fmt, scale_group, act): several 128-row tiles with ragged tails, K not a multiple of 256
    (256, 256, FMT_RVQ12, 64, DT_F16),
    (200, 576, FMT_RVQ12_4, 64, DT_F16),
    (300, 1536, FMT_RVQ12_4, 64, DT_BF16),
    (130, 4096, FMT_VQ16, 4096, DT_F16),
    (72, 1024, FMT_RVQ12, 1024, DT_BF16),
    (96, 14336, FMT_RVQ12_4, 64, DT_BF16),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"{s[0]}x{s[1]}f{s[2]}sg{s[3]}a{s[4]}")
def test_unpack_bit_exact(oracle, shape):
    N, K, fmt, sg, act = shape
    layer = make_layer(LayerSpec(N, K, fmt, sg), cfg_id=50, tensor_id=N)
    L = layer_on_gpu(layer, act, 1)
    i1 = torch.empty((N, K // 8), dtype=torch.int16, device="cuda")
    i2 = torch.empty((N, K // 8), dtype=torch.uint8, device="cuda")
    vq.vq_debug_unpack(L.handle, L.planes, i1, i2)
    torch.cuda.synchronize()
    r1, r2 = oracle.unpack(layer)
    assert np.array_equal(i1.cpu().numpy().view(np.uint16).astype(np.uint32), r1)
    assert np.array_equal(i2.cpu().numpy(), r2)


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"{s[0]}x{s[1]}f{s[2]}sg{s[3]}a{s[4]}")
@pytest.mark.parametrize("wdt", [DT_F16, DT_BF16])
def test_dequant_bit_exact(oracle, shape, wdt):
    N, K, fmt, sg, act = shape
    layer = make_layer(LayerSpec(N, K, fmt, sg), cfg_id=51, tensor_id=N)
    L = layer_on_gpu(layer, act, 1)
    w = torch.empty((N, K), dtype=torch.int16, device="cuda")
    vq.vq_debug_dequant(L.handle, L.planes, L.codebooks, L.t["scales"], w, wdt)
    torch.cuda.synchronize()
    _, ref = oracle.dequant(layer, wdt)
    got = w.cpu().numpy().view(np.uint16)
    assert np.array_equal(got, ref), f"{np.sum(got != ref)} weights differ"


def _check_forward(oracle, layer, act, M, path, seed=0):
    L = layer_on_gpu(layer, act, max(M, 1))
    x = make_x(M, layer["spec"].K, act, cfg_id=52, seed=seed)
    y = run_forward(L, x, act, path)
    y_ref = oracle.forward(layer, x, act)
    w, _ = oracle.dequant(layer)
    tol = oracle.tolerance(x, act, w, TOL)
    r = assert_y_within(y, act, y_ref, tol, what=f"path {path} M={M}")
    y2 = run_forward(L, x, act, path)
    assert np.array_equal(y, y2), "forward is not bit-identical run to run"
    return r


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"{s[0]}x{s[1]}f{s[2]}sg{s[3]}a{s[4]}")
@pytest.mark.parametrize("M", [1, 3, 8, 9, 16])
def test_gemv_forward_matches_oracle(oracle, shape, M):
    N, K, fmt, sg, act = shape
    layer = make_layer(LayerSpec(N, K, fmt, sg), cfg_id=53, tensor_id=N)
    _check_forward(oracle, layer, act, M, vq.VQ_PATH_GEMV)


LUT_SHAPES = [s for s in SHAPES if s[2] != FMT_VQ16 and s[1] % 128 == 0] + [
    (1000, 4096, FMT_RVQ12_4, 64, DT_BF16),   # several 256-row chunks, many K-slices
    (2052, 2048, FMT_RVQ12, 2048, DT_F16),    # ragged last chunk, per-row scales
]


@pytest.mark.parametrize("shape", LUT_SHAPES, ids=lambda s: f"{s[0]}x{s[1]}f{s[2]}sg{s[3]}a{s[4]}")
def test_lut_forward_matches_oracle(oracle, shape):
    N, K, fmt, sg, act = shape
    layer = make_layer(LayerSpec(N, K, fmt, sg), cfg_id=58, tensor_id=N)
    for seed in (0, 1):
        _check_forward(oracle, layer, act, 1, vq.VQ_PATH_LUT, seed=seed)


@pytest.mark.parametrize("N,K", [(64, 576), (66, 1024)])
def test_lut_rejects_unsupported_shapes(oracle, N, K):
    """K % 128 != 0 or N % 4 != 0: the table kernel refuses, AUTO takes the warp-MMA kernel."""
    layer = make_layer(LayerSpec(N, K, FMT_RVQ12_4, 64), cfg_id=58)
    L = layer_on_gpu(layer, DT_F16, 1)
    L.set_path(vq.VQ_PATH_LUT)
    with pytest.raises(vq.VQError) as ei:
        L.forward(torch.zeros((1, K), dtype=torch.float16, device="cuda"))
    assert ei.value.status == vq._binding.VQ_ERR_UNSUPPORTED
    _check_forward(oracle, layer, DT_F16, 1, vq.VQ_PATH_AUTO)


def test_lut_handles_extreme_activation_scales(oracle):
    """bf16 inputs far outside fp16 range, and tiny ones, go through the power-of-two rescaling."""
    N, K = 300, 1024
    layer = make_layer(LayerSpec(N, K, FMT_RVQ12_4, 64), cfg_id=59)
    L = layer_on_gpu(layer, DT_BF16, 1)
    w, _ = oracle.dequant(layer)
    for scale in (2.0 ** 40, 2.0 ** -60):
        xf = np.random.default_rng(3).standard_normal((1, K)).astype(np.float32) * np.float32(scale)
        import synth
        x = synth.f32_to_bf16_bits(xf)
        y = run_forward(L, x, DT_BF16, vq.VQ_PATH_LUT)
        y_ref = oracle.forward(layer, x, DT_BF16)
        assert_y_within(y, DT_BF16, y_ref, oracle.tolerance(x, DT_BF16, w, TOL), what=f"scale {scale}")


@pytest.mark.parametrize("shape", SHAPES[:3], ids=lambda s: f"{s[0]}x{s[1]}f{s[2]}")
def test_auto_path_matches_oracle(oracle, shape):
    N, K, fmt, sg, act = shape
    layer = make_layer(LayerSpec(N, K, fmt, sg), cfg_id=54, tensor_id=N)
    for M in (1, 2, 16):
        _check_forward(oracle, layer, act, M, vq.VQ_PATH_AUTO)


def test_one_hot_x_returns_materialised_column(oracle):
    N, K = 160, 512
    layer = make_layer(LayerSpec(N, K, FMT_RVQ12_4, 64), cfg_id=55)
    L = layer_on_gpu(layer, DT_F16, 16)
    ks = [0, 1, 63, 64, 255, 256, 511]
    x = np.zeros((len(ks), K), np.float16)
    for r, k in enumerate(ks):
        x[r, k] = 1.0
    y = run_forward(L, x.view(np.uint16), DT_F16, vq.VQ_PATH_GEMV)
    _, wb = oracle.dequant(layer, DT_F16)
    for r, k in enumerate(ks):
        assert np.array_equal(y[r], wb[:, k]), f"column {k}"


def test_zero_tokens_is_a_no_op():
    layer = make_layer(LayerSpec(64, 256, FMT_RVQ12, 64), cfg_id=56)
    L = layer_on_gpu(layer, DT_F16, 4)
    y = torch.full((1, 64), 7.0, dtype=torch.float16, device="cuda")
    x = torch.zeros((1, 256), dtype=torch.float16, device="cuda")
    vq.vq_linear_forward(L.handle, x, L.planes, L.codebooks, L.t["scales"], y, 0, 64, 256)
    torch.cuda.synchronize()
    assert bool((y == 7.0).all())
    assert L.launches(0) == 0


def test_forward_argument_errors():
    layer = make_layer(LayerSpec(64, 256, FMT_RVQ12_4, 64), cfg_id=57)
    L = layer_on_gpu(layer, DT_F16, 4)
    x = torch.zeros((4, 256), dtype=torch.float16, device="cuda")
    y = torch.zeros((4, 64), dtype=torch.float16, device="cuda")
    sc = L.t["scales"]
    cases = [
        dict(M=5),                     # above max_M
        dict(N=63), dict(K=192),       # shape mismatch
        dict(x=x.data_ptr() + 2),      # misaligned
        dict(y=x),                     # aliasing
    ]
    for c in cases:
        args = dict(x=x, y=y, M=4, N=64, K=256)
        args.update(c)
        with pytest.raises(vq.VQError) as ei:
            vq.vq_linear_forward(L.handle, args["x"], L.planes, L.codebooks, sc, args["y"], args["M"], args["N"],
                                 args["K"])
        assert ei.value.status == vq._binding.VQ_ERR_INVALID_ARG
    bad_planes = vq.make_planes(L.t["lo"], None, L.t["s2"])
    with pytest.raises(vq.VQError, match="hi4"):
        vq.vq_linear_forward(L.handle, x, bad_planes, L.codebooks, sc, y, 4, 64, 256)
    with pytest.raises(vq.VQError) as ei:
        L.set_path(vq.VQ_PATH_GEMV)
        big = layer_on_gpu(layer, DT_F16, 32)
        big.set_path(vq.VQ_PATH_GEMV)
        big.forward(torch.zeros((17, 256), dtype=torch.float16, device="cuda"))
    assert ei.value.status == vq._binding.VQ_ERR_UNSUPPORTED


# ------------------------------------------------------------------- rotation

def _rht_check(oracle, M, K, dt):
    x = make_x(M, K, dt, cfg_id=60)
    signs = make_signs(K, cfg_id=60)
    xt = dev(x)
    st = dev(signs)
    out = torch.empty_like(xt)
    vq.vq_rht_apply(xt, out, st, M, K, dt)
    torch.cuda.synchronize()
    got = widen(host_bits(out), dt)
    ref = oracle.rht(x, dt, signs)
    if dt == DT_F16:
        ulp = np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64)
    else:
        ulp = np.abs(ref) * 2.0 ** -7
    # fp32 butterflies vs the fp64 definition: rounding to the output type (<= 1 ulp with the
    # double rounding) plus the fp32 transform error, bounded by log2(K) stages of 2^-24
    # relative error on vectors whose 2-norm is ||x_m||_2 after the 1/sqrt(K) scaling.
    xn = np.linalg.norm(widen(x, dt), axis=1, keepdims=True)
    atol = 2 * np.log2(K) * 2.0 ** -24 * xn
    err = np.abs(got - ref)
    assert np.all(err <= ulp + atol), f"max err/(ulp+atol) = {np.max(err / (ulp + atol))}"
    # in place gives the same bits
    vq.vq_rht_apply(xt, xt, st, M, K, dt)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(xt), host_bits(out))
    return got


@pytest.mark.parametrize("K", [64, 128, 1024, 4096, 32768,
                               192, 2688, 12288, 32704])  # block-diagonal: 32704 has all nine blocks 16384..64
@pytest.mark.parametrize("dt", [DT_F16, DT_BF16])
def test_rht_matches_oracle(oracle, K, dt):
    _rht_check(oracle, 3, K, dt)


# ------------------------------------------------------------- full-size workloads

def _sampled_forward_check(oracle, layer, act, M, path, nrows=192, seed=0):
    """Full-size GPU forward; the oracle recomputes a random sample of output rows."""
    spec = layer["spec"]
    L = layer_on_gpu(layer, act, M)
    x = make_x(M, spec.K, act, cfg_id=70 + M, seed=seed)
    y = run_forward(L, x, act, path)
    rows = np.sort(np.random.default_rng(seed).choice(spec.N, size=min(nrows, spec.N), replace=False))
    y_ref = oracle.forward(layer, x, act, rows=rows)
    w, _ = oracle.dequant(layer, rows=rows)
    # max|w| over the whole layer bounds the sampled rows' tolerance from below; use the sample's
    tol = oracle.tolerance(x, act, w, TOL)
    return assert_y_within(y[:, rows], act, y_ref, tol, what=f"{spec} M={M}")


@pytest.mark.parametrize("M", [1, 2, 4, 16])
def test_llama3_8b_mlp_sampled(oracle, M):
    for label, spec in CONFIGS[4]["tensors"]:
        layer = make_layer(spec, cfg_id=4, tensor_id={"gate": 0, "up": 1, "down": 2}[label])
        _sampled_forward_check(oracle, layer, DT_BF16, M, vq.VQ_PATH_AUTO)


@pytest.mark.parametrize("M", [1, 4, 16])
def test_smollm_stack_layers(oracle, M):
    for layer_idx in (0, 29):
        for ti, (label, spec) in enumerate(CONFIGS[2]["tensors"]):
            layer = make_layer(spec, cfg_id=2, layer=layer_idx, tensor_id=ti)
            _check_forward(oracle, layer, DT_F16, M, vq.VQ_PATH_AUTO)


@pytest.mark.parametrize("M", [1, 8])
def test_vq16_rotated_end_to_end(oracle, M):
    spec = CONFIGS[3]["tensors"][0][1]
    layer = make_layer(spec, cfg_id=3)
    x = make_x(M, spec.K, DT_F16, cfg_id=3)
    signs = make_signs(spec.K, cfg_id=3)
    L = layer_on_gpu(layer, DT_F16, M)
    xt = dev(x).view(torch.float16)
    xr = torch.empty_like(xt)
    vq.vq_rht_apply(xt, xr, dev(signs), M, spec.K, DT_F16)
    y = host_bits(L.forward(xr))
    torch.cuda.synchronize()
    x_rot = oracle.round_to(oracle.rht(x, DT_F16, signs), DT_F16)
    rows = np.sort(np.random.default_rng(M).choice(spec.N, size=512, replace=False))
    y_ref = oracle.forward(layer, x_rot, DT_F16, rows=rows)
    w, _ = oracle.dequant(layer, rows=rows)
    assert_y_within(y[:, rows], DT_F16, y_ref, oracle.tolerance(x_rot, DT_F16, w, TOL), what="cfg3")


def test_single_256_layer(oracle):
    spec = CONFIGS[1]["tensors"][0][1]
    layer = make_layer(spec, cfg_id=1)
    _check_forward(oracle, layer, DT_F16, 1, vq.VQ_PATH_AUTO)

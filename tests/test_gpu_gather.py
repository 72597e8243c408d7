"""GPU parity of the batch-1 gather kernel for the 16-bit format (VQ_PATH_GATHER) and of
vq_linear_forward_rotated, the forward that applies the input rotation itself.

y must satisfy max|y_gpu - y_oracle| <= 2e-3 * ||x_m||_2 * max|w| per element and be
bit-identical from run to run.  For the fused rotation the kernel keeps the rotated x
in fp32, so its reference is the oracle's fp64 rotation, unrounded, times the oracle's
exact weights; the unfused fallback rounds the rotated x to the activation type, as
vq_rht_apply does, and is compared with the oracle forward of that rounded x."""

import numpy as np
import pytest
import torch

import compressed_index_matmul_b200 as vq
from synth import (CONFIGS, DT_BF16, DT_F16, FMT_RVQ12_4, FMT_VQ16, FMT_VQ16_RVQ, LayerSpec, make_layer, make_signs,
                   make_x)
from tests.gpu_util import assert_y_within, dev, host_bits, layer_on_gpu, require_gpu, run_forward, widen

pytestmark = pytest.mark.gpu

TOL = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _tdt(act):
    return torch.bfloat16 if act == DT_BF16 else torch.float16


SHAPES = [
    # (N, K, scale_group, act)
    (256, 256, 256, DT_F16),      # per-row scales, two slices
    (1000, 2048, 64, DT_BF16),    # block scales, ragged row chunks
    (4, 128, 128, DT_F16),        # one slice: no split-K, y written directly
    (132, 16384, 64, DT_F16),     # the largest K this kernel takes
    (2052, 1024, 1024, DT_BF16),  # rows not a multiple of the 512-row chunk
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"{s[0]}x{s[1]}sg{s[2]}a{s[3]}")
@pytest.mark.parametrize("path", [vq.VQ_PATH_GATHER, vq.VQ_PATH_AUTO], ids=["forced", "auto"])
def test_gather_matches_oracle(oracle, shape, path):
    N, K, sg, act = shape
    layer = make_layer(LayerSpec(N, K, FMT_VQ16, sg), cfg_id=70, tensor_id=N)
    L = layer_on_gpu(layer, act, 1)
    x = make_x(1, K, act, cfg_id=70)
    y1 = run_forward(L, x, act, path)
    y2 = run_forward(L, x, act, path)
    vq.vq_linear_check(L.handle)
    y_ref = oracle.forward(layer, x, act)
    w, _ = oracle.dequant(layer)
    assert_y_within(y1, act, y_ref, oracle.tolerance(x, act, w, TOL), what=f"gather {shape}")
    assert np.array_equal(y1, y2), "not bit-identical run to run"


MULTI = [
    # (N, K, scale_group, act, M): several tokens share every gathered codeword
    (256, 256, 256, DT_F16, 2),
    (1000, 2048, 64, DT_BF16, 3),
    (520, 4096, 4096, DT_F16, 8),
    (132, 8192, 64, DT_F16, 4),
    (2052, 1024, 64, DT_BF16, 5),
]


@pytest.mark.parametrize("shape", MULTI, ids=lambda s: f"{s[0]}x{s[1]}sg{s[2]}a{s[3]}M{s[4]}")
def test_gather_several_tokens(oracle, shape):
    N, K, sg, act, M = shape
    layer = make_layer(LayerSpec(N, K, FMT_VQ16, sg), cfg_id=76, tensor_id=N)
    L = layer_on_gpu(layer, act, M)
    x = make_x(M, K, act, cfg_id=76)
    y1 = run_forward(L, x, act, vq.VQ_PATH_GATHER)
    y2 = run_forward(L, x, act, vq.VQ_PATH_AUTO)  # the gather kernel up to M = 4, else another path
    vq.vq_linear_check(L.handle)
    y_ref = oracle.forward(layer, x, act)
    w, _ = oracle.dequant(layer)
    tol = oracle.tolerance(x, act, w, TOL)
    assert_y_within(y1, act, y_ref, tol, what=f"gather {shape}")
    if M <= 4:
        assert np.array_equal(y1, y2), "forced and automatic paths differ"
    else:
        assert_y_within(y2, act, y_ref, tol, what=f"auto {shape}")


def test_gather_config3_sampled(oracle):
    spec = CONFIGS[3]["tensors"][0][1]
    layer = make_layer(spec, cfg_id=3)
    L = layer_on_gpu(layer, DT_F16, 1)
    x = make_x(1, spec.K, DT_F16, cfg_id=71)
    y = run_forward(L, x, DT_F16, vq.VQ_PATH_GATHER)
    rows = np.sort(np.random.default_rng(3).choice(spec.N, size=512, replace=False))
    y_ref = oracle.forward(layer, x, DT_F16, rows=rows)
    w, _ = oracle.dequant(layer, rows=rows)
    assert_y_within(y[:, rows], DT_F16, y_ref, oracle.tolerance(x, DT_F16, w, TOL), what="cfg3 gather")


def test_gather_with_sm_budget(oracle):
    layer = make_layer(LayerSpec(1000, 2048, FMT_VQ16, 64), cfg_id=72)
    L = layer_on_gpu(layer, DT_F16, 1)
    x = make_x(1, 2048, DT_F16, cfg_id=72)
    y_ref = oracle.forward(layer, x, DT_F16)
    w, _ = oracle.dequant(layer)
    for budget in (1, 5, 0):
        L.set_sm_budget(budget)
        y = run_forward(L, x, DT_F16, vq.VQ_PATH_GATHER)
        assert_y_within(y, DT_F16, y_ref, oracle.tolerance(x, DT_F16, w, TOL), what=f"budget {budget}")


@pytest.mark.parametrize("N, K, fmt, M", [(256, 16512, FMT_VQ16, 1), (258, 256, FMT_VQ16, 1),
                                          (256, 256, FMT_VQ16, 9), (256, 8192, FMT_VQ16, 5),
                                          (256, 256, FMT_RVQ12_4, 1)])
def test_gather_rejects_what_it_does_not_take(N, K, fmt, M):
    layer = make_layer(LayerSpec(N, K, fmt, 64), cfg_id=73)
    L = layer_on_gpu(layer, DT_F16, M)
    L.set_path(vq.VQ_PATH_GATHER)
    x = torch.zeros((M, K), dtype=torch.float16, device="cuda")
    with pytest.raises(vq.VQError) as ei:
        L.forward(x)
    assert ei.value.status == vq._binding.VQ_ERR_UNSUPPORTED


def _rotated_reference(oracle, layer, x, act, signs, rows):
    """Unrounded fp64 rotation of x times the exact weights of `rows`, with its bound."""
    xr = oracle.rht(x, act, signs)
    w, _ = oracle.dequant(layer, rows=rows)
    y_ref = xr @ w.T
    tol = TOL * np.sqrt((xr * xr).sum(axis=1, keepdims=True)) * np.abs(w).max()
    return y_ref, tol


@pytest.mark.parametrize("shape", [(256, 256, 256, DT_F16), (520, 2048, 64, DT_BF16), (64, 128, 128, DT_F16),
                                   (256, 512, 512, DT_BF16), (128, 1024, 64, DT_F16), (132, 16384, 64, DT_F16),
                                   # K not a power of two: block-diagonal rotation (2048 + 512 + 128, ...)
                                   (256, 2688, 64, DT_BF16), (200, 384, 384, DT_F16), (132, 16256, 64, DT_F16)],
                         ids=lambda s: f"{s[0]}x{s[1]}sg{s[2]}a{s[3]}")
def test_rotated_fused_matches_oracle(oracle, shape):
    N, K, sg, act = shape
    layer = make_layer(LayerSpec(N, K, FMT_VQ16, sg), cfg_id=74, tensor_id=N)
    L = layer_on_gpu(layer, act, 1)
    assert L.launches(1) == 1
    x = make_x(1, K, act, cfg_id=74)
    signs = make_signs(K, cfg_id=74)
    xt, st = dev(x).view(_tdt(act)), dev(signs)
    y1 = host_bits(L.forward_rotated(xt, st))
    y2 = host_bits(L.forward_rotated(xt, st))
    torch.cuda.synchronize()
    vq.vq_linear_check(L.handle)
    y_ref, tol = _rotated_reference(oracle, layer, x, act, signs, None)
    assert_y_within(y1, act, y_ref, tol, what=f"fused rotation {shape}")
    assert np.array_equal(y1, y2), "not bit-identical run to run"


@pytest.mark.parametrize("M", [1, 4, 8])
def test_rotated_config3(oracle, M):
    """Config 3: M <= 4 runs the fused kernel, M = 8 the rotation into the handle's
    buffer followed by the tensor-core forward (the handle is created with rht = 1)."""
    spec = CONFIGS[3]["tensors"][0][1]
    layer = make_layer(spec, cfg_id=3)
    L = vq.VQLinear(spec.N, spec.K, spec.fmt, spec.scale_group, DT_F16, 8, layer, rht=1)
    x = make_x(M, spec.K, DT_F16, cfg_id=3)
    signs = make_signs(spec.K, cfg_id=3)
    y = host_bits(L.forward_rotated(dev(x).view(torch.float16), dev(signs)))
    torch.cuda.synchronize()
    vq.vq_linear_check(L.handle)
    rows = np.sort(np.random.default_rng(M).choice(spec.N, size=512, replace=False))
    if M <= 4:
        y_ref, tol = _rotated_reference(oracle, layer, x, DT_F16, signs, rows)
    else:
        x_rot = oracle.round_to(oracle.rht(x, DT_F16, signs), DT_F16)
        y_ref = oracle.forward(layer, x_rot, DT_F16, rows=rows)
        w, _ = oracle.dequant(layer, rows=rows)
        tol = oracle.tolerance(x_rot, DT_F16, w, TOL)
    assert_y_within(y[:, rows], DT_F16, y_ref, tol, what=f"cfg3 rotated M={M}")


@pytest.mark.parametrize("N, K, sg, act, M, bpw", [
    (256, 256, 256, DT_F16, 2, 0), (520, 2048, 64, DT_BF16, 3, 0), (128, 1024, 64, DT_F16, 4, 0),
    (256, 2688, 64, DT_BF16, 5, 0),      # block-diagonal rotation, 2048 + 512 + 128
    (384, 4096, 4096, DT_F16, 8, 0),     # M' K = 32768, the largest x the kernel holds
    (256, 1024, 1024, DT_F16, 3, 3),     # the residual ladder (16 + 8 bits)
], ids=lambda v: str(v))
def test_rotated_fused_several_tokens(oracle, N, K, sg, act, M, bpw):
    """1 < M <= 8 on the gather kernel (forced beyond M = 4): one kernel rotates every
    token in fp32 (the handle has no rotation buffer, so the unfused route would be
    refused) and matches the oracle's unrounded rotation."""
    spec = LayerSpec(N, K, FMT_VQ16_RVQ, sg, bpw=bpw) if bpw else LayerSpec(N, K, FMT_VQ16, sg)
    layer = make_layer(spec, cfg_id=77, tensor_id=N + M)
    L = layer_on_gpu(layer, act, M)
    L.set_path(vq.VQ_PATH_GATHER)
    x = make_x(M, K, act, cfg_id=77, seed=M)
    signs = make_signs(K, cfg_id=77)
    xt, st = dev(x).view(_tdt(act)), dev(signs)
    y1 = host_bits(L.forward_rotated(xt, st))
    y2 = host_bits(L.forward_rotated(xt, st))
    torch.cuda.synchronize()
    vq.vq_linear_check(L.handle)
    y_ref, tol = _rotated_reference(oracle, layer, x, act, signs, None)
    assert_y_within(y1, act, y_ref, tol, what=f"fused rotation M={M}")
    assert np.array_equal(y1, y2), "not bit-identical run to run"


def test_rotated_argument_errors():
    layer = make_layer(LayerSpec(256, 256, FMT_VQ16, 256), cfg_id=75)
    L = layer_on_gpu(layer, DT_F16, 8)  # rht = 0: no rotation buffer
    signs = dev(make_signs(256, cfg_id=75))
    x8 = torch.zeros((8, 256), dtype=torch.float16, device="cuda")
    with pytest.raises(vq.VQError) as ei:  # M = 8 is not fused by default and the handle has no buffer
        L.forward_rotated(x8, signs)
    assert ei.value.status == vq._binding.VQ_ERR_INVALID_ARG
    L.set_path(vq.VQ_PATH_TC)
    with pytest.raises(vq.VQError) as ei:  # a forced path other than the gather kernel is not fused
        L.forward_rotated(x8[:1], signs)
    assert ei.value.status == vq._binding.VQ_ERR_INVALID_ARG
    L.set_path(vq.VQ_PATH_AUTO)
    y = torch.empty((1, 256), dtype=torch.float16, device="cuda")
    with pytest.raises(vq.VQError) as ei:
        vq.vq_linear_forward_rotated(L.handle, x8[:1], None, L.planes, L.codebooks, L.t["scales"], y, 1, 256, 256)
    assert ei.value.status == vq._binding.VQ_ERR_INVALID_ARG
    layer2 = make_layer(LayerSpec(8, 65536, FMT_VQ16, 65536), cfg_id=75)
    L2 = layer_on_gpu(layer2, DT_F16, 1)
    with pytest.raises(vq.VQError) as ei:  # K above the rotation's 32768
        L2.forward_rotated(torch.zeros((1, 65536), dtype=torch.float16, device="cuda"),
                           dev(make_signs(65536, cfg_id=75)))
    assert ei.value.status == vq._binding.VQ_ERR_INVALID_ARG
    with pytest.raises(vq.VQError) as ei:  # signs not 16-byte aligned
        L.forward_rotated(x8[:1], dev(make_signs(264, cfg_id=75))[8:])
    assert ei.value.status == vq._binding.VQ_ERR_INVALID_ARG


def test_rotated_block_diagonal_unfused(oracle):
    """K = 2688 = 2048 + 512 + 128 at M = 8 on the tensor-core path (forced): the rotation
    kernel into the handle's buffer, then the forward, against the oracle's
    block-diagonal rotation rounded the same way."""
    N, K, M = 384, 2688, 8
    layer = make_layer(LayerSpec(N, K, FMT_VQ16, 64), cfg_id=76)
    L = vq.VQLinear(N, K, FMT_VQ16, 64, DT_BF16, M, layer, rht=1)
    L.set_path(vq.VQ_PATH_TC)
    x = make_x(M, K, DT_BF16, cfg_id=76)
    signs = make_signs(K, cfg_id=76)
    y = host_bits(L.forward_rotated(dev(x).view(torch.bfloat16), dev(signs)))
    torch.cuda.synchronize()
    vq.vq_linear_check(L.handle)
    x_rot = oracle.round_to(oracle.rht(x, DT_BF16, signs), DT_BF16)
    y_ref = oracle.forward(layer, x_rot, DT_BF16)
    w, _ = oracle.dequant(layer)
    assert_y_within(y, DT_BF16, y_ref, oracle.tolerance(x_rot, DT_BF16, w, TOL), what="K=2688 M=8 rotated")


# ------------------------------------------------------------------- output rotation

@pytest.mark.parametrize("N", [64, 1024, 4096, 32768, 2688, 32704])
@pytest.mark.parametrize("dt", [DT_F16, DT_BF16])
def test_rht_output_matches_oracle(oracle, N, dt):
    """signs * (1/sqrt N) H y against the oracle's explicit product: within one output ulp
    (double rounding) plus the fp32 transform error, and the same bits in place."""
    M = 3
    y = make_x(M, N, dt, cfg_id=77)
    signs = make_signs(N, cfg_id=77)
    yt, st = dev(y), dev(signs)
    out = torch.empty_like(yt)
    vq.vq_rht_apply_output(yt, out, st, M, N, dt)
    torch.cuda.synchronize()
    got = widen(host_bits(out), dt)
    ref = oracle.rht_out_f64(widen(y, dt), signs)
    ulp = np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64) if dt == DT_F16 else np.abs(ref) * 2.0 ** -7
    atol = 2 * np.log2(N) * 2.0 ** -24 * np.linalg.norm(widen(y, dt), axis=1, keepdims=True)
    err = np.abs(got - ref)
    assert np.all(err <= ulp + atol), f"max err/(ulp+atol) = {np.max(err / (ulp + atol))}"
    vq.vq_rht_apply_output(yt, yt, st, M, N, dt)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(yt), host_bits(out))


@pytest.mark.parametrize("shards", [(4096, 1024, 1024), (14336, 14336), (64,), (2688, 192, 64)],
                         ids=lambda s: "+".join(map(str, s)))
@pytest.mark.parametrize("dt", [DT_F16, DT_BF16])
def test_rht_output_sharded(oracle, shards, dt):
    """Fused QKV / gate-up shards rotated in one launch: every shard bit-identical to a
    separate vq_rht_apply_output call on it, within the oracle's bound, and in place."""
    M, N = 3, sum(shards)
    y = make_x(M, N, dt, cfg_id=89)
    signs = make_signs(N, cfg_id=89)
    yt, st = dev(y), dev(signs)
    out = torch.empty_like(yt)
    vq.vq_rht_apply_output_sharded(yt, out, st, M, N, shards, dt)
    torch.cuda.synchronize()
    got_all = host_bits(out)
    o = 0
    for w in shards:
        part = yt[:, o:o + w].contiguous()
        alone = torch.empty_like(part)
        vq.vq_rht_apply_output(part, alone, st[o:o + w].contiguous(), M, w, dt)
        torch.cuda.synchronize()
        assert np.array_equal(host_bits(alone), got_all[:, o:o + w]), f"shard at {o}"
        ref = oracle.rht_out_f64(widen(y[:, o:o + w], dt), signs[o:o + w])
        ulp = np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64) if dt == DT_F16 else np.abs(ref) * 2.0 ** -7
        atol = 2 * np.log2(w) * 2.0 ** -24 * np.linalg.norm(widen(y[:, o:o + w], dt), axis=1, keepdims=True)
        err = np.abs(widen(got_all[:, o:o + w], dt) - ref)
        assert np.all(err <= ulp + atol), f"shard at {o}: max err/(ulp+atol) = {np.max(err / (ulp + atol))}"
        o += w
    vq.vq_rht_apply_output_sharded(yt, yt, st, M, N, shards, dt)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(yt), got_all)


def test_two_sided_rotation(oracle):
    """A layer stored as W_hat = R_out W R_in^T: forward_rotated with the input signs, then
    the output rotation, against the oracle's rotations around the exact W_hat product.
    The output rotation is orthogonal, so the per-row error norm is bounded by sqrt(N)
    times the per-element bound of the unrotated product, plus the final rounding."""
    N, K = 1024, 2048
    layer = make_layer(LayerSpec(N, K, FMT_VQ16, 64), cfg_id=78)
    L = layer_on_gpu(layer, DT_F16, 1)
    x = make_x(1, K, DT_F16, cfg_id=78)
    s_in, s_out = make_signs(K, cfg_id=78), make_signs(N, cfg_id=79)
    yh = L.forward_rotated(dev(x).view(torch.float16), dev(s_in))
    y = torch.empty_like(yh)
    vq.vq_rht_apply_output(yh, y, dev(s_out), 1, N, DT_F16)
    torch.cuda.synchronize()
    got = widen(host_bits(y), DT_F16)
    w, _ = oracle.dequant(layer)
    xr = oracle.rht(x, DT_F16, s_in)
    ref = oracle.rht_out_f64(xr @ w.T, s_out)
    tau = TOL * np.linalg.norm(xr) * np.abs(w).max()
    bound = np.sqrt(N) * tau + np.linalg.norm(0.5 * np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64))
    assert np.linalg.norm(got - ref) <= bound, f"{np.linalg.norm(got - ref)} > {bound}"

"""GPU parity of the sparse correction sidecar (orka README, "How it works": the decode is
scale x sum(codebook[index]) (+ sparse correction)): y = x (W + C)^T on every forward path,
the corrected materialised weights bit for bit, and the argument checks."""

import numpy as np
import pytest
import torch

import compressed_index_matmul_b200 as vq
from synth import (CONFIGS, DT_BF16, DT_F16, FMT_RVQ12, FMT_RVQ12_4, FMT_VQ16, FMT_VQ16_RVQ, LayerSpec,
                   make_correction, make_layer, make_signs, make_x)
from tests.gpu_util import assert_y_within, dev, host_bits, layer_on_gpu, require_gpu, run_forward, widen

pytestmark = pytest.mark.gpu
TOL = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _corrected(spec, cfg_id, density=0.01, tensor_id=0):
    layer = make_layer(spec, cfg_id=cfg_id, tensor_id=tensor_id)
    layer["corr"] = make_correction(spec.N, spec.K, density=density, cfg_id=cfg_id, tensor_id=tensor_id)
    return layer


def _check(oracle, layer, act, M, path, what, rows=None):
    L = layer_on_gpu(layer, act, M)
    assert L.launches(M) >= 2  # the correction's kernel, then the forward
    x = make_x(M, layer["spec"].K, act, cfg_id=77, seed=M)
    y = run_forward(L, x, act, path)
    vq.vq_linear_check(L.handle)
    y2 = run_forward(L, x, act, path)
    assert np.array_equal(y, y2), "not bit-identical run to run"
    if rows is not None:
        y = y[:, rows]
    w, _ = oracle.dequant(layer, rows=rows)
    assert_y_within(y, act, oracle.forward(layer, x, act, rows=rows), oracle.tolerance(x, act, w, TOL), what=what)
    return L, x


PATH_CASES = [
    # (N, K, fmt, scale_group, act, M, path)
    (512, 1024, FMT_RVQ12_4, 64, DT_BF16, 1, vq.VQ_PATH_LUT),      # table kernel, split-K reduction
    (256, 128, FMT_RVQ12, 64, DT_F16, 1, vq.VQ_PATH_LUT),          # table kernel, one slice (no split)
    (520, 1024, FMT_RVQ12, 1024, DT_F16, 1, vq.VQ_PATH_LUT),       # one scale per row
    (200, 576, FMT_RVQ12_4, 64, DT_F16, 3, vq.VQ_PATH_GEMV),       # warp-MMA GEMV
    (576, 1536, FMT_RVQ12_4, 64, DT_BF16, 16, vq.VQ_PATH_GEMV),    # GEMV with split-K tickets
    (256, 512, FMT_RVQ12_4, 64, DT_BF16, 64, vq.VQ_PATH_TC),       # tensor cores, one split, TMA stores
    (2040, 512, FMT_RVQ12_4, 64, DT_BF16, 300, vq.VQ_PATH_TC),     # K-split pair over a 2-CTA cluster
    (132, 576, FMT_RVQ12_4, 64, DT_F16, 20, vq.VQ_PATH_TC),        # N % 8 != 0: per-element stores
    (256, 8192, FMT_RVQ12_4, 64, DT_BF16, 32, vq.VQ_PATH_TC),      # several splits: last-CTA reduction
    (512, 2048, FMT_VQ16, 2048, DT_F16, 1, vq.VQ_PATH_GATHER),     # 16-bit gather kernel
    (512, 2048, FMT_VQ16, 2048, DT_F16, 4, vq.VQ_PATH_GATHER),
]


@pytest.mark.parametrize("case", PATH_CASES, ids=lambda c: f"{c[0]}x{c[1]}f{c[2]}a{c[4]}M{c[5]}p{c[6]}")
def test_correction_on_every_path(oracle, case):
    N, K, fmt, sg, act, M, path = case
    layer = _corrected(LayerSpec(N, K, fmt, sg), cfg_id=170, tensor_id=N + M)
    _check(oracle, layer, act, M, path, what=f"corrected path {path} M={M}")


@pytest.mark.parametrize("wdt", [DT_F16, DT_BF16])
@pytest.mark.parametrize("fmt", [FMT_RVQ12, FMT_RVQ12_4, FMT_VQ16])
def test_corrected_dequant_is_bit_exact(oracle, fmt, wdt):
    sg = 64 if fmt != FMT_VQ16 else 320  # the 16-bit format with one scale per row
    layer = _corrected(LayerSpec(72, 320, fmt, sg), cfg_id=171, density=0.05, tensor_id=fmt)
    L = layer_on_gpu(layer, DT_F16, 1)
    w = torch.empty((72, 320), dtype=torch.int16, device="cuda")
    vq.vq_debug_dequant(L.handle, L.planes, L.codebooks, L.t["scales"], w, wdt)
    torch.cuda.synchronize()
    _, want = oracle.dequant(layer, wdt)
    got = w.cpu().numpy().view(np.uint16)
    assert np.array_equal(got, want), f"{np.sum(got != want)} corrected weights differ"


def test_correction_edge_rows(oracle):
    """Rows without entries, a row corrected at every column, entries at both ends of K."""
    N, K = 64, 256
    layer = make_layer(LayerSpec(N, K, FMT_RVQ12_4, 64), cfg_id=172)
    rng = np.random.default_rng(172)
    cols = [np.zeros(0, np.int64) for _ in range(N)]
    cols[3] = np.arange(K)                      # every column
    cols[5] = np.array([0, K - 1])              # both ends
    cols[40] = np.sort(rng.choice(K, 17, replace=False))
    row_ptr = np.zeros(N + 1, np.int32)
    row_ptr[1:] = np.cumsum([len(c) for c in cols])
    col = np.concatenate(cols).astype(np.int32)
    val = (rng.standard_normal(len(col)) * 0.05).astype(np.float16).view(np.uint16)
    layer["corr"] = {"row_ptr": row_ptr, "col": col, "val": val}
    for M, path in ((1, vq.VQ_PATH_LUT), (5, vq.VQ_PATH_GEMV), (24, vq.VQ_PATH_TC)):
        _check(oracle, layer, DT_F16, M, path, what=f"edge rows M={M}")


def test_correction_with_no_entries_at_all(oracle):
    """A correction sidecar whose rows are all empty gives exactly the uncorrected result."""
    spec = LayerSpec(256, 512, FMT_RVQ12_4, 64)
    layer = make_layer(spec, cfg_id=173)
    plain = layer_on_gpu(layer, DT_BF16, 4)
    x = make_x(4, spec.K, DT_BF16, cfg_id=173)
    y0 = run_forward(plain, x, DT_BF16, vq.VQ_PATH_GEMV)
    layer["corr"] = {"row_ptr": np.zeros(spec.N + 1, np.int32), "col": np.zeros(0, np.int32),
                     "val": np.zeros(0, np.uint16)}
    corrected = layer_on_gpu(layer, DT_BF16, 4)
    assert np.array_equal(run_forward(corrected, x, DT_BF16, vq.VQ_PATH_GEMV), y0)


@pytest.mark.parametrize("M", [1, 16])
def test_correction_llama_gate_sampled(oracle, M):
    """The Llama-3-8B gate shape with a 0.1 % correction, on the kernel the automatic choice
    takes (table kernel at M = 1, tensor cores at M = 16), sampled rows."""
    spec = CONFIGS[4]["tensors"][0][1]
    layer = _corrected(spec, cfg_id=4, density=0.001)
    rows = np.sort(np.random.default_rng(M).choice(spec.N, 128, replace=False)).astype(np.int32)
    _check(oracle, layer, DT_BF16, M, vq.VQ_PATH_AUTO, what=f"llama gate corrected M={M}", rows=rows)


def test_correction_with_the_rotated_forward(oracle):
    """A rotated 16-bit layer with a correction: vq_linear_forward_rotated takes the unfused
    route (rotation into the handle's buffer, rounded to fp16, then the corrected forward)."""
    N, K = 512, 1024
    layer = _corrected(LayerSpec(N, K, FMT_VQ16, K), cfg_id=174, density=0.01)
    L = vq.VQLinear(N, K, FMT_VQ16, K, DT_F16, 1, layer, rht=1)
    assert L.corr == 1
    signs = make_signs(K, cfg_id=174)
    x = make_x(1, K, DT_F16, cfg_id=174)
    y = host_bits(L.forward_rotated(dev(x).view(torch.float16), torch.from_numpy(signs).cuda()))
    torch.cuda.synchronize()
    x_rot = oracle.round_to(oracle.rht(x, DT_F16, signs), DT_F16)
    w, _ = oracle.dequant(layer)
    assert_y_within(y, DT_F16, oracle.forward(layer, x_rot, DT_F16), oracle.tolerance(x_rot, DT_F16, w, TOL),
                    what="rotated with a correction")


def test_correction_argument_errors():
    N, K = 64, 256
    spec = LayerSpec(N, K, FMT_RVQ12_4, 64)
    layer = _corrected(spec, cfg_id=175, density=0.05)
    L = layer_on_gpu(layer, DT_F16, 2)
    x = torch.zeros((1, K), dtype=torch.float16, device="cuda")
    y = torch.empty((1, N), dtype=torch.float16, device="cuda")
    # a handle made for corrections needs them on every forward
    bare = vq.make_planes(L.t["lo"], L.t["hi4"], L.t["s2"])
    with pytest.raises(vq.VQError) as ei:
        vq.vq_linear_forward(L.handle, x, bare, L.codebooks, L.t["scales"], y, 1, N, K)
    assert ei.value.status == vq._binding.VQ_ERR_INVALID_ARG
    # and a handle made without them refuses them
    plain = layer_on_gpu(make_layer(spec, cfg_id=175), DT_F16, 2)
    with pytest.raises(vq.VQError) as ei:
        vq.vq_linear_forward(plain.handle, x, L.planes, plain.codebooks, plain.t["scales"], y, 1, N, K)
    assert ei.value.status == vq._binding.VQ_ERR_INVALID_ARG
    # the allocation-free call has no buffer for the correction
    with pytest.raises(vq.VQError) as ei:
        vq.vq_linear_forward_noalloc(N, K, FMT_RVQ12_4, 64, DT_F16, x, L.planes, L.codebooks, L.t["scales"], y, 1,
                                     corr=1)
    assert ei.value.status == vq._binding.VQ_ERR_UNSUPPORTED
    # the residual ladder has no correction
    with pytest.raises(vq.VQError) as ei:
        vq.vq_linear_create(N, K, FMT_VQ16_RVQ, 64, DT_F16, 1, n16=2, n8=0, mult=(0.1,), corr=1)
    assert ei.value.status == vq._binding.VQ_ERR_UNSUPPORTED

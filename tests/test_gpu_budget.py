"""GPU tests of vq_linear_set_sm_budget: the batch-1 table kernel on a subset of the
SMs, alone and as two independent forwards running concurrently on two streams.

Each budget changes only how the (slice, row) work and the reduction are split
over CTAs, so y must stay within the oracle's tolerance and be bit-identical run
to run for a given budget."""

import numpy as np
import pytest
import torch

import compressed_index_matmul_b200 as vq
from synth import CONFIGS, DT_BF16, FMT_RVQ12, FMT_RVQ12_4, LayerSpec, make_layer, make_x
from tests.gpu_util import assert_y_within, dev, host_bits, layer_on_gpu, require_gpu

pytestmark = pytest.mark.gpu
TOL = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


@pytest.mark.parametrize("shape", [(1000, 4096, FMT_RVQ12_4, 64), (2052, 2048, FMT_RVQ12, 2048)],
                         ids=lambda s: f"{s[0]}x{s[1]}f{s[2]}")
def test_budget_keeps_parity(oracle, shape):
    N, K, fmt, sg = shape
    layer = make_layer(LayerSpec(N, K, fmt, sg), cfg_id=61, tensor_id=N)
    L = layer_on_gpu(layer, DT_BF16, 1)
    L.set_path(vq.VQ_PATH_LUT)
    xb = make_x(1, K, DT_BF16, cfg_id=61)
    x = dev(xb).view(torch.bfloat16)
    y_ref = oracle.forward(layer, xb, DT_BF16)
    w, _ = oracle.dequant(layer)
    tol = oracle.tolerance(xb, DT_BF16, w, TOL)
    for budget in (1, 7, 37, _sms() // 2, _sms(), 0):
        L.set_sm_budget(budget)
        y1 = host_bits(L.forward(x))
        y2 = host_bits(L.forward(x))
        vq.vq_linear_check(L.handle)
        assert_y_within(y1, DT_BF16, y_ref, tol, what=f"budget {budget}")
        assert np.array_equal(y1, y2), f"budget {budget}: not bit-identical run to run"


def test_budget_rejects_out_of_range():
    layer = make_layer(LayerSpec(256, 256, FMT_RVQ12, 64), cfg_id=61)
    L = layer_on_gpu(layer, DT_BF16, 1)
    for bad in (-1, _sms() + 1):
        with pytest.raises(vq.VQError) as ei:
            L.set_sm_budget(bad)
        assert ei.value.status == vq._binding.VQ_ERR_INVALID_ARG


def test_gate_and_up_concurrently_on_sm_halves(oracle):
    """The Llama-3-8B gate and up projections read the same x; on disjoint halves of the
    SMs they run at the same time on two streams and each matches the oracle (sampled
    rows) and its own sequential result bit for bit."""
    half = _sms() // 2
    layers, Ls = [], []
    for tid, (label, spec) in enumerate(CONFIGS[4]["tensors"][:2]):
        layer = make_layer(spec, cfg_id=4, tensor_id=tid)
        L = layer_on_gpu(layer, DT_BF16, 1)
        L.set_sm_budget(half)
        layers.append(layer)
        Ls.append(L)
    K = Ls[0].K
    xb = make_x(1, K, DT_BF16, cfg_id=62)
    x = dev(xb).view(torch.bfloat16)
    seq = [host_bits(L.forward(x)) for L in Ls]
    torch.cuda.synchronize()
    main, side = torch.cuda.current_stream(), torch.cuda.Stream()
    ys = [torch.empty((1, L.N), dtype=torch.bfloat16, device="cuda") for L in Ls]
    for _ in range(3):
        side.wait_stream(main)
        with torch.cuda.stream(side):
            Ls[1].forward(x, ys[1])
        Ls[0].forward(x, ys[0])
        main.wait_stream(side)
    torch.cuda.synchronize()
    for L in Ls:
        vq.vq_linear_check(L.handle)
    rows = np.sort(np.random.default_rng(5).choice(Ls[0].N, 256, replace=False)).astype(np.int32)
    for layer, L, y, y_seq in zip(layers, Ls, ys, seq):
        got = host_bits(y)
        assert np.array_equal(got, y_seq), "concurrent result differs from the sequential one"
        y_ref = oracle.forward(layer, xb, DT_BF16, rows=rows)
        w, _ = oracle.dequant(layer, rows=rows)
        assert_y_within(got[:, rows], DT_BF16, y_ref, oracle.tolerance(xb, DT_BF16, w, TOL),
                        what="concurrent")


def test_table_kernel_beside_a_busy_stream(oracle):
    """The batch-1 table kernel meets all of its CTAs at a grid barrier.  While a kernel on
    another stream holds an SM for longer than the barrier's bounded wait (about 1 s), the
    cooperative launch must still bring every CTA in (it starts when the SM frees up), so
    the forward completes without a timeout and matches the oracle; the default budgets
    (every SM) are used, and budgets that overlap the busy SM are also exercised."""
    spec = CONFIGS[4]["tensors"][0][1]  # 14336 x 4096, 32 K-slices
    layer = make_layer(spec, cfg_id=4, tensor_id=0)
    L = layer_on_gpu(layer, DT_BF16, 1)
    L.set_path(vq.VQ_PATH_LUT)
    xb = make_x(1, spec.K, DT_BF16, cfg_id=63)
    x = dev(xb).view(torch.bfloat16)
    y_alone = host_bits(L.forward(x))
    torch.cuda.synchronize()
    clock_hz = 1.965e9  # the B200's maximum SM clock: at any lower clock the sleep only lasts longer
    main, side = torch.cuda.current_stream(), torch.cuda.Stream()
    y = torch.empty((1, L.N), dtype=torch.bfloat16, device="cuda")
    side.wait_stream(main)
    with torch.cuda.stream(side):
        torch.cuda._sleep(int(1.5 * clock_hz))  # one CTA holding one SM for ~1.5 s
    L.forward(x, y)
    torch.cuda.synchronize()
    vq.vq_linear_check(L.handle)  # raises VQError(VQ_ERR_TIMEOUT) if the barrier gave up
    got = host_bits(y)
    assert np.array_equal(got, y_alone), "result beside the busy stream differs from the result alone"
    rows = np.sort(np.random.default_rng(7).choice(spec.N, 128, replace=False)).astype(np.int32)
    w, _ = oracle.dequant(layer, rows=rows)
    assert_y_within(got[:, rows], DT_BF16, oracle.forward(layer, xb, DT_BF16, rows=rows),
                    oracle.tolerance(xb, DT_BF16, w, TOL), what="beside a busy stream")

"""Failure detection without faulting the GPU.

- A bounded device-side wait that nothing completes gives up after about a second,
  sets the handle's error flag and ends normally: vq_linear_check reports
  VQ_ERR_TIMEOUT, and the same context then runs a correct forward.
- Allocation failure is injected on the host (VQ_TEST_FAIL_ALLOC=1) and reported
  as VQ_ERR_NOMEM, with no handle left behind."""

import os
import time

import numpy as np
import pytest

import compressed_index_matmul_b200 as vq
from synth import DT_F16, FMT_RVQ12_4, LayerSpec, make_layer, make_x
from tests.gpu_util import assert_y_within, layer_on_gpu, require_gpu, run_forward

pytestmark = pytest.mark.gpu
VQ_ERR_NOMEM, VQ_ERR_TIMEOUT = 4, 5


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def test_bounded_wait_gives_up_and_the_context_survives(oracle):
    layer = make_layer(LayerSpec(256, 512, FMT_RVQ12_4, 64), cfg_id=95)
    L = layer_on_gpu(layer, DT_F16, 32)
    t0 = time.monotonic()
    vq.vq_debug_wait_timeout(L.handle)
    with pytest.raises(vq.VQError) as ei:
        vq.vq_linear_check(L.handle)
    waited = time.monotonic() - t0
    assert ei.value.status == VQ_ERR_TIMEOUT
    assert 0.3 < waited < 10.0, f"the wait gave up after {waited:.2f} s"
    vq.vq_linear_check(L.handle)  # the flag was cleared
    # the context is still usable: every path gives a correct result afterwards
    x = make_x(32, 512, DT_F16, cfg_id=95)
    w, _ = oracle.dequant(layer)
    for path, M in ((vq.VQ_PATH_TC, 32), (vq.VQ_PATH_GEMV, 4), (vq.VQ_PATH_LUT, 1)):
        y = run_forward(L, x[:M], DT_F16, path)
        vq.vq_linear_check(L.handle)
        assert_y_within(y, DT_F16, oracle.forward(layer, x[:M], DT_F16), oracle.tolerance(x[:M], DT_F16, w, 2e-3),
                        what=f"after the timeout, path {path}")


def test_allocation_failure_is_reported():
    os.environ["VQ_TEST_FAIL_ALLOC"] = "1"
    try:
        with pytest.raises(vq.VQError) as ei:
            vq.vq_linear_create(256, 512, FMT_RVQ12_4, 64, DT_F16, 4)
        assert ei.value.status == VQ_ERR_NOMEM
        assert "VQ_TEST_FAIL_ALLOC" in str(ei.value)
    finally:
        del os.environ["VQ_TEST_FAIL_ALLOC"]
    h = vq.vq_linear_create(256, 512, FMT_RVQ12_4, 64, DT_F16, 4)
    vq.vq_linear_destroy(h)

"""GPU test of vq_linear_forward_noalloc: the handle-free forward that takes its
split-K scratch from a fixed in-library buffer instead of allocating.

It must give, bit for bit, what vq_linear_forward gives on the same (warp-MMA GEMV)
path, call after call (the buffer's counters must be back at zero after every call), and
refuse shapes whose scratch would not fit.  The file name puts it last in
collection, so it also runs after every other GPU test in one process."""

import numpy as np
import pytest
import torch

import compressed_index_matmul_b200 as vq
from synth import DT_BF16, DT_F16, FMT_RVQ12, FMT_RVQ12_4, FMT_VQ16, LayerSpec, make_layer, make_x
from tests.gpu_util import assert_y_within, dev, host_bits, layer_on_gpu, require_gpu

pytestmark = pytest.mark.gpu
TOL = 2e-3

CASES = [
    # (N, K, fmt, scale_group, act, M): each plan splits K, so the scratch and tickets are used
    (576, 1536, FMT_RVQ12_4, 64, DT_BF16, 16),
    (1000, 4096, FMT_RVQ12, 64, DT_F16, 5),
    (520, 2048, FMT_VQ16, 2048, DT_F16, 1),
]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _noalloc(L, x, M):
    y = torch.empty((M, L.N), dtype=x.dtype, device=x.device)
    vq.vq_linear_forward_noalloc(L.N, L.K, L.fmt, L.scale_group, L.act_dtype, x, L.planes, L.codebooks,
                                 L.t["scales"], y, M)
    return y


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}x{c[1]}f{c[2]}M{c[5]}")
def test_noalloc_matches_forward_twice(oracle, case):
    N, K, fmt, sg, act, M = case
    layer = make_layer(LayerSpec(N, K, fmt, sg), cfg_id=90, tensor_id=N)
    L = layer_on_gpu(layer, act, 16)
    L.set_path(vq.VQ_PATH_GEMV)
    assert L.launches(M) == 1
    xb = make_x(M, K, act, cfg_id=90, seed=M)
    x = dev(xb).view(torch.bfloat16 if act == DT_BF16 else torch.float16)
    y_ref = host_bits(L.forward(x))
    torch.cuda.synchronize()
    w, _ = oracle.dequant(layer)
    tol = oracle.tolerance(xb, act, w, TOL)
    want = oracle.forward(layer, xb, act)
    for call in range(2):
        y = host_bits(_noalloc(L, x, M))
        torch.cuda.synchronize()
        # the same kernel with the same plan: the same splits, summed in the same order
        assert np.array_equal(y, y_ref), f"call {call}: not bit-identical to vq_linear_forward"
        assert_y_within(y, act, want, tol, what=f"noalloc call {call}")


def test_noalloc_rejects_what_does_not_fit():
    # splits x M x N x 4 bytes = 16 x 16 x 8192 x 4 = 8 MiB of partial sums > the 4 MiB buffer
    N, K, M = 8192, 32768, 16
    x = torch.zeros((M, 64), dtype=torch.float16, device="cuda")   # only checked for NULL / alignment:
    y = torch.zeros((M, 64), dtype=torch.float16, device="cuda")   # the call fails before any launch
    b = torch.zeros(64, dtype=torch.uint8, device="cuda")
    planes = vq.make_planes(b, b, b)
    cbs = vq.make_codebooks(b, b)
    with pytest.raises(vq.VQError) as ei:
        vq.vq_linear_forward_noalloc(N, K, FMT_RVQ12_4, 64, DT_F16, x, planes, cbs, b, y, M)
    assert ei.value.status == 2 and "4194304" in str(ei.value)
    with pytest.raises(vq.VQError) as ei:
        vq.vq_linear_forward_noalloc(256, 256, FMT_RVQ12_4, 64, DT_F16, x, planes, cbs, b, y, 17)
    assert ei.value.status == 1

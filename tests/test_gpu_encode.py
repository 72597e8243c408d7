"""GPU parity of the nearest-entry encoder (vq_encode; orka README, "How it works":
encode -> nearest-entry index per group, stored as bit-planes).

The encoder decides integers from binary32 distances, so its reference is the oracle's
encoder taking the same decisions in binary32 (pinned bit for bit against numpy float32
and against the fp64 definition in tests/test_oracle_pins.py): the planes must match
byte for byte.  Exact codewords must encode back to their own indices."""

import numpy as np
import pytest
import torch

import compressed_index_matmul_b200 as vq
from synth import DT_F16, FMT_RVQ12, FMT_RVQ12_4, FMT_VQ16, LayerSpec, make_layer, make_x
from tests.gpu_util import assert_y_within, dev, layer_on_gpu, require_gpu, run_forward

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _encode_gpu(layer, w):
    spec = layer["spec"]
    N, K, G = spec.N, spec.K, spec.K // 8
    out = {}
    if spec.fmt == FMT_VQ16:
        out["idx16"] = torch.zeros(N * G, dtype=torch.int16, device="cuda")
    else:
        out["lo"] = torch.zeros(N * G, dtype=torch.uint8, device="cuda")
        out["hi4"] = torch.zeros(N * G // 2, dtype=torch.uint8, device="cuda")
        if spec.fmt == FMT_RVQ12_4:
            out["s2"] = torch.zeros(N * G // 2, dtype=torch.uint8, device="cuda")
    cb1, cb2 = dev(layer["cb1"]), (dev(layer["cb2"]) if "cb2" in layer else None)
    cbs = vq.make_codebooks(cb1, cb2)
    sc = dev(layer["scales"])
    wt = torch.from_numpy(np.ascontiguousarray(w, dtype=np.float32)).cuda()
    vq.vq_encode(N, K, spec.fmt, spec.scale_group, wt, sc, cbs, out.get("lo"), out.get("hi4"), out.get("s2"),
                 out.get("idx16"))
    torch.cuda.synchronize()
    del cb1, cb2, sc, wt  # alive until the encoder finished
    res = {k: v.cpu().numpy() for k, v in out.items()}
    if "idx16" in res:
        res["idx16"] = res["idx16"].view(np.uint16)
    return res


CASES = [
    # (fmt, N, K, scale_group)
    (FMT_RVQ12, 16, 448, 64),     # 3 full slices and a 64-wide tail
    (FMT_RVQ12, 8, 256, 256),     # one scale per row
    (FMT_RVQ12_4, 16, 256, 64),   # two stages
    (FMT_VQ16, 4, 128, 128),      # the 65,536-entry table through L2
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"f{c[0]}-{c[1]}x{c[2]}sg{c[3]}")
def test_encode_matches_the_binary32_oracle(oracle, case):
    fmt, N, K, sg = case
    layer = make_layer(LayerSpec(N, K, fmt, sg), cfg_id=140, tensor_id=fmt)
    w = (np.random.default_rng(140 + fmt).standard_normal((N, K)) * 0.02).astype(np.float32)
    ref = oracle.encode(layer["spec"], w.astype(np.float64), layer["scales"], layer["cb1"], layer.get("cb2"),
                        precision="f32")
    got = _encode_gpu(layer, w)
    for k, v in got.items():
        assert np.array_equal(v, ref[k]), f"{k}: {np.sum(v != ref[k])} entries differ"


@pytest.mark.parametrize("fmt", [FMT_RVQ12, FMT_RVQ12_4])
def test_encode_round_trips_exact_codewords(oracle, fmt):
    """W = s (c1 [+ c2]) exactly (binary32 values) encodes back to the layer's own planes;
    for two stages the stage-2 codebook is made small against the stage-1 spacing."""
    layer = make_layer(LayerSpec(24, 320, fmt, 64), cfg_id=141, tensor_id=fmt)
    if fmt == FMT_RVQ12_4:
        small = (layer["cb2"].view(np.float16).astype(np.float32) * np.float32(1e-3)).astype(np.float16)
        layer["cb2"] = small.view(np.uint16)
    w, _ = oracle.dequant(layer)
    w32 = w.astype(np.float32)
    if fmt == FMT_RVQ12:  # s * c1 (two fp16 values) is exact in binary32: the true entry is at distance 0
        assert np.array_equal(w32.astype(np.float64), w)
    # with two stages w is rounded to binary32; the true entries stay far nearer than any other
    got = _encode_gpu(layer, w32)
    ref = oracle.encode(layer["spec"], w32.astype(np.float64), layer["scales"], layer["cb1"], layer.get("cb2"),
                        precision="f32")
    for k, v in got.items():
        assert np.array_equal(ref[k], layer[k]), f"oracle {k}"
        assert np.array_equal(v, layer[k]), k


def test_encoded_layer_runs_forward(oracle):
    """Encode a dense W on the GPU, then run the forward on the planes it wrote: the result
    matches the oracle forward of the oracle's own encoding."""
    N, K = 64, 256
    layer = make_layer(LayerSpec(N, K, FMT_RVQ12_4, 64), cfg_id=142)
    w = (np.random.default_rng(142).standard_normal((N, K)) * 0.02).astype(np.float32)
    enc = dict(layer)
    enc.update(_encode_gpu(layer, w))
    ref_layer = oracle.encode(layer["spec"], w.astype(np.float64), layer["scales"], layer["cb1"], layer["cb2"],
                              precision="f32")
    for k in ("lo", "hi4", "s2"):
        assert np.array_equal(enc[k], ref_layer[k]), k
    L = layer_on_gpu(enc, DT_F16, 4)
    x = make_x(4, K, DT_F16, cfg_id=142)
    y = run_forward(L, x, DT_F16)
    wx, _ = oracle.dequant(ref_layer)
    assert_y_within(y, DT_F16, oracle.forward(ref_layer, x, DT_F16), oracle.tolerance(x, DT_F16, wx, 2e-3),
                    what="encoded layer forward")

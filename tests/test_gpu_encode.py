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


# --------------------------------------------------------------------------------------------
# The encoder against the fp64 definition (orka README, "How it works": the nearest entry per
# group).  The GPU decides with binary32 distances, so where two entries are closer than the
# binary32 error of the distances it may pick either: its entry must equal the fp64 nearest one
# wherever the fp64 gap to the runner-up exceeds twice that error, and lie within twice the
# error of the nearest distance elsewhere.  Stage 2 is checked the same way against the fp64
# greedy choice given the GPU's own stage-1 entry.

U32 = 2.0 ** -24


def _group_scales(oracle, layer):
    """Scale of every group [N, G], read back through the oracle's decode of a unit codebook
    (cb1 = 1.0 everywhere, no stage 2: each decoded weight is its scale exactly)."""
    unit = dict(layer)
    unit["cb1"] = np.full_like(layer["cb1"], 0x3C00)
    if "cb2" in unit:
        unit["cb2"] = np.zeros_like(layer["cb2"])
    w, _ = oracle.dequant(unit)
    return w[:, ::8]


def _cb(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64).reshape(-1, 8)


def _dist64(w8, s, c8):
    """sum_j (w_j - s c_j)^2 in fp64, per row of the [n, 8] arrays."""
    e = w8 - s[:, None] * c8
    return (e * e).sum(axis=1)


def _bound(w8, s, c8, stages):
    """Twice a bound on |binary32 distance - fp64 distance| (each product, difference, square and
    sum rounded once; a two-stage codeword adds the rounding of c1 + c2)."""
    a = np.abs(w8) + np.abs(s[:, None] * c8)
    return 2.0 * (16.0 + 4.0 * (stages - 1)) * U32 * (a * a).sum(axis=1)


def _nearest64(w8, s, C, chunk=128):
    """fp64 nearest and runner-up entries of C [E, 8] for each group of w8 [n, 8] (scale s [n])."""
    best = np.empty((len(w8), 2), np.int64)
    cc = (C * C).sum(axis=1)
    for a in range(0, len(w8), chunk):
        ww, ss = w8[a:a + chunk], s[a:a + chunk]
        d = (ww * ww).sum(axis=1)[:, None] - 2.0 * ss[:, None] * (ww @ C.T) + (ss * ss)[:, None] * cc[None, :]
        two = np.argpartition(d, 1, axis=1)[:, :2]
        # order the pair by their exact distances (ties: the smaller index, as the definition)
        d0 = _dist64(ww, ss, C[two[:, 0]])
        d1 = _dist64(ww, ss, C[two[:, 1]])
        swap = (d1 < d0) | ((d1 == d0) & (two[:, 1] < two[:, 0]))
        best[a:a + chunk, 0] = np.where(swap, two[:, 1], two[:, 0])
        best[a:a + chunk, 1] = np.where(swap, two[:, 0], two[:, 1])
    return best


def _check_against_fp64(oracle, layer, w, got, sample=None):
    spec = layer["spec"]
    enc = dict(layer)
    enc.update(got)
    i1, i2 = oracle.unpack(enc)
    s = _group_scales(oracle, layer)
    wg = np.asarray(w, np.float64).reshape(spec.N, spec.G, 8)
    n_idx, g_idx = (np.unravel_index(sample, (spec.N, spec.G)) if sample is not None
                    else np.unravel_index(np.arange(spec.N * spec.G), (spec.N, spec.G)))
    w8, sv = wg[n_idx, g_idx], s[n_idx, g_idx]
    C1 = _cb(layer["cb1"])
    gpu1 = i1[n_idx, g_idx].astype(np.int64)
    ref = _nearest64(w8, sv, C1)
    d_gpu = _dist64(w8, sv, C1[gpu1])
    d_best, d_next = _dist64(w8, sv, C1[ref[:, 0]]), _dist64(w8, sv, C1[ref[:, 1]])
    tol = np.maximum(_bound(w8, sv, C1[gpu1], 1), _bound(w8, sv, C1[ref[:, 0]], 1))
    clear = d_next - d_best > tol
    assert np.array_equal(gpu1[clear], ref[clear, 0]), \
        f"stage 1: {np.sum(gpu1[clear] != ref[clear, 0])} of {clear.sum()} clear-cut groups differ"
    assert (d_gpu - d_best <= tol).all(), "stage 1: an entry farther than the binary32 error from the nearest"
    if spec.fmt == FMT_RVQ12_4:
        C2 = _cb(layer["cb2"])
        c1 = C1[gpu1]
        d2 = np.stack([_dist64(w8, sv, c1 + C2[t]) for t in range(16)], axis=1)
        ref2 = np.argmin(d2, axis=1)  # first minimum: equal distances go to the smaller index
        srt = np.sort(d2, axis=1)
        gpu2 = i2[n_idx, g_idx].astype(np.int64)
        tol2 = np.maximum(_bound(w8, sv, c1 + C2[gpu2], 2), _bound(w8, sv, c1 + C2[ref2], 2))
        clear2 = srt[:, 1] - srt[:, 0] > tol2
        assert np.array_equal(gpu2[clear2], ref2[clear2]), \
            f"stage 2: {np.sum(gpu2[clear2] != ref2[clear2])} of {clear2.sum()} clear-cut groups differ"
        assert (d2[np.arange(len(gpu2)), gpu2] - srt[:, 0] <= tol2).all(), "stage 2: beyond the error bound"
    return int(clear.sum()), len(clear)


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"f{c[0]}-{c[1]}x{c[2]}sg{c[3]}")
def test_encode_agrees_with_the_fp64_definition(oracle, case):
    fmt, N, K, sg = case
    layer = make_layer(LayerSpec(N, K, fmt, sg), cfg_id=140, tensor_id=fmt)
    w = (np.random.default_rng(140 + fmt).standard_normal((N, K)) * 0.02).astype(np.float32)
    got = _encode_gpu(layer, w)
    clear, total = _check_against_fp64(oracle, layer, w, got)
    assert clear >= 0.99 * total


@pytest.mark.parametrize("fmt", [FMT_RVQ12_4, FMT_VQ16])
def test_encode_layer_size_sampled(oracle, fmt):
    """A whole 4096 x 4096 layer (block-64 scales for the two-stage format, one scale per row
    for the 65,536-entry table), checked on 1024 sampled groups against the fp64 definition."""
    sg = 64 if fmt == FMT_RVQ12_4 else 4096
    layer = make_layer(LayerSpec(4096, 4096, fmt, sg), cfg_id=143, tensor_id=fmt)
    w = (np.random.default_rng(143 + fmt).standard_normal((4096, 4096)) * 0.02).astype(np.float32)
    got = _encode_gpu(layer, w)
    sample = np.random.default_rng(fmt).choice(4096 * 512, size=1024, replace=False)
    clear, total = _check_against_fp64(oracle, layer, w, got, sample)
    assert clear >= 0.99 * total

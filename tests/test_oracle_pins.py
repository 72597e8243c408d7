"""Pins for the CPU oracle against facts that do not come from the oracle itself.

Each test fixes one part of the oracle to something independent: an exhaustive
comparison with numpy/torch IEEE conversions, hand-worked golden values, a
brute-force dense matmul written separately here, the Sylvester Hadamard matrix
from scipy, or an algebraic identity (one-hot columns, linearity, involution).
"""

import json
import os

import numpy as np
import pytest
import scipy.linalg
import torch

from synth import (FMT_RVQ12, FMT_RVQ12_4, FMT_VQ16, FMT_VQ16_RVQ, DT_BF16, DT_F16, LayerSpec, f32_to_bf16_bits,
                   make_correction,
                   make_layer, make_x)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------- converters

def test_f16_decode_exhaustive(oracle):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.decode(bits, DT_F16)
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    # signed zeros keep their sign
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))


def test_f16_round_trip_exhaustive(oracle):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = bits.view(np.float16).astype(np.float64)
    keep = ~np.isnan(vals)
    assert np.array_equal(oracle.round_to(vals[keep], DT_F16), bits[keep])


def test_f16_round_matches_numpy_on_doubles(oracle):
    rng = np.random.default_rng(1)
    mag = np.exp2(rng.uniform(-30, 17, size=200_000))
    v = mag * rng.choice([-1.0, 1.0], size=mag.size)
    v = np.concatenate([v, rng.standard_normal(50_000) * 1e-6])
    ours = oracle.round_to(v, DT_F16)
    ref = v.astype(np.float16).view(np.uint16)  # numpy rounds double -> half directly (RN-even)
    assert np.array_equal(ours, ref)


def test_f16_ties_and_limits_by_hand(oracle):
    cases = {
        1.0 + 2.0 ** -11: 0x3C00,         # halfway between 1 and 1+2^-10 -> even (1.0)
        1.0 + 3 * 2.0 ** -11: 0x3C02,     # halfway between 1+2^-10 and 1+2^-9 -> even
        65504.0: 0x7BFF,                  # largest finite
        65519.99: 0x7BFF,
        65520.0: 0x7C00,                  # halfway to 2^16 rounds to even = inf
        2.0 ** -24: 0x0001,               # smallest subnormal
        2.0 ** -25: 0x0000,               # halfway to zero -> even (0)
        3 * 2.0 ** -25: 0x0002,           # halfway between 1 and 2 subnormal steps -> even
        -2.0 ** -14: 0x8400,              # smallest normal, negative
        -0.0: 0x8000,
    }
    got = oracle.round_to(np.array(list(cases.keys())), DT_F16)
    assert [int(g) for g in got] == list(cases.values())


def test_bf16_decode_exhaustive(oracle):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.decode(bits, DT_BF16)
    ref = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_bf16_round_matches_torch(oracle):
    rng = np.random.default_rng(2)
    f = (np.exp2(rng.uniform(-130, 127, size=200_000)) * rng.choice([-1.0, 1.0], size=200_000)).astype(np.float32)
    f = np.concatenate([f, rng.standard_normal(50_000).astype(np.float32)])
    ours = oracle.round_to(f.astype(np.float64), DT_BF16)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_fl32_matches_numpy(oracle):
    rng = np.random.default_rng(3)
    v = np.exp2(rng.uniform(-140, 120, size=2000)) * rng.choice([-1.0, 1.0], size=2000)
    for a in v:
        assert oracle.fl32(a) == float(np.float32(a))


# --------------------------------------------------------------------------- unpack

def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_unpack_golden_layout(oracle):
    # K=32: a single slice, so the sliced order equals the row-major order of the fixture
    g = _golden("unpack_layout.json")
    spec = LayerSpec(g["N"], g["K"], FMT_RVQ12_4, 32)
    layer = {"spec": spec, "lo": np.array(g["lo"], np.uint8).ravel(), "hi4": np.array(g["hi4"], np.uint8).ravel(),
             "s2": np.array(g["s2"], np.uint8).ravel()}
    i1, i2 = oracle.unpack(layer)
    assert i1.tolist() == g["i1"]
    assert i2.tolist() == g["i2"]


def _slices(G):
    """(first group, width) of every 16-group slice of a row of G groups."""
    return [(g0, min(16, G - g0)) for g0 in range(0, G, 16)]


def to_sliced(a2d: np.ndarray, per_group: float) -> np.ndarray:
    """Row-major [N][G*per_group] -> flat K-slice-major order (written from the layout description)."""
    N, E = a2d.shape
    G = int(round(E / per_group))
    out = []
    for g0, w in _slices(G):
        e0, e1 = int(g0 * per_group), int((g0 + w) * per_group)
        out.append(a2d[:, e0:e1].reshape(-1))
    return np.concatenate(out)


def from_sliced(flat: np.ndarray, N: int, G: int, per_group: float) -> np.ndarray:
    """Inverse of to_sliced."""
    cols = []
    pos = 0
    for g0, w in _slices(G):
        e = int(w * per_group)
        cols.append(flat[pos:pos + N * e].reshape(N, e))
        pos += N * e
    return np.concatenate(cols, axis=1)


def _pack12(i1, i2=None):
    """Pack indices [N][G] into the plane format (written here from the layout description)."""
    N, G = i1.shape
    lo = (i1 & 0xFF).astype(np.uint8)
    hi = (i1 >> 8).astype(np.uint8)
    hi4 = (hi[:, 0::2] | (hi[:, 1::2] << 4)).astype(np.uint8)
    out = {"lo": to_sliced(lo, 1), "hi4": to_sliced(hi4, 0.5)}
    if i2 is not None:
        out["s2"] = to_sliced((i2[:, 0::2] | (i2[:, 1::2] << 4)).astype(np.uint8), 0.5)
    return out


def test_slice_layout_golden(oracle):
    g = _golden("slice_layout.json")
    for case in g["cases"]:
        N, K = case["N"], case["K"]
        G = K // 8
        layer = {"spec": LayerSpec(N, K, FMT_RVQ12, K), "lo": (np.arange(N * G) % 256).astype(np.uint8),
                 "hi4": (np.arange(N * G // 2) % 256).astype(np.uint8)}
        i1, _ = oracle.unpack(layer)
        for n, grp, expect in case["checks"]:
            assert int(i1[n, grp]) == expect, (K, n, grp)


def test_scale_layout_by_hand(oracle):
    """Block scales follow the planes' slice order: K=192 (slices of 16 and 8 groups), N=2,
    scale_group=64 -> per row 2 scales in slice 0 and 1 in slice 1; storage order
    [r0b0, r0b1, r1b0, r1b1, r0b2, r1b2].  With cb1 entry 0 = all ones and index 0
    everywhere, W[n][k] equals the scale of (n, k)."""
    N, K = 2, 192
    vals = np.array([1, 2, 3, 4, 5, 6], np.float16)
    cb1 = np.zeros((4096, 8), np.float16)
    cb1[0] = 1
    layer = {"spec": LayerSpec(N, K, FMT_RVQ12, 64), "lo": np.zeros(N * K // 8, np.uint8),
             "hi4": np.zeros(N * K // 16, np.uint8), "cb1": cb1.view(np.uint16), "scales": vals.view(np.uint16)}
    w, _ = oracle.dequant(layer)
    expect = {(0, 0): 1, (0, 64): 2, (1, 0): 3, (1, 127): 4, (0, 128): 5, (1, 191): 6}
    for (n, k), v in expect.items():
        assert w[n, k] == v, (n, k)


def test_layout_helpers_round_trip():
    rng = np.random.default_rng(9)
    for N, G in ((3, 16), (5, 48), (4, 24), (2, 8)):
        a = rng.integers(0, 256, size=(N, G), dtype=np.uint8)
        assert np.array_equal(from_sliced(to_sliced(a, 1), N, G, 1), a)
        h = rng.integers(0, 256, size=(N, G // 2), dtype=np.uint8)
        assert np.array_equal(from_sliced(to_sliced(h, 0.5), N, G, 0.5), h)


def test_unpack_round_trip_all_12bit_values_both_parities(oracle):
    vals = np.arange(4096, dtype=np.uint32)
    G = 64
    # every value at an even group and at an odd group
    i1 = np.concatenate([vals.reshape(-1, G), np.roll(vals, 1).reshape(-1, G)])
    i2 = ((np.arange(i1.size, dtype=np.uint32) // 2) % 16).reshape(i1.shape)
    layer = {"spec": LayerSpec(i1.shape[0], G * 8, FMT_RVQ12_4, 64), **_pack12(i1, i2)}
    o1, o2 = oracle.unpack(layer)
    assert np.array_equal(o1, i1)
    assert np.array_equal(o2, i2)
    # every stage-2 value at both parities
    assert set(map(int, o2[:, 0::2].ravel())) == set(range(16))
    assert set(map(int, o2[:, 1::2].ravel())) == set(range(16))


def test_unpack_round_trip_all_16bit_values(oracle):
    vals = np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(-1, 256)
    layer = {"spec": LayerSpec(vals.shape[0], 256 * 8, FMT_VQ16, 2048), "idx16": to_sliced(vals, 1)}
    o1, o2 = oracle.unpack(layer)
    assert np.array_equal(o1, vals.astype(np.uint32))
    assert not o2.any()


# --------------------------------------------------------------------------- decode

def _tiny_layer_from_golden(g):
    cb1 = np.zeros((4096, 8), np.float16)
    for k, row in g["cb1_rows"].items():
        cb1[int(k)] = row
    cb2 = np.zeros((16, 8), np.float16)
    for k, row in g["cb2_rows"].items():
        cb2[int(k)] = row
    i1 = np.array([g["i1"]], np.uint32)
    i2 = np.array([g["i2"]], np.uint32)
    spec = LayerSpec(g["N"], g["K"], g["fmt"], g["scale_group"])
    # one row, one slice: the row's block scales in order
    return {"spec": spec, "cb1": cb1.view(np.uint16), "cb2": cb2.view(np.uint16),
            "scales": np.array(g["scales"], np.float16).view(np.uint16), **_pack12(i1, i2)}


def test_decode_golden_tiny_codebooks(oracle):
    g = _golden("decode_tiny.json")
    layer = _tiny_layer_from_golden(g)
    w, wb = oracle.dequant(layer, DT_F16)
    assert w[0].tolist() == g["w"]
    # every golden weight is exact in fp16, so the materialised weights are those values
    assert wb[0].view(np.float16).astype(np.float64).tolist() == g["w"]


def _one_group_layer(c1, c2, s, fmt=FMT_RVQ12_4):
    cb1 = np.zeros((4096, 8), np.float16)
    cb2 = np.zeros((16, 8), np.float16)
    cb1[5, 0] = c1
    cb2[7, 0] = c2
    i1 = np.array([[5, 5]], np.uint32)
    i2 = np.array([[7, 7]], np.uint32)
    return {"spec": LayerSpec(1, 16, fmt, 16), "cb1": cb1.view(np.uint16), "cb2": cb2.view(np.uint16),
            "scales": np.array([[s]], np.float16).view(np.uint16), **_pack12(i1, i2)}


@pytest.mark.parametrize("c1,c2,s,dt,expect", [
    (2048.0, 2.0 ** -14, 1.0, DT_F16, 0x6800),             # fl32(2048 + 2^-14) = 2048
    (1.0, 2.0 ** -11, 1.0, DT_F16, 0x3C00),                # 1 + 2^-11 ties to even in fp16
    (1.0, 3 * 2.0 ** -11, 1.0, DT_F16, 0x3C02),            # 1 + 3*2^-11 ties to even (up)
    (1.0, 2.0 ** -8, 1.0, DT_BF16, 0x3F80),                # 1 + 2^-8 ties to even in bf16
    (1.0, 3 * 2.0 ** -8, 1.0, DT_BF16, 0x3F82),
    (3.0, 0.0, -0.5, DT_F16, 0xBE00),                      # scale applied after the stage sum
    (1024.0, 1.0, 2.0 ** -10, DT_F16, 0x3C01),             # (1025) * 2^-10 = 1 + 2^-10
])
def test_decode_rounding_points_by_hand(oracle, c1, c2, s, dt, expect):
    w, wb = oracle.dequant(_one_group_layer(c1, c2, s), dt)
    assert int(wb[0, 0]) == expect
    assert w[0, 0] == s * (c1 + c2)


# --------------------------------------------------------------------------- forward

def _dense_numpy(layer):
    """Brute-force dense W, built here independently with numpy fancy indexing."""
    spec = layer["spec"]
    N, G = spec.N, spec.G
    cb1 = layer["cb1"].view(np.float16).astype(np.float64)
    if spec.fmt == FMT_VQ16:
        i1 = from_sliced(layer["idx16"], N, G, 1).astype(np.int64)
    else:
        h4 = from_sliced(layer["hi4"], N, G, 0.5)
        hi = np.empty((N, G), np.int64)
        hi[:, 0::2] = h4 & 15
        hi[:, 1::2] = h4 >> 4
        i1 = from_sliced(layer["lo"], N, G, 1).astype(np.int64) + 256 * hi
    W = cb1[i1]  # [N, G, 8]
    if spec.fmt == FMT_RVQ12_4:
        s2 = from_sliced(layer["s2"], N, G, 0.5)
        i2 = np.empty((N, G), np.int64)
        i2[:, 0::2] = s2 & 15
        i2[:, 1::2] = s2 >> 4
        W = W + layer["cb2"].view(np.float16).astype(np.float64)[i2]
    W = W.reshape(N, spec.K)
    sc = layer["scales"].view(np.float16).astype(np.float64)
    if spec.scale_group == spec.K:
        scm = sc.reshape(N, 1)
    else:  # K-slice-major with 8 / scale_group entries per group
        scm = from_sliced(sc, N, G, 8 / spec.scale_group)
    return W * np.repeat(scm, spec.scale_group, axis=1)


@pytest.mark.parametrize("fmt,sg,K", [(FMT_RVQ12, 8, 16), (FMT_RVQ12_4, 16, 16), (FMT_VQ16, 16, 16),
                                      (FMT_RVQ12_4, 8, 16), (FMT_RVQ12_4, 64, 384), (FMT_RVQ12, 192, 192),
                                      (FMT_VQ16, 64, 320), (FMT_RVQ12_4, 32, 192)])
@pytest.mark.parametrize("xdt", [DT_F16, DT_BF16])
def test_forward_brute_force_16x16(oracle, fmt, sg, K, xdt):
    # 16 rows; K=16 (one slice) and K=384 / 192 / 320 (several slices, some ragged)
    layer = make_layer(LayerSpec(16, K, fmt, sg), cfg_id=99, tensor_id=fmt * 10 + sg)
    x = make_x(5, K, xdt, cfg_id=99)
    W = _dense_numpy(layer)
    xd = x.view(np.float16).astype(np.float64) if xdt == DT_F16 else \
        (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ref = xd @ W.T
    y = oracle.forward(layer, x, xdt)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    w, _ = oracle.dequant(layer)
    assert np.array_equal(w, W)
    rows = [15, 0, 7]
    assert np.array_equal(oracle.forward(layer, x, xdt, rows=rows), y[:, rows])
    assert np.array_equal(oracle.dequant(layer, rows=rows)[0], W[rows])


def test_forward_one_hot_returns_columns(oracle):
    spec = LayerSpec(24, 64, FMT_RVQ12_4, 64)
    layer = make_layer(spec, cfg_id=98)
    w, _ = oracle.dequant(layer)
    ks = [0, 7, 8, 33, 63]
    x = np.zeros((len(ks), spec.K), np.float16)
    for r, k in enumerate(ks):
        x[r, k] = 1.0
    y = oracle.forward(layer, x.view(np.uint16), DT_F16)
    for r, k in enumerate(ks):
        assert np.array_equal(y[r], w[:, k])


def test_forward_linearity(oracle):
    spec = LayerSpec(32, 128, FMT_RVQ12_4, 64)
    layer = make_layer(spec, cfg_id=97)
    rng = np.random.default_rng(4)
    x1 = rng.integers(-8, 9, size=(3, spec.K)).astype(np.float16)
    x2 = rng.integers(-8, 9, size=(3, spec.K)).astype(np.float16)
    x3 = (2 * x1.astype(np.float64) - 3 * x2.astype(np.float64)).astype(np.float16)  # exact small integers
    y1, y2, y3 = (oracle.forward(layer, v.view(np.uint16), DT_F16) for v in (x1, x2, x3))
    assert np.allclose(y3, 2 * y1 - 3 * y2, rtol=1e-12, atol=1e-12 * np.abs(y3).max())


# --------------------------------------------------------------------------- rotation

@pytest.mark.parametrize("K", [1, 2, 4, 8, 64, 256])
def test_rht_matches_sylvester_hadamard(oracle, K):
    rng = np.random.default_rng(K)
    x = rng.standard_normal((3, K))
    signs = rng.choice([-1, 1], size=K).astype(np.int8)
    ref = (scipy.linalg.hadamard(K).astype(np.float64) @ (signs * x).T).T / np.sqrt(K)
    assert np.allclose(oracle.rht_f64(x, signs), ref, rtol=1e-13, atol=1e-13)


def test_rht_small_cases_by_hand(oracle):
    out = oracle.rht_f64(np.array([[3.0]]), np.array([-1], np.int8))
    assert out.tolist() == [[-3.0]]
    a, b = 5.0, 2.0
    out = oracle.rht_f64(np.array([[a, b]]), np.array([1, -1], np.int8))
    r = 1 / np.sqrt(2)
    assert np.allclose(out, [[(a - b) * r, (a + b) * r]], rtol=1e-15)


def test_rht_identities(oracle):
    K = 128
    rng = np.random.default_rng(5)
    x = rng.standard_normal((4, K))
    ones = np.ones(K, np.int8)
    assert np.allclose(oracle.rht_f64(oracle.rht_f64(x, ones), ones), x, atol=1e-13)  # H/sqrt(K) is an involution
    signs = rng.choice([-1, 1], size=K).astype(np.int8)
    y = oracle.rht_f64(x, signs)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)  # orthogonal
    assert np.allclose(y @ y.T, x @ x.T, atol=1e-12)
    e0 = np.zeros((1, K))
    e0[0, 0] = 1.0
    assert np.allclose(oracle.rht_f64(e0, ones), np.full((1, K), 1 / np.sqrt(K)), rtol=1e-15)


def test_rht_bits_entry_matches_f64(oracle):
    K = 64
    x = make_x(2, K, DT_BF16, cfg_id=96)
    signs = np.where(np.arange(K) % 3 == 0, -1, 1).astype(np.int8)
    xd = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.array_equal(oracle.rht(x, DT_BF16, signs), oracle.rht_f64(xd, signs))


# ------------------------------------------------------------------- encode (F4)

@pytest.mark.parametrize("fmt,N,K", [(FMT_RVQ12, 24, 448), (FMT_VQ16, 8, 256)])
def test_encode_round_trips_exact_codewords(oracle, fmt, N, K):
    """W made exactly of scaled codewords encodes back to its own indices (orka README, "How it
    works": encode = nearest entry; the true entry is at distance 0 and the codewords are
    distinct)."""
    layer = make_layer(LayerSpec(N, K, fmt, 64), cfg_id=120, tensor_id=fmt)
    assert np.unique(layer["cb1"], axis=0).shape[0] == layer["cb1"].shape[0]
    w, _ = oracle.dequant(layer)
    enc = oracle.encode(layer["spec"], w, layer["scales"], layer["cb1"])
    for k in ("lo", "hi4", "idx16"):
        if k in layer:
            assert np.array_equal(enc[k], layer[k]), k


def test_encode_two_stage_round_trip(oracle):
    """With a stage-2 codebook much smaller than the spacing of stage 1, W = s (c1 + c2) encodes
    back to both indices (stage 2 takes the residual stage 1 leaves)."""
    N, K = 16, 320
    layer = make_layer(LayerSpec(N, K, FMT_RVQ12_4, 64), cfg_id=121)
    small = (layer["cb2"].view(np.float16).astype(np.float32) * np.float32(1e-3)).astype(np.float16)
    layer["cb2"] = small.view(np.uint16)
    assert np.unique(layer["cb2"], axis=0).shape[0] == 16
    w, _ = oracle.dequant(layer)
    enc = oracle.encode(layer["spec"], w, layer["scales"], layer["cb1"], layer["cb2"])
    for k in ("lo", "hi4", "s2"):
        assert np.array_equal(enc[k], layer[k]), k


@pytest.mark.parametrize("fmt", [FMT_RVQ12, FMT_RVQ12_4])
def test_encode_matches_numpy_brute_force(oracle, fmt):
    """Arbitrary W (not made of codewords): numpy argmin over every entry, stage by stage, read
    back through the pinned unpack."""
    N, K = 5, 192
    rng = np.random.default_rng(122 + fmt)
    layer = make_layer(LayerSpec(N, K, fmt, 64), cfg_id=122, tensor_id=fmt)
    w = rng.standard_normal((N, K)) * 0.02
    enc = oracle.encode(layer["spec"], w, layer["scales"], layer["cb1"], layer.get("cb2"))
    i1, i2 = oracle.unpack(enc)
    f = lambda b: b.view(np.float16).astype(np.float64)  # noqa: E731
    c1 = f(layer["cb1"])
    G = K // 8
    for n in range(N):
        for g in range(G):
            sl, o = g // 16, g % 16
            wsl = min(16, G - 16 * sl)
            s = f(layer["scales"][2 * sl * N + n * (wsl // 8) + o // 8])
            v = w[n, 8 * g:8 * g + 8]
            a = int(np.argmin(((v[None, :] - s * c1) ** 2).sum(axis=1)))
            assert i1[n, g] == a, (n, g)
            if fmt == FMT_RVQ12_4:
                c2 = f(layer["cb2"])
                b = int(np.argmin(((v[None, :] - s * (c1[a][None, :] + c2)) ** 2).sum(axis=1)))
                assert i2[n, g] == b, (n, g)


@pytest.mark.parametrize("fmt", [FMT_RVQ12, FMT_RVQ12_4])
def test_encode32_matches_numpy_float32(oracle, fmt):
    """The binary32 decision (the GPU encoder's precision) against numpy float32 arithmetic in
    the same order: e_j = w_j - s * c_j, d = ((e_0^2 + e_1^2) + ...) + e_7^2, argmin first."""
    N, K = 4, 192
    rng = np.random.default_rng(130 + fmt)
    layer = make_layer(LayerSpec(N, K, fmt, 64), cfg_id=130, tensor_id=fmt)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    enc = oracle.encode(layer["spec"], w.astype(np.float64), layer["scales"], layer["cb1"], layer.get("cb2"),
                        precision="f32")
    i1, i2 = oracle.unpack(enc)
    c1 = layer["cb1"].view(np.float16).astype(np.float32)
    G = K // 8

    def nearest(v, s, c):
        d = np.zeros(c.shape[0], np.float32)
        for j in range(8):
            e = v[j] - s * c[:, j]
            d = d + e * e
        return int(np.argmin(d))

    for n in range(N):
        for g in range(G):
            sl, o = g // 16, g % 16
            s = layer["scales"][2 * sl * N + n * (min(16, G - 16 * sl) // 8) + o // 8].view(np.float16).astype(np.float32)
            v = w[n, 8 * g:8 * g + 8]
            a = nearest(v, s, c1)
            assert i1[n, g] == a, (n, g)
            if fmt == FMT_RVQ12_4:
                c2 = c1[a][None, :] + layer["cb2"].view(np.float16).astype(np.float32)
                assert i2[n, g] == nearest(v, s, c2), (n, g)


def test_dist32_is_bit_exact_binary32(oracle):
    """Every product, difference and sum rounded to binary32, in the stated order: the value
    equals numpy float32 arithmetic bit for bit (an fma, another order or fp64 accumulation
    changes some of these)."""
    rng = np.random.default_rng(132)
    for _ in range(3000):
        w = (rng.standard_normal(8) * 10.0 ** rng.uniform(-3, 1)).astype(np.float32)
        c = rng.standard_normal(8).astype(np.float16).astype(np.float32)
        s = np.float32(np.float16(rng.lognormal(-4, 1)))
        d = np.float32(0)
        for j in range(8):
            e = np.float32(w[j] - np.float32(s * c[j]))
            d = np.float32(d + np.float32(e * e))
        assert oracle.dist32(w.astype(np.float64), float(s), c.astype(np.float64)) == float(d)


def test_encode32_agrees_with_the_definition(oracle):
    """binary32 and fp64 decisions agree except where the two candidates' exact distances
    are within the binary32 error of each other; exact codewords round trip in both."""
    N, K = 32, 256
    layer = make_layer(LayerSpec(N, K, FMT_RVQ12, 64), cfg_id=131)
    w = (np.random.default_rng(131).standard_normal((N, K)) * 0.02).astype(np.float32).astype(np.float64)
    a64, _ = oracle.unpack(oracle.encode(layer["spec"], w, layer["scales"], layer["cb1"]))
    a32, _ = oracle.unpack(oracle.encode(layer["spec"], w, layer["scales"], layer["cb1"], precision="f32"))
    c1 = layer["cb1"].view(np.float16).astype(np.float64)
    G = K // 8
    differ = np.argwhere(a64 != a32)
    assert len(differ) <= 0.01 * N * G
    for n, g in differ:
        sl, o = g // 16, g % 16
        s = layer["scales"][2 * sl * N + n * 2 + o // 8].view(np.float16).astype(np.float64)
        v = w[n, 8 * g:8 * g + 8]
        d = lambda i: float(((v - s * c1[i]) ** 2).sum())  # noqa: E731
        assert d(a32[n, g]) - d(a64[n, g]) <= 1e-5 * d(a64[n, g]), (n, g)
    wx, _ = oracle.dequant(layer)
    rt = oracle.encode(layer["spec"], wx, layer["scales"], layer["cb1"], precision="f32")
    assert np.array_equal(rt["lo"], layer["lo"]) and np.array_equal(rt["hi4"], layer["hi4"])


def test_encode_ties_go_to_the_smaller_index(oracle):
    N, K = 1, 16
    cb1 = np.full((4096, 8), np.float16(30.0)).view(np.uint16).copy()
    target = np.array([0.5, -1, 2, 0.25, -0.5, 1, 1.5, -2], np.float16)
    cb1[9] = target.view(np.uint16)
    cb1[5] = target.view(np.uint16)
    sc = np.array([np.float16(0.5)], np.float16).view(np.uint16)
    w = np.tile(0.5 * target.astype(np.float64), 2)[None, :]
    enc = oracle.encode(LayerSpec(N, K, FMT_RVQ12, K), w, sc, cb1)
    i1, _ = oracle.unpack(enc)
    assert i1.tolist() == [[5, 5]]


# ------------------------------------------------------------ residual ladder (F3)

def _f16(a):
    return np.asarray(a, np.float32).astype(np.float16).view(np.uint16)


def _hand_ladder(N, K, bpw, sg, seed=0):
    """A small ladder layer drawn here (not by synth), for the by-hand pins."""
    rng = np.random.default_rng(seed)
    n16, n8 = {2: (1, 0), 3: (1, 1), 4: (2, 0), 5: (2, 1), 6: (3, 0), 7: (3, 1), 8: (4, 0)}[bpw]
    G = K // 8
    lay = {"spec": LayerSpec(N, K, FMT_VQ16_RVQ, sg, bpw=bpw),
           "cb1": _f16(rng.standard_normal((65536, 8))),
           "cbr": _f16(rng.standard_normal((max(n16 - 1, 1), 65536, 8))),
           "cb8": _f16(rng.standard_normal((256, 8))),
           "idx16": rng.integers(0, 65536, size=n16 * N * G).astype(np.uint16),
           "idx8": rng.integers(0, 256, size=N * G).astype(np.uint8) if n8 else None,
           "mult": rng.uniform(0.01, 0.5, size=n16 - 1 + n8).astype(np.float32),
           "scales": _f16(rng.uniform(0.5, 2.0, size=N * K // sg))}
    return lay, n16, n8


@pytest.mark.parametrize("bpw", [3, 4, 5, 6, 7, 8])
def test_ladder_by_hand_one_slice(oracle, bpw):
    """GLQ README, "Bit widths": W = s * (cb1[i1] + sum of mult_t * codebook_t[i_t]).  K = 128 is
    one slice, so group g of row n is entry 16 n + g of every plane, and the two 64-wide
    block scales of row n are scales[2 n], scales[2 n + 1]."""
    N, K = 3, 128
    lay, n16, n8 = _hand_ladder(N, K, bpw, 64, seed=bpw)
    f = lambda b: b.view(np.float16).astype(np.float64)  # noqa: E731
    NG = N * 16
    W = np.zeros((N, K))
    for n in range(N):
        for g in range(16):
            e = 16 * n + g
            c = f(lay["cb1"][lay["idx16"][e]])
            for t in range(1, n16):
                c = c + float(lay["mult"][t - 1]) * f(lay["cbr"][t - 1][lay["idx16"][t * NG + e]])
            if n8:
                c = c + float(lay["mult"][n16 - 1]) * f(lay["cb8"][lay["idx8"][e]])
            W[n, 8 * g:8 * g + 8] = f(lay["scales"][2 * n + g // 8]) * c
    w, _ = oracle.dequant(lay)
    assert np.allclose(w, W, rtol=1e-14, atol=1e-15)
    x = make_x(2, K, DT_F16, cfg_id=97)
    xd = x.view(np.float16).astype(np.float64)
    assert np.allclose(oracle.forward(lay, x, DT_F16), xd @ W.T, rtol=1e-12, atol=1e-12)


def test_ladder_two_bits_is_the_16bit_format(oracle):
    """bpw = 2 is the primary stage alone: the same weights as the single-stage 16-bit
    format on the same plane, codebook and scales, bit for bit."""
    lay, _, _ = _hand_ladder(40, 384, 2, 64, seed=5)
    plain = {"spec": LayerSpec(40, 384, FMT_VQ16, 64), "cb1": lay["cb1"], "idx16": lay["idx16"],
             "scales": lay["scales"]}
    for wdt in (DT_F16, DT_BF16):
        w1, b1 = oracle.dequant(lay, wdt)
        w2, b2 = oracle.dequant(plain, wdt)
        assert np.array_equal(w1, w2) and np.array_equal(b1, b2)


@pytest.mark.parametrize("bpw", [3, 5, 8])
def test_ladder_is_a_sum_of_single_stage_layers(oracle, bpw):
    """Linearity in the stages: the ladder equals the sum, over its stages, of multiplier x the
    single-stage 16-bit decode of that stage's plane and codebook (the 8-bit stage as a
    16-bit layer whose codebook starts with the 256 entries), several slices, ragged tail."""
    N, K = 24, 448  # 3 full slices + a 64-wide tail
    lay, n16, n8 = _hand_ladder(N, K, bpw, 64, seed=10 + bpw)
    NG = N * K // 8
    def single(plane, cb):
        return oracle.dequant({"spec": LayerSpec(N, K, FMT_VQ16, 64), "cb1": cb, "idx16": plane,
                               "scales": lay["scales"]})[0]
    ref = single(lay["idx16"][:NG], lay["cb1"])
    for t in range(1, n16):
        ref += float(lay["mult"][t - 1]) * single(lay["idx16"][t * NG:(t + 1) * NG], lay["cbr"][t - 1])
    if n8:
        cb = np.zeros((65536, 8), np.uint16)
        cb[:256] = lay["cb8"]
        ref += float(lay["mult"][n16 - 1]) * single(lay["idx8"].astype(np.uint16), cb)
    w, _ = oracle.dequant(lay)
    assert np.allclose(w, ref, rtol=1e-13, atol=1e-13 * np.abs(ref).max())


@pytest.mark.parametrize("wdt", [DT_F16, DT_BF16])
def test_ladder_materialised_bits(oracle, wdt):
    """Materialised weights: v = c1, v = fl32(mult * c + v) per stage, RN(fl32(s * v)), checked
    against numpy float32 arithmetic (the product mult * c is exact in float64)."""
    N, K = 16, 256
    lay, n16, n8 = _hand_ladder(N, K, 7, 64, seed=21)
    _, wb = oracle.dequant(lay, wdt)
    f = lambda b: b.view(np.float16).astype(np.float64)  # noqa: E731
    NG = N * K // 8
    G = K // 8
    v = np.zeros((N, K), np.float32)
    s = np.zeros((N, K), np.float32)
    for n in range(N):
        for g in range(G):
            sl, o = g // 16, g % 16
            e = 16 * sl * N + n * 16 + o
            vv = f(lay["cb1"][lay["idx16"][e]]).astype(np.float32)
            for t in range(1, n16):
                vv = (float(lay["mult"][t - 1]) * f(lay["cbr"][t - 1][lay["idx16"][t * NG + e]])
                      + vv.astype(np.float64)).astype(np.float32)
            vv = (float(lay["mult"][n16 - 1]) * f(lay["cb8"][lay["idx8"][e]]) + vv.astype(np.float64)).astype(np.float32)
            v[n, 8 * g:8 * g + 8] = vv
            s[n, 8 * g:8 * g + 8] = f(lay["scales"][2 * sl * N + 2 * n + o // 8])  # two 64-wide blocks per slice
    p = (s.astype(np.float64) * v.astype(np.float64)).astype(np.float32)
    ref = _f16(p) if wdt == DT_F16 else f32_to_bf16_bits(p)
    assert np.array_equal(wb, ref), f"{np.sum(wb != ref)} weights differ"


def test_ladder_stage_sum_rounds_once(oracle):
    """A tie the fp64 sum alone would get wrong: v = 1 + 2^-11 after stage 2, then
    mult * c = 2^-24 + 2^-57 (mult = 14245331 * 2^-48, c = 1206 / 1024; 14245331 * 1206 =
    2^34 + 2).  The exact stage sum is just above the binary32 midpoint 1 + 2^-11 + 2^-24, so
    one rounding gives 1 + 2^-11 + 2^-23, which is above the fp16 midpoint 1 + 2^-11: the
    weight is fp16 1 + 2^-10 (0x3C01).  Rounding the fp64 sum instead lands on the midpoint,
    ties to 1 + 2^-11 and then to fp16 1.0 (0x3C00)."""
    assert 14245331 * 1206 == 2 ** 34 + 2
    lay = {"spec": LayerSpec(1, 16, FMT_VQ16_RVQ, 16, bpw=6),
           "cb1": np.zeros((65536, 8), np.uint16), "cbr": np.zeros((2, 65536, 8), np.uint16),
           "cb8": np.zeros((256, 8), np.uint16), "idx16": np.zeros(6, np.uint16), "idx8": None,
           "mult": np.array([2.0 ** -11, 14245331 * 2.0 ** -48], np.float32),
           "scales": _f16([1.0])}
    assert float(lay["mult"][1]) == 14245331 * 2.0 ** -48  # exact in binary32
    lay["cb1"][0] = _f16([1.0] * 8)
    lay["cbr"][0][0] = _f16([1.0] * 8)
    lay["cbr"][1][0] = _f16([1206 / 1024] * 8)
    w, wb = oracle.dequant(lay, DT_F16)
    assert np.all(wb[0, :8] == 0x3C01), wb[0, :8]
    assert np.allclose(w[0, :8], 1 + 2.0 ** -11 + 2.0 ** -24 + 2.0 ** -57, rtol=0, atol=1e-16)


# ------------------------------------------------- block-diagonal rotation (K not 2^p)

def _block_diag_hadamard(K):
    """GLQ README, "Bit widths": 2688 is cut as 2048 + 512 + 128.  The dense orthonormal
    matrix built from scipy's Sylvester blocks in that order (binary expansion of K,
    largest block first)."""
    sizes = [1 << b for b in range(30, -1, -1) if K & (1 << b)]
    return scipy.linalg.block_diag(*[scipy.linalg.hadamard(b).astype(np.float64) / np.sqrt(b) for b in sizes]), sizes


def test_block_sizes_of_the_pages_example():
    assert _block_diag_hadamard(2688)[1] == [2048, 512, 128]


@pytest.mark.parametrize("K", [3, 192, 320, 2688])
def test_rht_block_diagonal_matches_dense_blocks(oracle, K):
    rng = np.random.default_rng(200 + K)
    x = rng.standard_normal((2, K))
    signs = rng.choice([-1, 1], size=K).astype(np.int8)
    H, _ = _block_diag_hadamard(K)
    assert np.allclose(oracle.rht_f64(x, signs), (H @ (signs * x).T).T, rtol=1e-12, atol=1e-12)
    assert np.allclose(oracle.rht_out_f64(x, signs), signs * (H @ x.T).T, rtol=1e-12, atol=1e-12)


def test_rht_block_diagonal_by_hand(oracle):
    """K = 3 = 2 + 1: a 2-point butterfly on the first two entries, the last one only
    sign-flipped."""
    a, b, c = 5.0, 2.0, 7.0
    out = oracle.rht_f64(np.array([[a, b, c]]), np.array([1, -1, -1], np.int8))
    r = 1 / np.sqrt(2)
    assert np.allclose(out, [[(a - b) * r, (a + b) * r, -c]], rtol=1e-15)


def test_rht_block_diagonal_invariants(oracle):
    """Blocks do not mix (a one-hot input in block j stays in block j), norms are kept,
    and the output rotation undoes the input one."""
    K = 2688
    rng = np.random.default_rng(9)
    x = rng.standard_normal((2, K))
    signs = rng.choice([-1, 1], size=K).astype(np.int8)
    y = oracle.rht_f64(x, signs)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)
    assert np.allclose(oracle.rht_out_f64(y, signs), x, atol=1e-12)
    ones = np.ones(K, np.int8)
    for off, b in ((0, 2048), (2048, 512), (2560, 128)):
        e = np.zeros((1, K))
        e[0, off + 5] = 1.0
        out = oracle.rht_f64(e, ones)[0]
        assert np.allclose(np.abs(out[off:off + b]), 1 / np.sqrt(b), rtol=1e-14)
        assert np.count_nonzero(out) == b


# ----------------------------------------------------------------- output rotation

@pytest.mark.parametrize("N", [1, 2, 8, 128])
def test_rht_out_matches_sylvester_hadamard(oracle, N):
    """signs * (1/sqrt N) H y: the library's Sylvester matrix, signs applied after it."""
    rng = np.random.default_rng(100 + N)
    y = rng.standard_normal((3, N))
    signs = rng.choice([-1, 1], size=N).astype(np.int8)
    ref = signs * (scipy.linalg.hadamard(N).astype(np.float64) @ y.T).T / np.sqrt(N)
    assert np.allclose(oracle.rht_out_f64(y, signs), ref, rtol=1e-13, atol=1e-13)


def test_rht_out_small_case_by_hand(oracle):
    a, b = 5.0, 2.0
    out = oracle.rht_out_f64(np.array([[a, b]]), np.array([1, -1], np.int8))
    r = 1 / np.sqrt(2)
    # H y = (a + b, a - b), then the signs (+1, -1): differs from the input rotation's (a - b, a + b)
    assert np.allclose(out, [[(a + b) * r, -(a - b) * r]], rtol=1e-15)


def test_rht_out_undoes_the_input_rotation(oracle):
    """R^T R = I: rotating an input, then applying the output rotation with the same signs,
    returns it (the two differ in where the signs go)."""
    K = 256
    rng = np.random.default_rng(7)
    x = rng.standard_normal((3, K))
    signs = rng.choice([-1, 1], size=K).astype(np.int8)
    assert np.allclose(oracle.rht_out_f64(oracle.rht_f64(x, signs), signs), x, atol=1e-12)
    assert not np.allclose(oracle.rht_f64(oracle.rht_f64(x, signs), signs), x, atol=1e-3)


def test_two_sided_rotation_end_to_end(oracle):
    """A layer stored as W_hat = R_out W R_in^T gives back y = W x through
    y = R_out^T (W_hat (R_in x)), with R = (1/sqrt n) H diag(signs) built explicitly."""
    N, K = 16, 32
    rng = np.random.default_rng(11)
    W = rng.standard_normal((N, K))
    x = rng.standard_normal((2, K))
    s_in = rng.choice([-1, 1], size=K).astype(np.int8)
    s_out = rng.choice([-1, 1], size=N).astype(np.int8)
    R_in = scipy.linalg.hadamard(K) * s_in[None, :] / np.sqrt(K)
    R_out = scipy.linalg.hadamard(N) * s_out[None, :] / np.sqrt(N)
    W_hat = R_out @ W @ R_in.T
    y = oracle.rht_out_f64(oracle.rht_f64(x, s_in) @ W_hat.T, s_out)
    assert np.allclose(y, x @ W.T, atol=1e-12)


# --------------------------------------------------------------------------- sparse correction
# orka README, "How it works": decode = scale x sum(codebook[index]) (+ sparse correction).
# Reading: W' = W + C with C sparse, by output row (CSR); materialised weights take one more
# fp32 rounding, RN(fl32(fl32(s * fl32(c1 + c2)) + C)).

def _csr(N, entries):
    """(row, col, value) triples -> the CSR arrays, rows in order."""
    entries = sorted(entries)
    row_ptr = np.zeros(N + 1, np.int32)
    for n, _, _ in entries:
        row_ptr[n + 1:] += 1
    col = np.array([c for _, c, _ in entries], np.int32)
    val = np.array([v for _, _, v in entries], np.float16).view(np.uint16)
    return {"row_ptr": row_ptr, "col": col, "val": val}


def _dense_corr(corr, N, K):
    C = np.zeros((N, K))
    for n in range(N):
        for j in range(corr["row_ptr"][n], corr["row_ptr"][n + 1]):
            C[n, corr["col"][j]] += float(corr["val"][j:j + 1].view(np.float16)[0])
    return C


def test_correction_by_hand(oracle):
    """Two rows of 16 weights, every codeword 1.0 except entry 0 (dims 0..7 = 0..7), scale 0.5;
    corrections (0, 3, +0.25), (1, 0, -2.0), (1, 15, +0.5)."""
    cb1 = np.ones((4096, 8), np.float16)
    cb1[0] = np.arange(8)
    i1 = np.array([[0, 1], [1, 0]], np.uint32)  # row 0: groups (entry 0, entry 1); row 1: (entry 1, entry 0)
    layer = {"spec": LayerSpec(2, 16, FMT_RVQ12, 16), "cb1": cb1.view(np.uint16),
             "scales": np.array([0.5, 0.5], np.float16).view(np.uint16), **_pack12(i1, np.zeros_like(i1))}
    layer["corr"] = _csr(2, [(0, 3, 0.25), (1, 0, -2.0), (1, 15, 0.5)])
    want = np.array([[0, .5, 1, 1.5 + .25, 2, 2.5, 3, 3.5] + [.5] * 8,
                     [.5 - 2.0] + [.5] * 7 + [0, .5, 1, 1.5, 2, 2.5, 3, 3.5 + .5]])
    w, wb = oracle.dequant(layer, DT_F16)
    assert w.tolist() == want.tolist()
    assert wb.view(np.float16).astype(np.float64).tolist() == want.tolist()  # all exact in fp16
    x = np.ones((1, 16), np.float16).view(np.uint16)
    assert oracle.forward(layer, x, DT_F16).tolist() == [want.sum(axis=1).tolist()]


@pytest.mark.parametrize("p,v,dt,expect", [
    (1.0, 2.0 ** -11, DT_F16, 0x3C00),       # 1 + 2^-11 is exact in fp32, then ties to even in fp16
    (1.0, 3 * 2.0 ** -11, DT_F16, 0x3C02),   # ... and rounds up to 1 + 2^-9
    (2048.0, 2.0 ** -14, DT_F16, 0x6800),    # fl32(2048 + 2^-14) = 2048 (below half an fp32 ulp)
    (1.0, 2.0 ** -8, DT_BF16, 0x3F80),       # bf16 tie to even
    (-3.0, 0.5, DT_BF16, 0xC020),            # -2.5 exactly
])
def test_correction_rounding_points_by_hand(oracle, p, v, dt, expect):
    layer = _one_group_layer(p, 0.0, 1.0, fmt=FMT_RVQ12)
    layer.pop("cb2")
    layer["corr"] = _csr(1, [(0, 0, v)])
    w, wb = oracle.dequant(layer, dt)
    assert int(wb[0, 0]) == expect
    assert w[0, 0] == p + v
    assert int(wb[0, 1]) == int(oracle.dequant(_one_group_layer(p, 0.0, 1.0, fmt=FMT_RVQ12), dt)[1][0, 1])


@pytest.mark.parametrize("fmt,sg,K", [(FMT_RVQ12, 64, 384), (FMT_RVQ12_4, 64, 320), (FMT_VQ16, 192, 192)])
def test_correction_matches_dense_numpy(oracle, fmt, sg, K):
    """W' = W + C built independently (numpy dense W, dense C from the triples) against the
    oracle's dequant and forward, on all rows and on a row subset."""
    N = 24
    layer = make_layer(LayerSpec(N, K, fmt, sg), cfg_id=96, tensor_id=fmt)
    layer["corr"] = make_correction(N, K, density=0.05, cfg_id=96, tensor_id=fmt)
    assert layer["corr"]["row_ptr"][-1] > 0
    Wc = _dense_numpy(layer) + _dense_corr(layer["corr"], N, K)
    w, _ = oracle.dequant(layer)
    assert np.array_equal(w, Wc)
    x = make_x(3, K, DT_BF16, cfg_id=96)
    xd = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ref = xd @ Wc.T
    y = oracle.forward(layer, x, DT_BF16)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    rows = [20, 3, 11]
    assert np.array_equal(oracle.forward(layer, x, DT_BF16, rows=rows), y[:, rows])


def test_correction_of_zeros_is_the_identity(oracle):
    N, K = 16, 256
    layer = make_layer(LayerSpec(N, K, FMT_RVQ12_4, 64), cfg_id=95)
    x = make_x(2, K, DT_F16, cfg_id=95)
    base_y, (base_w, base_wb) = oracle.forward(layer, x, DT_F16), oracle.dequant(layer, DT_F16)
    corr = make_correction(N, K, density=0.1, cfg_id=95)
    corr["val"] = np.zeros_like(corr["val"])
    layer["corr"] = corr
    assert np.array_equal(oracle.forward(layer, x, DT_F16), base_y)
    w, wb = oracle.dequant(layer, DT_F16)
    assert np.array_equal(w, base_w) and np.array_equal(wb, base_wb)


def test_correction_layout_is_checked(oracle):
    ok = _csr(3, [(0, 1, 1.0), (0, 5, 1.0), (2, 0, 1.0)])
    assert oracle.corr_check(3, 8, ok["row_ptr"], ok["col"]) == 0
    assert oracle.corr_check(3, 8, ok["row_ptr"], np.array([5, 1, 0], np.int32)) != 0   # columns not increasing
    assert oracle.corr_check(3, 8, ok["row_ptr"], np.array([1, 5, 8], np.int32)) != 0   # column beyond K
    assert oracle.corr_check(3, 8, np.array([0, 2, 1, 3], np.int32), ok["col"]) != 0    # row_ptr decreasing
    assert oracle.corr_check(3, 8, np.array([1, 2, 2, 3], np.int32), ok["col"]) != 0    # row_ptr[0] != 0

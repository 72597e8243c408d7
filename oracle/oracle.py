"""ctypes front end for the plain-C oracle (oracle/vq_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, by __graft_entry__.smoke() and by
bench.py's cpu_baseline / reference arm.  The product library never imports it.

All arrays are numpy arrays; fp16/bf16 data are uint16 bit patterns.  Results are
fp64 numpy arrays (or uint16 bits for rounded weights).
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "vq_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

FMT_RVQ12, FMT_RVQ12_4, FMT_VQ16, FMT_VQ16_RVQ = 1, 2, 3, 4

# GLQ README, "Bit widths" table: bits per weight -> (16-bit stages including the
# primary, 8-bit residual stages).
LADDER_STAGES = {2: (1, 0), 3: (1, 1), 4: (2, 0), 5: (2, 1), 6: (3, 0), 7: (3, 1), 8: (4, 0)}
DT_F16, DT_BF16 = 0, 1

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile vq_oracle.c into liboracle.so with gcc (strict IEEE: no contraction, no fast-math)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                               "-shared", "-fPIC", "-o", tmp, SRC, "-lm"])
        os.replace(tmp, LIB)
    return LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(LIB)
            P = ctypes.c_void_p
            I = ctypes.c_int
            lib.vqo_f16_to_f64.restype = ctypes.c_double
            lib.vqo_f16_to_f64.argtypes = [ctypes.c_uint16]
            lib.vqo_bf16_to_f64.restype = ctypes.c_double
            lib.vqo_bf16_to_f64.argtypes = [ctypes.c_uint16]
            lib.vqo_f64_to_f16.restype = ctypes.c_uint16
            lib.vqo_f64_to_f16.argtypes = [ctypes.c_double]
            lib.vqo_f64_to_bf16.restype = ctypes.c_uint16
            lib.vqo_f64_to_bf16.argtypes = [ctypes.c_double]
            lib.vqo_fl32.restype = ctypes.c_double
            lib.vqo_fl32.argtypes = [ctypes.c_double]
            lib.vqo_decode_array.restype = None
            lib.vqo_decode_array.argtypes = [P, ctypes.c_int64, I, P]
            lib.vqo_rht_f64.restype = I
            lib.vqo_rht_f64.argtypes = [I, I, P, P, P]
            lib.vqo_rht_out_f64.restype = I
            lib.vqo_rht_out_f64.argtypes = [I, I, P, P, P]
            lib.vqo_round_array.restype = None
            lib.vqo_round_array.argtypes = [P, ctypes.c_int64, I, P]
            lib.vqo_unpack.restype = I
            lib.vqo_unpack.argtypes = [I, I, I, P, P, P, P, P, P]
            lib.vqo_dequant.restype = I
            lib.vqo_dequant.argtypes = [I, I, I, P, P, P, P, P, P, P, I, P, I, P, P, I]
            lib.vqo_forward.restype = I
            lib.vqo_forward.argtypes = [I, I, I, I, P, I, P, P, P, P, P, P, P, I, P, I, P]
            lib.vqo_rht.restype = I
            lib.vqo_rht.argtypes = [I, I, P, I, P, P]
            lib.vqo_corr_check.restype = I
            lib.vqo_corr_check.argtypes = [I, I, P, P]
            lib.vqo_dequant_corr.restype = I
            lib.vqo_dequant_corr.argtypes = [I, I, I, P, P, P, P, P, P, P, I, P, P, P, P, I, P, P, I]
            lib.vqo_forward_corr.restype = I
            lib.vqo_forward_corr.argtypes = [I, I, I, I, P, I, P, P, P, P, P, P, P, I, P, P, P, P, I, P]
            lib.vqo_encode.restype = I
            lib.vqo_encode.argtypes = [I, I, I, P, P, I, P, P, P, P, P, P]
            lib.vqo_dist32.restype = ctypes.c_double
            lib.vqo_dist32.argtypes = [P, ctypes.c_double, P]
            lib.vqo_encode32.restype = I
            lib.vqo_encode32.argtypes = [I, I, I, P, P, I, P, P, P, P, P, P]
            lib.vqo_ladder_dequant.restype = I
            lib.vqo_ladder_dequant.argtypes = [I, I, I, I, P, P, P, P, P, P, P, I, P, I, P, P, I]
            lib.vqo_ladder_forward.restype = I
            lib.vqo_ladder_forward.argtypes = [I, I, I, I, I, P, I, P, P, P, P, P, P, P, I, P, I, P]
            _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def decode(bits, dt: int) -> np.ndarray:
    """fp16 (dt=0) or bf16 (dt=1) bit patterns -> fp64 values."""
    lib = _load()
    b = _c(bits, np.uint16)
    out = np.empty(b.shape, dtype=np.float64)
    lib.vqo_decode_array(_p(b), b.size, dt, _p(out))
    return out


def f16_to_f64(bits) -> np.ndarray:
    return decode(bits, DT_F16)


def bf16_to_f64(bits) -> np.ndarray:
    return decode(bits, DT_BF16)


def round_to(values, dt: int) -> np.ndarray:
    """Round fp64 values to fp16 (dt=0) or bf16 (dt=1) bits, ties to even."""
    lib = _load()
    v = _c(values, np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    lib.vqo_round_array(_p(v), v.size, dt, _p(out))
    return out


def fl32(v: float) -> float:
    return _load().vqo_fl32(float(v))


def _planes(layer):
    return (_c(layer.get("lo"), np.uint8), _c(layer.get("hi4"), np.uint8), _c(layer.get("s2"), np.uint8),
            _c(layer.get("idx16"), np.uint16))


def unpack(layer) -> tuple[np.ndarray, np.ndarray]:
    """Return (i1 uint32 [N,G], i2 uint8 [N,G]) for a layer dict from ``synth.make_layer``."""
    lib = _load()
    spec = layer["spec"]
    lo, hi4, s2, idx16 = _planes(layer)
    fmt = spec.fmt
    if fmt == FMT_VQ16_RVQ:  # the primary stage's plane
        fmt, idx16 = FMT_VQ16, np.ascontiguousarray(idx16[: spec.N * spec.G])
    i1 = np.empty((spec.N, spec.G), dtype=np.uint32)
    i2 = np.empty((spec.N, spec.G), dtype=np.uint8)
    rc = lib.vqo_unpack(fmt, spec.N, spec.K, _p(lo), _p(hi4), _p(s2), _p(idx16), _p(i1), _p(i2))
    if rc:
        raise ValueError(f"vqo_unpack failed rc={rc}")
    return i1, i2


def _rows(rows):
    if rows is None:
        return None, 0
    r = np.ascontiguousarray(rows, dtype=np.int32)
    return r, int(r.size)


def _ladder(layer):
    """The residual ladder's arrays (GLQ README, "Bit widths") in the oracle's calling form."""
    spec = layer["spec"]
    n16, _ = LADDER_STAGES[spec.bpw]
    cbr = layer["cbr"] if n16 > 1 else np.zeros((1, 65536, 8), np.uint16)
    return (_c(layer["idx16"], np.uint16), _c(layer.get("idx8"), np.uint8), _c(layer["cb1"], np.uint16),
            _c(cbr, np.uint16), _c(layer["cb8"], np.uint16), _c(layer["mult"], np.float32).astype(np.float64),
            _c(layer["scales"], np.uint16))


def dequant(layer, wdt: int = DT_F16, rows=None) -> tuple[np.ndarray, np.ndarray]:
    """Return (W exact fp64 [n,K], W materialised fp16/bf16 bits [n,K]) for `rows` (default: all)."""
    lib = _load()
    spec = layer["spec"]
    if spec.fmt == FMT_VQ16_RVQ:
        idx16, idx8, cb1, cbr, cb8, mult, sc = _ladder(layer)
        r, nr = _rows(rows)
        n = spec.N if r is None else nr
        w = np.empty((n, spec.K), dtype=np.float64)
        wb = np.empty((n, spec.K), dtype=np.uint16)
        n16, n8 = LADDER_STAGES[spec.bpw]
        rc = lib.vqo_ladder_dequant(spec.N, spec.K, n16, n8, _p(idx16), _p(idx8), _p(cb1), _p(cbr),
                                    _p(cb8), _p(mult), _p(sc), spec.scale_group, _p(r), nr, _p(w), _p(wb), wdt)
        if rc:
            raise ValueError(f"vqo_ladder_dequant failed rc={rc}")
        return w, wb
    lo, hi4, s2, idx16 = _planes(layer)
    cb1, cb2, sc = _c(layer["cb1"], np.uint16), _c(layer.get("cb2"), np.uint16), _c(layer["scales"], np.uint16)
    r, nr = _rows(rows)
    n = spec.N if r is None else nr
    w = np.empty((n, spec.K), dtype=np.float64)
    wb = np.empty((n, spec.K), dtype=np.uint16)
    if "corr" in layer:  # the sparse correction (orka README, "How it works")
        rp, cl, vl = _corr(layer)
        rc = lib.vqo_dequant_corr(spec.fmt, spec.N, spec.K, _p(lo), _p(hi4), _p(s2), _p(idx16), _p(cb1), _p(cb2),
                                  _p(sc), spec.scale_group, _p(rp), _p(cl), _p(vl), _p(r), nr, _p(w), _p(wb), wdt)
    else:
        rc = lib.vqo_dequant(spec.fmt, spec.N, spec.K, _p(lo), _p(hi4), _p(s2), _p(idx16), _p(cb1), _p(cb2),
                             _p(sc), spec.scale_group, _p(r), nr, _p(w), _p(wb), wdt)
    if rc:
        raise ValueError(f"vqo_dequant failed rc={rc}")
    return w, wb


def _corr(layer):
    """The sparse correction of a layer dict in the oracle's calling form (CSR by output row)."""
    c = layer["corr"]
    if layer["spec"].fmt == FMT_VQ16_RVQ:
        raise ValueError("the sparse correction is defined for the 12-bit and 16-bit formats only")
    return _c(c["row_ptr"], np.int32), _c(c["col"], np.int32), _c(c["val"], np.uint16)


def corr_check(N: int, K: int, row_ptr, col) -> int:
    """0 if (row_ptr, col) is a valid correction layout for an N x K layer, else nonzero."""
    return _load().vqo_corr_check(N, K, _p(_c(row_ptr, np.int32)), _p(_c(col, np.int32)))


def dist32(w8, s, c8) -> float:
    """The binary32 distance the GPU encoder decides with (binary32 inputs)."""
    w8, c8 = _c(w8, np.float64), _c(c8, np.float64)
    return _load().vqo_dist32(_p(w8), float(s), _p(c8))


def encode(spec, w, scales, cb1, cb2=None, precision: str = "f64") -> dict:
    """Nearest-entry encode of a dense W [N,K] (orka README, "How it works") into the
    planes of `spec.fmt`, with the given scales (fp16 bits, storage order) and codebooks.
    precision "f64": the definition, distances in fp64; "f32": the same decisions taken
    with binary32 distances in a fixed operation order (W must hold binary32 values), the
    precision of the GPU encoder.  Returns a layer dict like ``synth.make_layer``'s."""
    lib = _load()
    fn = {"f64": lib.vqo_encode, "f32": lib.vqo_encode32}[precision]
    N, K, G = spec.N, spec.K, spec.K // 8
    wd = _c(w, np.float64)
    if wd.shape != (N, K):
        raise ValueError("w has the wrong shape")
    sc, c1, c2 = _c(scales, np.uint16), _c(cb1, np.uint16), _c(cb2, np.uint16)
    out = {"spec": spec, "cb1": c1, "scales": sc}
    lo = hi4 = s2 = idx16 = None
    if spec.fmt == FMT_VQ16:
        idx16 = np.zeros(N * G, np.uint16)
        out["idx16"] = idx16
    else:
        lo, hi4 = np.zeros(N * G, np.uint8), np.zeros(N * G // 2, np.uint8)
        out["lo"], out["hi4"] = lo, hi4
        if spec.fmt == FMT_RVQ12_4:
            s2 = np.zeros(N * G // 2, np.uint8)
            out["s2"], out["cb2"] = s2, c2
    rc = fn(spec.fmt, N, K, _p(wd), _p(sc), spec.scale_group, _p(c1), _p(c2), _p(lo), _p(hi4), _p(s2), _p(idx16))
    if rc:
        raise ValueError(f"vqo_encode failed rc={rc}")
    return out


def forward(layer, x_bits, xdt: int, rows=None) -> np.ndarray:
    """y[m][t] = sum_k x[m][k] W[rows[t]][k] in fp64 (x as fp16/bf16 bits [M,K]; rows default: all)."""
    lib = _load()
    spec = layer["spec"]
    x = _c(x_bits, np.uint16)
    M = x.shape[0]
    if x.shape[1] != spec.K:
        raise ValueError("x has the wrong K")
    r, nr = _rows(rows)
    n = spec.N if r is None else nr
    y = np.empty((M, n), dtype=np.float64)
    if spec.fmt == FMT_VQ16_RVQ:
        idx16, idx8, cb1, cbr, cb8, mult, sc = _ladder(layer)
        n16, n8 = LADDER_STAGES[spec.bpw]
        rc = lib.vqo_ladder_forward(M, spec.N, spec.K, n16, n8, _p(x), xdt, _p(idx16), _p(idx8),
                                    _p(cb1), _p(cbr), _p(cb8), _p(mult), _p(sc), spec.scale_group, _p(r), nr,
                                    _p(y))
        if rc:
            raise ValueError(f"vqo_ladder_forward failed rc={rc}")
        return y
    lo, hi4, s2, idx16 = _planes(layer)
    cb1, cb2, sc = _c(layer["cb1"], np.uint16), _c(layer.get("cb2"), np.uint16), _c(layer["scales"], np.uint16)
    if "corr" in layer:  # y = x (W + C)^T with the sparse correction C
        rp, cl, vl = _corr(layer)
        rc = lib.vqo_forward_corr(spec.fmt, M, spec.N, spec.K, _p(x), xdt, _p(lo), _p(hi4), _p(s2), _p(idx16),
                                  _p(cb1), _p(cb2), _p(sc), spec.scale_group, _p(rp), _p(cl), _p(vl), _p(r), nr,
                                  _p(y))
    else:
        rc = lib.vqo_forward(spec.fmt, M, spec.N, spec.K, _p(x), xdt, _p(lo), _p(hi4), _p(s2), _p(idx16),
                             _p(cb1), _p(cb2), _p(sc), spec.scale_group, _p(r), nr, _p(y))
    if rc:
        raise ValueError(f"vqo_forward failed rc={rc}")
    return y


def rht(x_bits, xdt: int, signs) -> np.ndarray:
    """Rotated activations (1/sqrt K) H (signs * x) in fp64, x given as bits [M,K]
    (block-diagonal over the binary expansion of K when K is not a power of two)."""
    lib = _load()
    x = _c(x_bits, np.uint16)
    sg = _c(signs, np.int8)
    M, K = x.shape
    out = np.empty((M, K), dtype=np.float64)
    rc = lib.vqo_rht(M, K, _p(x), xdt, _p(sg), _p(out))
    if rc:
        raise ValueError(f"vqo_rht failed rc={rc}")
    return out


def rht_f64(x, signs) -> np.ndarray:
    """Rotation of fp64 activations [M,K]: (1/sqrt K) H (signs * x).

    GLQ README, "Bit widths": a K that is not a power of two is cut into the powers of
    two of its binary expansion, largest first along K (2688 = 2048 + 512 + 128), and
    each block b is rotated by its own (1/sqrt b) H_b."""
    lib = _load()
    xd = _c(x, np.float64)
    sg = _c(signs, np.int8)
    M, K = xd.shape
    out = np.empty((M, K), dtype=np.float64)
    rc = lib.vqo_rht_f64(M, K, _p(xd), _p(sg), _p(out))
    if rc:
        raise ValueError(f"vqo_rht_f64 failed rc={rc}")
    return out


def rht_out_f64(y, signs) -> np.ndarray:
    """Output-side rotation of fp64 values [M,N]: signs * (1/sqrt N) H y (transform, then
    signs); block-diagonal like rht_f64 when N is not a power of two."""
    lib = _load()
    yd = _c(y, np.float64)
    sg = _c(signs, np.int8)
    M, N = yd.shape
    out = np.empty((M, N), dtype=np.float64)
    rc = lib.vqo_rht_out_f64(M, N, _p(yd), _p(sg), _p(out))
    if rc:
        raise ValueError(f"vqo_rht_out_f64 failed rc={rc}")
    return out


def tolerance(x_bits, xdt: int, w_exact: np.ndarray, coeff: float = 2e-3) -> np.ndarray:
    """Per-token bound coeff * ||x_m||_2 * max|w| used for the y comparison, shape [M, 1]."""
    xd = widen(np.asarray(x_bits, dtype=np.uint16), xdt)
    return coeff * np.sqrt((xd * xd).sum(axis=1, keepdims=True)) * np.abs(w_exact).max()


def widen(bits: np.ndarray, xdt: int) -> np.ndarray:
    """fp16/bf16 bits -> fp64 through numpy widening (exact); used to size tolerances."""
    if xdt == DT_F16:
        return bits.view(np.float16).astype(np.float64)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)

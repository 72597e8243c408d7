"""ctypes binding of libvqlinear's C ABI (include/vqlinear.h).

Argument marshalling only: every function here passes plain pointers and sizes
to the library of the same name and turns a non-OK status into ``VQError``.
Tensors are torch CUDA tensors (device memory and streams come from PyTorch);
their ``data_ptr()`` is what crosses the ABI.  There is no fallback: if the
shared library is missing or fails to load, ``load()`` raises.
"""

from __future__ import annotations

import ctypes
import os
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libvqlinear.so")

VQ_OK, VQ_ERR_INVALID_ARG, VQ_ERR_UNSUPPORTED, VQ_ERR_CUDA, VQ_ERR_NOMEM, VQ_ERR_TIMEOUT = range(6)
VQ_FMT_RVQ12, VQ_FMT_RVQ12_4, VQ_FMT_VQ16, VQ_FMT_VQ16_RVQ = 1, 2, 3, 4

# GLQ README, "Bit widths": bits per weight of the residual ladder -> (16-bit stages
# including the primary, 8-bit stages after them).
LADDER_STAGES = {2: (1, 0), 3: (1, 1), 4: (2, 0), 5: (2, 1), 6: (3, 0), 7: (3, 1), 8: (4, 0)}
VQ_F16, VQ_BF16 = 0, 1
VQ_PATH_AUTO, VQ_PATH_LUT, VQ_PATH_GEMV, VQ_PATH_TC, VQ_PATH_GATHER = 0, 1, 2, 3, 4

STATUS_NAMES = {0: "VQ_OK", 1: "VQ_ERR_INVALID_ARG", 2: "VQ_ERR_UNSUPPORTED", 3: "VQ_ERR_CUDA",
                4: "VQ_ERR_NOMEM", 5: "VQ_ERR_TIMEOUT"}

# Every entry point the header declares (checked by the tests against the .so).
EXPORTS = ("vq_abi_version", "vq_linear_create", "vq_linear_destroy", "vq_linear_set_path", "vq_linear_set_sm_budget",
           "vq_linear_forward",
           "vq_linear_forward_noalloc", "vq_linear_forward_rotated", "vq_linear_launches", "vq_linear_plan", "vq_plan_for_device", "vq_rht_apply", "vq_rht_apply_output", "vq_rht_apply_output_sharded", "vq_encode", "vq_linear_check", "vq_last_error",
           "vq_debug_unpack", "vq_debug_dequant", "vq_debug_wait_timeout")


class VQError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class vq_linear_desc(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int32), ("K", ctypes.c_int32), ("fmt", ctypes.c_int32),
                ("scale_group", ctypes.c_int32), ("act_dtype", ctypes.c_int32), ("max_M", ctypes.c_int32),
                ("rht", ctypes.c_int32), ("n16", ctypes.c_int32), ("n8", ctypes.c_int32),
                ("mult", ctypes.c_float * 3), ("corr", ctypes.c_int32)]


class vq_planes(ctypes.Structure):
    _fields_ = [("lo", ctypes.c_void_p), ("hi4", ctypes.c_void_p), ("s2", ctypes.c_void_p),
                ("idx16", ctypes.c_void_p), ("idx8", ctypes.c_void_p),
                ("corr_rows", ctypes.c_void_p), ("corr_cols", ctypes.c_void_p), ("corr_vals", ctypes.c_void_p)]


class vq_plan_info(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int32), ("launches", ctypes.c_int32), ("ctas", ctypes.c_int32),
                ("splits", ctypes.c_int32)]


class vq_codebooks(ctypes.Structure):
    _fields_ = [("cb1", ctypes.c_void_p), ("cb2", ctypes.c_void_p), ("cbr", ctypes.c_void_p * 3),
                ("cb8", ctypes.c_void_p)]


_lock = threading.Lock()
_lib = None


def load(path: str | None = None):
    """Load libvqlinear.so and declare its signatures (raises if it is missing)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise ImportError(f"{p} is missing: build it with compressed_index_matmul_b200.build.build()")
        lib = ctypes.CDLL(p)
        P, I32 = ctypes.c_void_p, ctypes.c_int32
        st = ctypes.c_int
        lib.vq_abi_version.restype = I32
        lib.vq_abi_version.argtypes = []
        lib.vq_last_error.restype = ctypes.c_char_p
        lib.vq_last_error.argtypes = []
        lib.vq_linear_create.restype = st
        lib.vq_linear_create.argtypes = [ctypes.POINTER(vq_linear_desc), ctypes.POINTER(P)]
        lib.vq_linear_destroy.restype = st
        lib.vq_linear_destroy.argtypes = [P]
        lib.vq_linear_set_path.restype = st
        lib.vq_linear_set_path.argtypes = [P, I32]
        lib.vq_linear_set_sm_budget.restype = st
        lib.vq_linear_set_sm_budget.argtypes = [P, I32]
        lib.vq_linear_forward.restype = st
        lib.vq_linear_forward.argtypes = [P, P, ctypes.POINTER(vq_planes), ctypes.POINTER(vq_codebooks), P, P,
                                          I32, I32, I32, P]
        lib.vq_linear_forward_noalloc.restype = st
        lib.vq_linear_forward_noalloc.argtypes = [ctypes.POINTER(vq_linear_desc), P, ctypes.POINTER(vq_planes),
                                                  ctypes.POINTER(vq_codebooks), P, P, I32, P]
        lib.vq_debug_wait_timeout.restype = st
        lib.vq_debug_wait_timeout.argtypes = [P, P]
        lib.vq_linear_launches.restype = I32
        lib.vq_linear_launches.argtypes = [P, I32]
        lib.vq_linear_plan.restype = st
        lib.vq_linear_plan.argtypes = [P, I32, ctypes.POINTER(vq_plan_info)]
        lib.vq_plan_for_device.restype = st
        lib.vq_plan_for_device.argtypes = [ctypes.POINTER(vq_linear_desc), I32, I32, I32, I32,
                                           ctypes.POINTER(vq_plan_info)]
        lib.vq_linear_forward_rotated.restype = st
        lib.vq_linear_forward_rotated.argtypes = [P, P, P, ctypes.POINTER(vq_planes), ctypes.POINTER(vq_codebooks), P,
                                                  P, I32, I32, I32, P]
        lib.vq_rht_apply.restype = st
        lib.vq_rht_apply.argtypes = [P, P, P, I32, I32, I32, P]
        lib.vq_rht_apply_output.restype = st
        lib.vq_rht_apply_output.argtypes = [P, P, P, I32, I32, I32, P]
        lib.vq_encode.restype = st
        lib.vq_encode.argtypes = [ctypes.POINTER(vq_linear_desc), P, P, ctypes.POINTER(vq_codebooks), P, P, P, P, P]
        lib.vq_rht_apply_output_sharded.restype = st
        lib.vq_rht_apply_output_sharded.argtypes = [P, P, P, I32, I32, ctypes.POINTER(I32), I32, I32, P]
        lib.vq_linear_check.restype = st
        lib.vq_linear_check.argtypes = [P, P]
        lib.vq_debug_unpack.restype = st
        lib.vq_debug_unpack.argtypes = [P, ctypes.POINTER(vq_planes), P, P, P]
        lib.vq_debug_dequant.restype = st
        lib.vq_debug_dequant.argtypes = [P, ctypes.POINTER(vq_planes), ctypes.POINTER(vq_codebooks), P, P, I32, P]
        _lib = lib
        return lib


def _check(status: int):
    if status != VQ_OK:
        raise VQError(status, load().vq_last_error().decode(errors="replace"))


def _ptr(t) -> int | None:
    """Device address of a tensor (or an int address, or None)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def make_planes(lo=None, hi4=None, s2=None, idx16=None, idx8=None, corr_rows=None, corr_cols=None,
                corr_vals=None) -> vq_planes:
    """corr_*: the sparse correction sidecar (CSR by output row), or None."""
    return vq_planes(_ptr(lo), _ptr(hi4), _ptr(s2), _ptr(idx16), _ptr(idx8), _ptr(corr_rows), _ptr(corr_cols),
                     _ptr(corr_vals))


def make_codebooks(cb1, cb2=None, cbr=(), cb8=None) -> vq_codebooks:
    """cbr: up to three codebooks (tensors or raw device addresses) of the ladder's 16-bit
    residual stages."""
    cbr = list(cbr) + [None] * (3 - len(cbr))
    return vq_codebooks(_ptr(cb1), _ptr(cb2), (ctypes.c_void_p * 3)(*[_ptr(c) for c in cbr]), _ptr(cb8))


def make_desc(N, K, fmt, scale_group, act_dtype, max_M, rht=0, n16=0, n8=0, mult=(), corr=0) -> vq_linear_desc:
    m = list(mult) + [0.0] * (3 - len(mult))
    return vq_linear_desc(N, K, fmt, scale_group, act_dtype, max_M, rht, n16, n8, (ctypes.c_float * 3)(*m), corr)


def vq_abi_version() -> int:
    return load().vq_abi_version()


def vq_linear_create(N, K, fmt, scale_group, act_dtype, max_M, rht=0, n16=0, n8=0, mult=(), corr=0) -> int:
    d = make_desc(N, K, fmt, scale_group, act_dtype, max_M, rht, n16, n8, mult, corr)
    h = ctypes.c_void_p()
    _check(load().vq_linear_create(ctypes.byref(d), ctypes.byref(h)))
    return h.value


def vq_linear_destroy(h) -> None:
    _check(load().vq_linear_destroy(h))


def vq_linear_set_path(h, path: int) -> None:
    _check(load().vq_linear_set_path(h, path))


def vq_linear_set_sm_budget(h, sms: int) -> None:
    _check(load().vq_linear_set_sm_budget(h, sms))


def vq_linear_launches(h, M: int) -> int:
    return load().vq_linear_launches(h, M)


def vq_linear_plan(h, M: int) -> dict:
    """How vq_linear_forward runs this M: path, launches, ctas, splits."""
    info = vq_plan_info()
    _check(load().vq_linear_plan(h, M, ctypes.byref(info)))
    return {name: getattr(info, name) for name, _ in vq_plan_info._fields_}


B200_SMS, B200_SMEM_OPTIN = 148, 232448


def vq_plan_for_device(N, K, fmt, scale_group, act_dtype, max_M, M, path=0, num_sms=B200_SMS,
                       smem_optin=B200_SMEM_OPTIN, rht=0, n16=0, n8=0, mult=(), corr=0) -> dict:
    """The plan of a forward of M tokens for such a layer on such a device (path 0 =
    automatic choice), computed on the host without a handle or a GPU."""
    d = make_desc(N, K, fmt, scale_group, act_dtype, max_M, rht, n16, n8, mult, corr)
    info = vq_plan_info()
    _check(load().vq_plan_for_device(ctypes.byref(d), M, path, num_sms, smem_optin, ctypes.byref(info)))
    return {name: getattr(info, name) for name, _ in vq_plan_info._fields_}


def vq_linear_forward(h, x, planes: vq_planes, codebooks: vq_codebooks, scales, y, M, N, K, stream=None) -> None:
    _check(load().vq_linear_forward(h, _ptr(x), ctypes.byref(planes), ctypes.byref(codebooks), _ptr(scales),
                                    _ptr(y), M, N, K, _stream(stream)))


def vq_linear_forward_rotated(h, x, signs, planes: vq_planes, codebooks: vq_codebooks, scales, y, M, N, K,
                              stream=None) -> None:
    """y = rotate(x) . W^T with the rotation's +-1 `signs` (int8 device tensor [K])."""
    _check(load().vq_linear_forward_rotated(h, _ptr(x), _ptr(signs), ctypes.byref(planes), ctypes.byref(codebooks),
                                            _ptr(scales), _ptr(y), M, N, K, _stream(stream)))


def vq_linear_forward_noalloc(N, K, fmt, scale_group, act_dtype, x, planes: vq_planes, codebooks: vq_codebooks,
                              scales, y, M, stream=None, rht=0, n16=0, n8=0, mult=(), corr=0) -> None:
    """Handle-free forward of 0 <= M <= 16 tokens that allocates nothing (fixed in-library scratch)."""
    d = make_desc(N, K, fmt, scale_group, act_dtype, max(M, 1), rht, n16, n8, mult, corr)
    _check(load().vq_linear_forward_noalloc(ctypes.byref(d), _ptr(x), ctypes.byref(planes), ctypes.byref(codebooks),
                                            _ptr(scales), _ptr(y), M, _stream(stream)))


def vq_rht_apply(x, x_out, signs, M, K, dtype, stream=None) -> None:
    _check(load().vq_rht_apply(_ptr(x), _ptr(x_out), _ptr(signs), M, K, dtype, _stream(stream)))


def vq_rht_apply_output(y, y_out, signs, M, N, dtype, stream=None) -> None:
    _check(load().vq_rht_apply_output(_ptr(y), _ptr(y_out), _ptr(signs), M, N, dtype, _stream(stream)))


def vq_encode(N, K, fmt, scale_group, w, scales, codebooks: vq_codebooks, lo=None, hi4=None, s2=None, idx16=None,
              stream=None) -> None:
    """Nearest-entry encode of fp32 W [N, K] (device) into the index planes (device outputs)."""
    d = make_desc(N, K, fmt, scale_group, VQ_F16, 1)
    _check(load().vq_encode(ctypes.byref(d), _ptr(w), _ptr(scales), ctypes.byref(codebooks), _ptr(lo), _ptr(hi4),
                            _ptr(s2), _ptr(idx16), _stream(stream)))


def vq_rht_apply_output_sharded(y, y_out, signs, M, N, shard_n, dtype, stream=None) -> None:
    """Output rotation of each column shard of y (sizes `shard_n`, a sequence of ints) in one launch."""
    arr = (ctypes.c_int32 * max(1, len(shard_n)))(*[int(v) for v in shard_n])
    _check(load().vq_rht_apply_output_sharded(_ptr(y), _ptr(y_out), _ptr(signs), M, N, arr if len(shard_n) else None,
                                              len(shard_n), dtype, _stream(stream)))


def vq_linear_check(h, stream=None) -> None:
    _check(load().vq_linear_check(h, _stream(stream)))


def vq_debug_unpack(h, planes: vq_planes, i1_out, i2_out=None, stream=None) -> None:
    _check(load().vq_debug_unpack(h, ctypes.byref(planes), _ptr(i1_out), _ptr(i2_out), _stream(stream)))


def vq_debug_dequant(h, planes: vq_planes, codebooks: vq_codebooks, scales, w_out, wdt, stream=None) -> None:
    _check(load().vq_debug_dequant(h, ctypes.byref(planes), ctypes.byref(codebooks), _ptr(scales), _ptr(w_out),
                                   wdt, _stream(stream)))


def vq_debug_wait_timeout(h, stream=None) -> None:
    _check(load().vq_debug_wait_timeout(h, _stream(stream)))

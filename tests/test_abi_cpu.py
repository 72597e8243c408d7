"""C-ABI checks that need no GPU: the library builds, loads, exports every entry
point include/vqlinear.h declares, and rejects bad arguments on the host before
touching CUDA."""

import ctypes
import os
import re

import pytest

from compressed_index_matmul_b200 import _binding as B
from compressed_index_matmul_b200 import build as libbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "vqlinear.h")


@pytest.fixture(scope="module")
def lib():
    libbuild.build()
    return B.load()


def declared_functions():
    import glob

    src = "".join(open(h).read() for h in sorted(glob.glob(os.path.join(ROOT, "include", "*.h"))))
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(vq_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(B.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert lib.vq_abi_version() == 3


def test_no_symbols_beyond_the_abi(lib):
    import subprocess

    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True, text=True).stdout
    syms = {ln.split()[-1] for ln in out.splitlines() if ln.strip()}
    ours = {s for s in syms if s.startswith("vq_")}
    assert ours == set(B.EXPORTS)


def _create(**kw):
    d = dict(N=64, K=256, fmt=B.VQ_FMT_RVQ12_4, scale_group=64, act_dtype=B.VQ_F16, max_M=4, rht=0)
    d.update(kw)
    return B.vq_linear_create(**d)


@pytest.mark.parametrize("kw,status", [
    (dict(N=0), B.VQ_ERR_INVALID_ARG),
    (dict(K=-64), B.VQ_ERR_INVALID_ARG),
    (dict(K=72), B.VQ_ERR_INVALID_ARG),         # not a multiple of 16
    (dict(K=80), B.VQ_ERR_UNSUPPORTED),         # multiple of 16, not of 64
    (dict(fmt=7), B.VQ_ERR_INVALID_ARG),
    (dict(scale_group=12), B.VQ_ERR_INVALID_ARG),
    (dict(scale_group=128), B.VQ_ERR_UNSUPPORTED),
    (dict(act_dtype=5), B.VQ_ERR_INVALID_ARG),
    (dict(max_M=0), B.VQ_ERR_INVALID_ARG),
    # residual ladder: stage counts and multipliers
    (dict(fmt=B.VQ_FMT_VQ16_RVQ, n16=0, n8=0), B.VQ_ERR_INVALID_ARG),
    (dict(fmt=B.VQ_FMT_VQ16_RVQ, n16=5, n8=0), B.VQ_ERR_INVALID_ARG),
    (dict(fmt=B.VQ_FMT_VQ16_RVQ, n16=2, n8=2), B.VQ_ERR_INVALID_ARG),
    (dict(fmt=B.VQ_FMT_VQ16_RVQ, n16=4, n8=1), B.VQ_ERR_INVALID_ARG),  # 9 bpw: not in the table
    (dict(fmt=B.VQ_FMT_VQ16_RVQ, n16=2, n8=1, mult=(0.1, float("nan"))), B.VQ_ERR_INVALID_ARG),
    (dict(fmt=B.VQ_FMT_VQ16_RVQ, n16=3, n8=0, mult=(float("inf"), 0.1)), B.VQ_ERR_INVALID_ARG),
    # sparse correction: a flag, and not defined for the residual ladder
    (dict(corr=2), B.VQ_ERR_INVALID_ARG),
    (dict(fmt=B.VQ_FMT_VQ16_RVQ, n16=2, n8=0, mult=(0.1,), corr=1), B.VQ_ERR_UNSUPPORTED),
])
def test_create_rejects_bad_descriptors(lib, kw, status):
    with pytest.raises(B.VQError) as ei:
        _create(**kw)
    assert ei.value.status == status
    assert lib.vq_last_error()


def test_ladder_struct_layout_matches_the_header():
    """The ctypes mirrors of the three ABI structs have the C layout: the ladder fields
    follow the original ones, the sparse correction's fields follow those (ABI 3)."""
    assert ctypes.sizeof(B.vq_linear_desc) == 7 * 4 + 2 * 4 + 3 * 4 + 4
    assert B.vq_linear_desc.n16.offset == 28 and B.vq_linear_desc.mult.offset == 36
    assert B.vq_linear_desc.corr.offset == 48
    assert ctypes.sizeof(B.vq_planes) == 8 * 8 and B.vq_planes.idx8.offset == 32
    assert B.vq_planes.corr_rows.offset == 40 and B.vq_planes.corr_vals.offset == 56
    assert ctypes.sizeof(B.vq_codebooks) == 6 * 8 and B.vq_codebooks.cb8.offset == 40


def test_ladder_stage_table():
    """GLQ README, "Bit widths": bits per weight = 2 n16 + n8, at most four stages."""
    for bpw, (n16, n8) in B.LADDER_STAGES.items():
        assert 2 * n16 + n8 == bpw and n16 + n8 <= 4 and n8 <= 1


def test_null_arguments_are_rejected(lib):
    assert lib.vq_linear_create(None, None) == B.VQ_ERR_INVALID_ARG
    assert lib.vq_linear_forward(None, None, None, None, None, None, 1, 1, 1, None) == B.VQ_ERR_INVALID_ARG
    assert lib.vq_linear_set_path(None, 0) == B.VQ_ERR_INVALID_ARG
    assert lib.vq_linear_set_sm_budget(None, 0) == B.VQ_ERR_INVALID_ARG
    assert lib.vq_linear_launches(None, 1) == -1
    assert lib.vq_linear_plan(None, 1, None) == B.VQ_ERR_INVALID_ARG
    assert lib.vq_linear_destroy(None) == B.VQ_OK
    assert lib.vq_linear_check(None, None) == B.VQ_ERR_INVALID_ARG


@pytest.mark.parametrize("M,K,dt,x,xo,signs", [
    (1, 100, 0, 16, 16, 16),      # K not a multiple of 64
    (1, 96, 0, 16, 16, 16),       # K not a multiple of 64
    (1, 32, 0, 16, 16, 16),       # K below 64
    (1, 65536, 0, 16, 16, 16),    # K above 32768
    (-1, 64, 0, 16, 16, 16),
    (1, 64, 3, 16, 16, 16),       # bad dtype
    (1, 64, 0, 0, 16, 16),        # NULL x
    (1, 64, 0, 24, 16, 16),       # misaligned x
    (1, 64, 0, 16, 16, 0),        # NULL signs
    (1, 64, 0, 16, 16, 24),       # misaligned signs (read in 8-byte words)
    (2, 64, 0, 1024, 1024 + 64, 16),  # partial overlap
])
def test_rht_rejects_bad_arguments_without_a_gpu(lib, M, K, dt, x, xo, signs):
    assert lib.vq_rht_apply(x or None, xo or None, signs or None, M, K, dt, None) == B.VQ_ERR_INVALID_ARG
    assert lib.vq_rht_apply_output(x or None, xo or None, signs or None, M, K, dt, None) == B.VQ_ERR_INVALID_ARG


@pytest.mark.parametrize("shards,N,signs,xo", [
    (None, 64, 16, 16),              # NULL shard sizes
    ((), 64, 16, 16),                # no shard
    ((64,) * 17, 64 * 17, 16, 16),   # more than 16 shards
    ((96,), 96, 16, 16),             # not a multiple of 64
    ((65536,), 65536, 16, 16),       # above 32768
    ((64, 128), 256, 16, 16),        # the shards do not add up to N
    ((64, 128), 192, 24, 16),        # misaligned signs
    ((64, 128), 192, 16, 16 + 64),   # y_out partially overlaps y (M = 2)
])
def test_rht_sharded_rejects_bad_arguments_without_a_gpu(lib, shards, N, signs, xo):
    if shards is None:
        rc = lib.vq_rht_apply_output_sharded(16, xo, signs, 2, N, None, 1, 0, None)
    else:
        arr = (ctypes.c_int32 * max(1, len(shards)))(*shards)
        rc = lib.vq_rht_apply_output_sharded(16, xo, signs, 2, N, arr, len(shards), 0, None)
    assert rc == B.VQ_ERR_INVALID_ARG


def test_python_binding_raises_with_message(lib):
    with pytest.raises(B.VQError, match="multiple of 64"):
        B.vq_rht_apply(16, 16, 16, 1, 100, 0, stream=0)


def test_zero_rows_return_before_touching_the_device(lib):
    """M = 0 is valid for every rotation entry point and returns VQ_OK after the host-side
    checks, without a launch (so without a GPU)."""
    assert lib.vq_rht_apply(16, 16, 16, 0, 2688, 0, None) == B.VQ_OK
    assert lib.vq_rht_apply_output(16, 16, 16, 0, 192, 1, None) == B.VQ_OK
    arr = (ctypes.c_int32 * 3)(4096, 1024, 1024)
    assert lib.vq_rht_apply_output_sharded(16, 16, 16, 0, 6144, arr, 3, 0, None) == B.VQ_OK


def test_encode_rejects_bad_arguments_without_a_gpu(lib):
    cbs = B.make_codebooks(16, 16)
    def enc(**kw):
        a = dict(N=8, K=128, fmt=B.VQ_FMT_RVQ12_4, scale_group=64, w=16, scales=16, lo=16, hi4=16, s2=16, idx16=None)
        a.update(kw)
        d = B.make_desc(a["N"], a["K"], a["fmt"], a["scale_group"], B.VQ_F16, 1)
        return lib.vq_encode(ctypes.byref(d), a["w"], a["scales"], ctypes.byref(cbs), a["lo"], a["hi4"], a["s2"],
                             a["idx16"], None)
    assert lib.vq_encode(None, 16, 16, ctypes.byref(cbs), 16, 16, 16, None, None) == B.VQ_ERR_INVALID_ARG
    assert enc(w=None) == B.VQ_ERR_INVALID_ARG
    assert enc(w=24) == B.VQ_ERR_INVALID_ARG          # misaligned
    assert enc(s2=None) == B.VQ_ERR_INVALID_ARG       # the two-stage format writes s2
    assert enc(fmt=B.VQ_FMT_VQ16, idx16=None) == B.VQ_ERR_INVALID_ARG
    assert enc(K=72) == B.VQ_ERR_INVALID_ARG
    assert enc(K=256, scale_group=128) == B.VQ_ERR_UNSUPPORTED
    assert enc(fmt=B.VQ_FMT_VQ16_RVQ) == B.VQ_ERR_INVALID_ARG  # ladder stage counts of zero


def test_missing_library_fails_loudly():
    """No CPU fallback: loading a library that is not there raises ImportError."""
    import subprocess
    import sys

    code = ("from compressed_index_matmul_b200 import _binding as B\n"
            "try:\n    B.load('/nonexistent/libvqlinear.so')\nexcept ImportError:\n    raise SystemExit(7)\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True)
    assert r.returncode == 7, r.stderr


def test_product_package_never_uses_the_oracle():
    """The oracle is test infrastructure: nothing in the product package imports, loads or
    names its module or library."""
    pkg = os.path.join(ROOT, "compressed_index_matmul_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"\boracle\b|vq_oracle|vqo_", src), os.path.join(dirpath, f)


def test_struct_offsets_match_the_c_header(tmp_path):
    """The ctypes mirrors against the real header: a C program built with gcc prints every
    field's offsetof and each struct's sizeof."""
    import subprocess

    fields = {"vq_linear_desc": [f for f, _ in B.vq_linear_desc._fields_],
              "vq_planes": [f for f, _ in B.vq_planes._fields_],
              "vq_codebooks": [f for f, _ in B.vq_codebooks._fields_],
              "vq_plan_info": [f for f, _ in B.vq_plan_info._fields_]}
    src = ["#include <stddef.h>", "#include <stdio.h>", '#include "vqlinear.h"', "int main(void) {"]
    for st, fs in fields.items():
        src.append(f'  printf("{st} sizeof %zu\\n", sizeof({st}));')
        for f in fs:
            src.append(f'  printf("{st} {f} %zu\\n", offsetof({st}, {f}));')
    src.append("  return 0;\n}")
    c = tmp_path / "offsets.c"
    c.write_text("\n".join(src))
    exe = tmp_path / "offsets"
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    subprocess.run(["gcc", "-std=c11", "-I", inc, "-I", "/usr/local/cuda/include", str(c), "-o", str(exe)],
                   check=True)
    got = {}
    for ln in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.splitlines():
        st, f, v = ln.split()
        got[(st, f)] = int(v)
    for st, fs in fields.items():
        cls = getattr(B, st)
        assert got[(st, "sizeof")] == ctypes.sizeof(cls), st
        for f in fs:
            assert got[(st, f)] == getattr(cls, f).offset, (st, f)

"""Build libvqlinear.so (CUDA sm_100a + C++ host code) in-tree with nvcc.

Every .cu file under csrc/ is compiled to an object with
``-gencode arch=compute_100a,code=sm_100a -lineinfo -O3`` and linked into one
shared library with a static CUDA runtime, so the library does not depend on
which libcudart the host process has loaded.  Only the ``extern "C"`` entry
points of include/vqlinear.h are exported.
"""

from __future__ import annotations

import concurrent.futures as cf
import glob
import hashlib
import re
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libvqlinear.so")
BUILD_DIR = os.path.join(ROOT, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr", "-Xcompiler",
                     "-fPIC,-fvisibility=hidden", "-I", INCLUDE, "-I", CSRC]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


_INCLUDE_RE = re.compile(r'^\s*#\s*include\s+"([^"]+)"', re.M)


def _unit_files(unit: str) -> list:
    """A translation unit under csrc/ and every header it includes, transitively (quoted
    includes, looked up in csrc/ and include/ as the compile flags do)."""
    seen, todo = set(), [os.path.join(CSRC, unit)]
    while todo:
        f = todo.pop()
        if f in seen:
            continue
        seen.add(f)
        with open(f) as fh:
            for name in _INCLUDE_RE.findall(fh.read()):
                for d in (CSRC, INCLUDE):
                    cand = os.path.join(d, name)
                    if os.path.exists(cand):
                        todo.append(cand)
                        break
    return sorted(seen)


def _deps_hash(unit: str | None = None) -> str:
    h = hashlib.sha256()
    if unit is None:
        files = _sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) +
                                    glob.glob(os.path.join(INCLUDE, "*.h")))
    else:
        files = _unit_files(unit)
    # paths relative to the repository root, so the same sources hash the same wherever
    # the repository is checked out
    for f in files:
        h.update(os.path.relpath(f, ROOT).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    h.update(" ".join(NVCC_FLAGS).replace(ROOT, "<root>").encode())
    return h.hexdigest()


def source_digest(unit: str | None = None) -> str:
    """Hash of every kernel/ABI source and the compile flags (identifies a build of the kernels);
    with `unit` (a file name under csrc/), of that translation unit, the headers it includes
    (transitively) and the flags (identifies a build of the kernels defined in it)."""
    return _deps_hash(unit)[:16]


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    """Compile the library if any source changed; return the path of the .so."""
    stamp = LIB + ".hash"
    digest = _deps_hash()
    if not force and os.path.exists(LIB) and os.path.exists(stamp) and open(stamp).read() == digest:
        return LIB
    os.makedirs(BUILD_DIR, exist_ok=True)
    nvcc = _nvcc()
    extra = ["-Xptxas", "-v"] if ptxas_info else []

    def compile_one(src):
        obj = os.path.join(BUILD_DIR, os.path.basename(src) + ".o")
        cmd = [nvcc, *NVCC_FLAGS, *extra, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
        if verbose or ptxas_info:
            sys.stderr.write(r.stdout + r.stderr)
        return obj

    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(compile_one, _sources()))
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    with open(stamp, "w") as f:
        f.write(digest)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, ptxas_info="--ptxas" in sys.argv))

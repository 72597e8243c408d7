"""Host-side logic of bench.py on CPU: the max-over-ranks aggregation with two
gloo ranks, and the algorithmic byte counts."""

import os
import socket

import pytest
import torch.multiprocessing as mp

import bench
from synth import CONFIGS, LayerSpec, FMT_RVQ12_4, FMT_VQ16


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    local = [10.0, 30.0][rank]  # rank 1 is the slow one
    out = bench.aggregate_over_ranks(local, steps=5, layers_per_step=3, world=world)
    q.put((rank, out))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in (0, 1):
        ms_per_step, us_per_layer = res[r]
        assert ms_per_step == pytest.approx(30.0 / 5)
        assert us_per_layer == pytest.approx(1e3 * 6.0 / (3 * 2))


def test_single_rank_is_identity():
    assert bench.aggregate_over_ranks(12.0, 4, 3, 1) == (3.0, 1e3 * 3.0 / 3)


def test_layer_bytes_match_the_format_arithmetic():
    spec = LayerSpec(14336, 4096, FMT_RVQ12_4, 64)
    b = bench.layer_bytes(spec, 1)
    per_weight = 0.28125
    assert b == int(spec.N * spec.K * per_weight) + 4096 * 16 + 256 + 4096 * 2 + 14336 * 2
    spec16 = LayerSpec(4096, 4096, FMT_VQ16, 4096)
    assert bench.layer_bytes(spec16, 8) == 4096 * 512 * 2 + 4096 * 2 + 65536 * 16 + 8 * 4096 * 2 * 2
    # the headline workload's three tensors have equal byte counts
    sizes = {bench.layer_bytes(s, 1) for _, s in CONFIGS[4]["tensors"]}
    assert len(sizes) == 1


def test_ladder_bytes_and_workloads():
    """The residual ladder's algorithmic bytes: one 2-byte index per group per 16-bit stage and
    one byte for the 8-bit stage, a 1 MiB codebook per 16-bit stage and 4 KiB for the 8-bit one
    (GLQ README, "Bit widths": 5 bpw = 16 + 16 + 8)."""
    from synth import FMT_VQ16_RVQ

    spec = LayerSpec(4096, 4096, FMT_VQ16_RVQ, 4096, bpw=5)
    G = 512
    assert bench.layer_bytes(spec, 1) == 4096 * G * 5 + 4096 * 2 + 2 * 65536 * 16 + 256 * 16 + 4096 * 2 * 2
    # bits per weight of the planes alone
    planes = bench.layer_bytes(spec, 0) - 4096 * 2 - 2 * 65536 * 16 - 256 * 16
    assert planes * 8 / (4096 * 4096) == 5.0
    for bpw in (3, 4, 5):
        cfg = bench._workload_config(f"vq16-ladder-4096-{bpw}bpw")
        (_, s), = cfg["tensors"]
        assert (s.fmt, s.bpw, s.N, s.K) == (FMT_VQ16_RVQ, bpw, 4096, 4096)
    assert bench._workload_config("llama3-8b-mlp") is CONFIGS[4]


def test_source_digest_does_not_depend_on_the_checkout_path(tmp_path):
    """The traffic figures are keyed by a digest of each kernel's translation unit and the
    headers it includes; a copy of the sources elsewhere (as on a GPU machine) hashes the same."""
    import importlib.util
    import shutil

    from compressed_index_matmul_b200 import build as b

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    pkg = tmp_path / "compressed_index_matmul_b200"
    shutil.copytree(os.path.join(root, "compressed_index_matmul_b200", "csrc"), pkg / "csrc")
    shutil.copy(os.path.join(root, "compressed_index_matmul_b200", "build.py"), pkg / "build.py")
    shutil.copytree(os.path.join(root, "include"), tmp_path / "include")
    spec = importlib.util.spec_from_file_location("build_copy", pkg / "build.py")
    copy = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(copy)
    for unit in ("lut_gemv.cu", "vq16_gemv.cu", "tc_gemm.cu"):
        assert copy.source_digest(unit) == b.source_digest(unit)
        assert [os.path.relpath(f, tmp_path) for f in copy._unit_files(unit)] == \
               [os.path.relpath(f, root) for f in b._unit_files(unit)]

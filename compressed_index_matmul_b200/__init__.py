"""Codebook-VQ linear layer for NVIDIA B200 (sm_100a), computed from compressed indices.

The compute lives in ``libvqlinear.so`` (CUDA kernels behind the C ABI declared in
``include/vqlinear.h``).  This package only marshals arguments to it:

* ``_binding``  -- ctypes binding with the C ABI's names
* ``layer``     -- ``VQLinear``: one layer's device tensors plus a handle
* ``build``     -- compiles the library in-tree with nvcc
"""

from ._binding import (  # noqa: F401
    EXPORTS,
    VQ_BF16,
    VQ_F16,
    VQ_FMT_RVQ12,
    VQ_FMT_RVQ12_4,
    VQ_FMT_VQ16,
    VQ_FMT_VQ16_RVQ,
    LADDER_STAGES,
    VQ_PATH_AUTO,
    VQ_PATH_GATHER,
    VQ_PATH_GEMV,
    VQ_PATH_LUT,
    VQ_PATH_TC,
    VQError,
    load,
    make_codebooks,
    make_planes,
    vq_abi_version,
    vq_debug_dequant,
    vq_debug_unpack,
    vq_debug_wait_timeout,
    vq_encode,
    vq_linear_check,
    vq_linear_create,
    vq_linear_destroy,
    vq_linear_forward,
    vq_linear_forward_noalloc,
    vq_linear_forward_rotated,
    vq_linear_launches,
    vq_linear_plan,
    vq_linear_set_path,
    vq_linear_set_sm_budget,
    vq_plan_for_device,
    vq_rht_apply,
    vq_rht_apply_output,
    vq_rht_apply_output_sharded,
)
from .layer import VQLinear  # noqa: F401

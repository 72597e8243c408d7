"""Seeded synthetic inputs for the codebook-VQ linear layer.

This module is shared by the CPU oracle's tests and by the CUDA path's tests and
benchmark.  It only draws random numbers and lays them out in the storage format;
it holds none of the method's arithmetic (no unpacking, no decoding, no matmul,
no Hadamard transform).  Because stage indices are drawn uniformly, the packed
bit-planes are themselves uniform random bytes, so no packing step is needed.

Storage format (the encoder's output, consumed by both implementations):

* weights W are N x K (out x in); each run of 8 consecutive weights along K is
  one group, G = K // 8 groups per row (orka README, "How it works": each group
  of 8 values is replaced by one codebook index).
* planes are flat arrays in K-slice-major order: K is cut into slices of 16
  groups (128 inputs); slice s holds w_s = min(16, G - 16 s) groups; inside a
  slice the rows' entries are contiguous, one row after another.
* ``lo``  uint8  [N*G]      low 8 bits of the 12-bit stage-1 index
* ``hi4`` uint8  [N*G/2]    high 4 bits of the stage-1 index, two groups per
  byte within a row's slice entries: group 2t in bits 0..3, group 2t+1 in 4..7
* ``s2``  uint8  [N*G/2]    4-bit stage-2 index, packed like ``hi4``
* ``idx16`` uint16 [N*G]    16-bit single-stage index (GLQ README, "How it
  works", E8 lattice codebooks: one 16-bit index per group of 8); for the
  residual ladder [n16*N*G], one plane per 16-bit stage, stage-major
* ``idx8`` uint8 [N*G]      the ladder's 8-bit stage index, same layout as ``lo``
* ``cbr`` fp16 [n16-1, 65536, 8], ``cb8`` fp16 [256, 8], ``mult`` fp32 [n16-1+n8]:
  the ladder's residual codebooks and stage multipliers (GLQ README, "Bit widths")
* ``cb1`` fp16 [4096, 8] (or [65536, 8] for 16-bit indices), ``cb2`` fp16 [16, 8]
* ``scales`` fp16 [N * K // scale_group]: block scales (scale_group dividing 64)
  in K-slice-major order like the planes (a row's scales of one slice are
  adjacent); ``scale_group == K`` is one scale per row, [N]
* ``x`` fp16 or bf16 [M, K]; ``signs`` int8 [K] of +-1 for the input rotation
* ``corr`` (optional, ``make_correction``): a sparse correction by output row,
  ``row_ptr`` int32 [N+1], ``col`` int32 [nnz] (increasing within a row),
  ``val`` fp16 [nnz] (orka README, "How it works": "(+ sparse correction)")

fp16/bf16 arrays are returned as raw uint16 bit patterns.
"""

from .layers import (  # noqa: F401
    FMT_RVQ12,
    FMT_RVQ12_4,
    FMT_VQ16,
    FMT_VQ16_RVQ,
    DT_F16,
    DT_BF16,
    LayerSpec,
    make_layer,
    make_correction,
    make_x,
    make_signs,
    f32_to_bf16_bits,
    f32_to_f16_bits,
    CONFIGS,
    config_layers,
)

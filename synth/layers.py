"""Seeded generators for synthetic compressed layers and activations.

Recipe (one ``numpy.random.Generator`` per tensor, seeded from
``SeedSequence([cfg_id, layer, tensor_id, seed])``):

* stage-1 codebook: 4096 x 8 (12-bit) or 65536 x 8 (16-bit) fp16 values ~ N(0, 1)
* stage-2 codebook: 16 x 8 fp16 ~ N(0, 1)
* residual ladder (16-bit primary + residual stages): one 65536 x 8 codebook per
  16-bit stage and a 256 x 8 codebook for the 8-bit stage, all fp16 ~ N(0, 1);
  stage multipliers (inverse residual scales) fp32 4^-(s-1) * U(0.25, 0.5) for
  residual stage s = 1, 2, 3
* indices: uniform over their range, i.e. the packed planes are uniform random bytes
* scales: fp16 lognormal(mu=-4, sigma=0.5), per 64-weight block along K or per row
* activations: fp16 or bf16 ~ N(0, 1); rotation signs: +-1 with probability 1/2

No arithmetic of the method lives here.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

FMT_RVQ12 = 1     # one 12-bit stage (lo byte + packed hi nibble)
FMT_RVQ12_4 = 2   # 12-bit stage 1 + 4-bit stage 2
FMT_VQ16 = 3      # one 16-bit index into a 65,536 x 8 codebook
FMT_VQ16_RVQ = 4  # 16-bit primary + residual stages (16-bit ones, then at most one 8-bit)

DT_F16 = 0
DT_BF16 = 1


def f32_to_f16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to fp16 (numpy's IEEE round-to-nearest-even) and return the bits."""
    return np.asarray(a, dtype=np.float32).astype(np.float16).view(np.uint16)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 with torch's CPU conversion and return the bits."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


@dataclass(frozen=True)
class LayerSpec:
    N: int
    K: int
    fmt: int
    scale_group: int  # 64, or K for one scale per row
    bpw: int = 2      # FMT_VQ16_RVQ: bits per weight, 2..8 (GLQ README, "Bit widths")

    @property
    def G(self) -> int:
        return self.K // 8

    @property
    def n16(self) -> int:
        """16-bit stages of the ladder (primary included): bpw // 2."""
        return self.bpw // 2

    @property
    def n8(self) -> int:
        """8-bit stages after them: 1 for odd bpw."""
        return self.bpw % 2


def _rng(cfg_id: int, layer: int, tensor_id: int, seed: int, stream: int = 0) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([cfg_id, layer, tensor_id, seed, stream]))


def make_layer(spec: LayerSpec, cfg_id: int = 0, layer: int = 0, tensor_id: int = 0, seed: int = 0) -> dict:
    """Draw one compressed layer in the storage format described in the package docstring."""
    N, K, G = spec.N, spec.K, spec.G
    if K % 16 != 0 or K % spec.scale_group != 0:
        raise ValueError(f"K={K} must be a multiple of 16 and of scale_group={spec.scale_group}")
    r = _rng(cfg_id, layer, tensor_id, seed)
    out: dict = {"spec": spec}
    # Planes are flat arrays (their element order is the K-slice-major storage order;
    # the values are iid uniform, so the generator needs no layout arithmetic).
    if spec.fmt == FMT_VQ16:
        out["cb1"] = f32_to_f16_bits(r.standard_normal((65536, 8), dtype=np.float32))
        out["idx16"] = r.integers(0, 65536, size=N * G, dtype=np.uint16)
    elif spec.fmt == FMT_VQ16_RVQ:
        if not 2 <= spec.bpw <= 8:
            raise ValueError(f"bpw={spec.bpw} outside 2..8")
        n16, n8 = spec.n16, spec.n8
        out["cb1"] = f32_to_f16_bits(r.standard_normal((65536, 8), dtype=np.float32))
        # residual 16-bit codebooks, stage-major [n16 - 1, 65536, 8]
        out["cbr"] = f32_to_f16_bits(r.standard_normal((n16 - 1, 65536, 8), dtype=np.float32))
        out["cb8"] = f32_to_f16_bits(r.standard_normal((256, 8), dtype=np.float32))
        # stage-major planes: 16-bit stage s at entries [s N G, (s + 1) N G)
        out["idx16"] = r.integers(0, 65536, size=n16 * N * G, dtype=np.uint16)
        out["idx8"] = r.integers(0, 256, size=N * G, dtype=np.uint8) if n8 else None
        nres = n16 - 1 + n8
        out["mult"] = (4.0 ** -np.arange(nres) * r.uniform(0.25, 0.5, size=nres)).astype(np.float32)
    else:
        out["cb1"] = f32_to_f16_bits(r.standard_normal((4096, 8), dtype=np.float32))
        out["lo"] = r.integers(0, 256, size=N * G, dtype=np.uint8)
        out["hi4"] = r.integers(0, 256, size=N * G // 2, dtype=np.uint8)
        if spec.fmt == FMT_RVQ12_4:
            out["cb2"] = f32_to_f16_bits(r.standard_normal((16, 8), dtype=np.float32))
            out["s2"] = r.integers(0, 256, size=N * G // 2, dtype=np.uint8)
    nblk = K // spec.scale_group
    # flat, in the scales' storage order (K-slice-major for block scales, [N] per row)
    out["scales"] = f32_to_f16_bits(r.lognormal(-4.0, 0.5, size=N * nblk).astype(np.float32))
    return out


def make_correction(N: int, K: int, density: float = 0.002, cfg_id: int = 0, layer: int = 0, tensor_id: int = 0,
                    seed: int = 0, scale: float = 0.05) -> dict:
    """A sparse correction sidecar for an N x K layer (orka README, "How it works": the
    decode's "(+ sparse correction)"), by output row: row n's entries are
    row_ptr[n] .. row_ptr[n+1]-1, with distinct columns in increasing order and fp16
    values.  Each weight is corrected with probability `density`; values ~ N(0, scale^2),
    a few times the synthetic layers' decoded weights, as corrections of outliers are."""
    r = _rng(cfg_id, layer, tensor_id, seed, stream=7)
    counts = r.binomial(K, density, size=N).astype(np.int64)
    row_ptr = np.zeros(N + 1, dtype=np.int32)
    row_ptr[1:] = np.cumsum(counts)
    cols = [np.sort(r.choice(K, size=int(c), replace=False)) for c in counts]
    col = (np.concatenate(cols) if N else np.zeros(0)).astype(np.int32)
    val = f32_to_f16_bits((r.standard_normal(int(row_ptr[-1])) * scale).astype(np.float32))
    return {"row_ptr": row_ptr, "col": col, "val": val}


def make_x(M: int, K: int, dtype: int, cfg_id: int = 0, seed: int = 0, stream: int = 1) -> np.ndarray:
    """Activations [M, K] ~ N(0, 1) as fp16 or bf16 bits."""
    r = _rng(cfg_id, 1_000_000, M, seed, stream)
    a = r.standard_normal((M, K), dtype=np.float32)
    return f32_to_f16_bits(a) if dtype == DT_F16 else f32_to_bf16_bits(a)


def make_signs(K: int, cfg_id: int = 0, seed: int = 0) -> np.ndarray:
    """Random +-1 signs for the input rotation, as int8."""
    r = _rng(cfg_id, 2_000_000, K, seed)
    return np.where(r.integers(0, 2, size=K) == 1, 1, -1).astype(np.int8)


# The five workloads: (name, cfg_id, list of (label, LayerSpec), activation dtype, token counts, rht)
def _smollm_layer_specs():
    f = FMT_RVQ12_4
    return [
        ("q", LayerSpec(576, 576, f, 64)),
        ("k", LayerSpec(192, 576, f, 64)),
        ("v", LayerSpec(192, 576, f, 64)),
        ("o", LayerSpec(576, 576, f, 64)),
        ("gate", LayerSpec(1536, 576, f, 64)),
        ("up", LayerSpec(1536, 576, f, 64)),
        ("down", LayerSpec(576, 1536, f, 64)),
    ]


CONFIGS = {
    1: dict(name="single-256x256-rvq12", layers=1,
            tensors=[("w", LayerSpec(256, 256, FMT_RVQ12, 64))], act=DT_F16, Ms=(1,), rht=False),
    2: dict(name="smollm-135m-stack-rvq12_4", layers=30, tensors=_smollm_layer_specs(),
            act=DT_F16, Ms=(1, 4, 16), rht=False),
    3: dict(name="vq16-4096x4096-rht", layers=1,
            tensors=[("w", LayerSpec(4096, 4096, FMT_VQ16, 4096))], act=DT_F16, Ms=(1, 8), rht=True),
    4: dict(name="llama3-8b-mlp-rvq12_4", layers=1,
            tensors=[("gate", LayerSpec(14336, 4096, FMT_RVQ12_4, 64)),
                     ("up", LayerSpec(14336, 4096, FMT_RVQ12_4, 64)),
                     ("down", LayerSpec(4096, 14336, FMT_RVQ12_4, 64))],
            act=DT_BF16, Ms=(1, 4, 16), rht=False),
    5: dict(name="prefill-8192x8192-rvq12_4", layers=1,
            tensors=[("w", LayerSpec(8192, 8192, FMT_RVQ12_4, 64))], act=DT_BF16, Ms=(64, 256, 1024), rht=False),
}


def config_layers(cfg_id: int, seed: int = 0, layers: int | None = None):
    """Yield (layer, label, tensor_id, layer_dict) for every tensor of a workload."""
    c = CONFIGS[cfg_id]
    nl = c["layers"] if layers is None else layers
    for li in range(nl):
        for ti, (label, spec) in enumerate(c["tensors"]):
            yield li, label, ti, make_layer(spec, cfg_id=cfg_id, layer=li, tensor_id=ti, seed=seed)

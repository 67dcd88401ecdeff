"""Seeded synthetic BF16 workloads, shared by the tests, the bench and the smoke check.

This module only draws inputs. It holds none of the codec's arithmetic, so the oracle
and the GPU library can both consume what it produces.

The five workloads:

1. ``tensor_1m``: one 1024x1024 tensor, N(0, 0.02) rounded to BF16.
2. ``gemma2_layer``: one decoder layer shaped like Gemma-2-9B. The Gemma 2 article
   gives 42 layers, hidden 3584, 16 heads and 8 KV heads (head dim 256).
   * matrices q 3584x4096, k 3584x2048, v 3584x2048, o 4096x3584,
     gate 3584x14336, up 3584x14336, down 14336x3584;
   * weights N(0, sigma) with sigma ~ U[0.01, 0.05] per tensor;
   * four RMSNorm vectors of 3584 drawn N(1.0, 0.05).
3. ``gemma2_9b``: 42 such layers plus a 256000x3584 embedding, N(0, 0.02)
   (9,241,702,400 weights).
4. ``edge_mix``:
   * five 4096x4096 tensors: Student-t nu=3 scaled to std 0.02, N(0, 0.02) with 0.1%
     of entries multiplied by 50, all zeros, all 1.0, and uniform random 16-bit
     patterns;
   * a 1-element and a 4097-element N(0, 0.02) tensor;
   * a 1 KiB opaque byte span.
5. ``qwen_27b_scale``: 64 layers (q/o 5120x6144 and 6144x5120, k/v 5120x1024,
   gate/up 5120x25600, down 25600x5120, sigma ~ U[0.005, 0.04]) plus a 152064x5120
   embedding (30,642,012,160 weights: the literal shapes).

Every tensor has its own seed, ``1_000_003 * workload_seed + index``. Draws use
``torch.Generator`` on the device asked for, so the values depend on the device. Each
test regenerates its originals on the device it checks on. BF16 rounding is torch's
float32 -> bfloat16 conversion (round to nearest even).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class TensorSpec:
    name: str
    shape: tuple
    dist: str          # normal | norm_vec | t3 | outliers | zeros | ones | uniform16 | raw
    sigma: float = 0.0
    seed: int = 0

    @property
    def numel(self) -> int:
        return math.prod(self.shape)

    @property
    def is_raw(self) -> bool:
        return self.dist == "raw"


def _seed(workload_seed: int, index: int) -> int:
    return 1_000_003 * workload_seed + index


def _sigma(seed: int, lo: float, hi: float) -> float:
    g = torch.Generator().manual_seed(seed ^ 0x5EED)
    return lo + (hi - lo) * float(torch.rand(1, generator=g, dtype=torch.float64))


def _layer(prefix: str, shapes: dict, lo: float, hi: float, norms: int, hidden: int, seed0: int, idx: list):
    out = []
    for nm, shp in shapes.items():
        s = _seed(seed0, idx[0])
        out.append(TensorSpec(f"{prefix}.{nm}", shp, "normal", _sigma(s, lo, hi), s))
        idx[0] += 1
    for k in range(norms):
        s = _seed(seed0, idx[0])
        out.append(TensorSpec(f"{prefix}.norm{k}", (hidden,), "norm_vec", 0.05, s))
        idx[0] += 1
    return out


GEMMA2_LAYER = {"q": (3584, 4096), "k": (3584, 2048), "v": (3584, 2048), "o": (4096, 3584),
                "gate": (3584, 14336), "up": (3584, 14336), "down": (14336, 3584)}
QWEN27_LAYER = {"q": (5120, 6144), "k": (5120, 1024), "v": (5120, 1024), "o": (6144, 5120),
                "gate": (5120, 25600), "up": (5120, 25600), "down": (25600, 5120)}

WORKLOADS = ("tensor_1m", "gemma2_layer", "gemma2_9b", "edge_mix", "qwen_27b_scale")


def workload(name: str, seed: int = 0, layers: int | None = None) -> list:
    """Tensor list of a workload. ``layers`` truncates the multi-layer workloads
    (for bounded samples); None means the full workload."""
    idx = [0]
    if name == "tensor_1m":
        return [TensorSpec("w", (1024, 1024), "normal", 0.02, _seed(seed, 0))]
    if name == "gemma2_layer":
        return _layer("layers.0", GEMMA2_LAYER, 0.01, 0.05, 4, 3584, seed, idx)
    if name == "gemma2_9b":
        n = 42 if layers is None else layers
        out = []
        for L in range(n):
            out += _layer(f"layers.{L}", GEMMA2_LAYER, 0.01, 0.05, 4, 3584, seed, idx)
        if layers is None:
            out.append(TensorSpec("embed", (256000, 3584), "normal", 0.02, _seed(seed, idx[0])))
        return out
    if name == "qwen_27b_scale":
        n = 64 if layers is None else layers
        out = []
        for L in range(n):
            out += _layer(f"layers.{L}", QWEN27_LAYER, 0.005, 0.04, 0, 5120, seed, idx)
        if layers is None:
            out.append(TensorSpec("embed", (152064, 5120), "normal", 0.02, _seed(seed, idx[0])))
        return out
    if name == "edge_mix":
        kinds = [("t3", "t3"), ("outliers", "outliers"), ("zeros", "zeros"), ("ones", "ones"),
                 ("uniform16", "uniform16")]
        out = [TensorSpec(nm, (4096, 4096), d, 0.02, _seed(seed, k)) for k, (nm, d) in enumerate(kinds)]
        out.append(TensorSpec("one", (1,), "normal", 0.02, _seed(seed, 5)))
        out.append(TensorSpec("ragged", (4097,), "normal", 0.02, _seed(seed, 6)))
        out.append(TensorSpec("raw_span", (1024,), "raw", 0.0, _seed(seed, 7)))
        return out
    raise KeyError(name)


def _to_words(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.bfloat16).view(torch.int16)


def generate(spec: TensorSpec, device="cpu") -> torch.Tensor:
    """The tensor's contents. BF16 kinds come back as int16 words (the BF16 bit
    patterns) in ``spec.shape``; raw spans come back as uint8."""
    dev = torch.device(device)
    g = torch.Generator(device=dev).manual_seed(spec.seed)
    n = spec.numel
    if spec.dist == "raw":
        return torch.randint(0, 256, (n,), generator=g, device=dev, dtype=torch.int32).to(torch.uint8)
    if spec.dist == "zeros":
        return torch.zeros(spec.shape, dtype=torch.int16, device=dev)
    if spec.dist == "ones":
        return _to_words(torch.ones(spec.shape, device=dev))
    if spec.dist == "uniform16":
        return torch.randint(-32768, 32768, spec.shape, generator=g, device=dev, dtype=torch.int32).to(torch.int16)
    if spec.dist == "normal":
        return _to_words(torch.randn(spec.shape, generator=g, device=dev) * spec.sigma)
    if spec.dist == "norm_vec":
        return _to_words(1.0 + torch.randn(spec.shape, generator=g, device=dev) * spec.sigma)
    if spec.dist == "t3":
        # Student-t, nu = 3: Z / sqrt(chi2_3 / 3); its variance is 3, so scale by 0.02/sqrt(3)
        z = torch.randn(spec.shape, generator=g, device=dev)
        v = torch.randn((3,) + tuple(spec.shape), generator=g, device=dev).square().sum(0)
        t = z / torch.sqrt(v / 3.0)
        return _to_words(t * (spec.sigma / math.sqrt(3.0)))
    if spec.dist == "outliers":
        x = torch.randn(n, generator=g, device=dev) * spec.sigma
        k = int(round(0.001 * n))
        idx = torch.randperm(n, generator=g, device=dev)[:k]
        x[idx] *= 50.0
        return _to_words(x.view(spec.shape))
    raise KeyError(spec.dist)


def words_numpy(t: torch.Tensor):
    """Host numpy view: uint16 for BF16 words, uint8 for raw spans."""
    import numpy as np
    a = t.detach().cpu().contiguous().numpy()
    return a.view(np.uint16) if a.dtype == np.int16 else a

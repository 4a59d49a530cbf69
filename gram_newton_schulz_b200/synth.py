"""Seeded synthetic inputs shaped like the pages' workloads.

This module only draws random numbers; it holds none of the method's
arithmetic.  Both the CUDA path (tests, bench) and the fp64 oracle consume
the bytes it produces: GPU tests copy sampled matrices back to the host, so
the oracle sees exactly what the kernels saw.

Recipes (one entry per workload):

* ``single-64x256-fp32``: one 64 x 256 fp32 gradient, i.i.d. N(0, 1).
* ``uniform-64x512x2048``: 64 gradients 512 x 2048, noise N(0, 1e-3)
  (variance 1e-3, std ~0.0316) plus a rank-8 component
  (10 * std / sqrt(8)) * U V^T with U, V i.i.d. N(0, 1), so every spike
  entry has std 10 * std; rounded to bf16.
* ``qwen2.5-7b-layer-set-x28``: 28 decoder layers of the Qwen2.5-7B
  projection shapes (q, o 3584 x 3584; k, v 512 x 3584; gate, up
  18944 x 3584; down 3584 x 18944), each drawn like the uniform workload.
  Only the shapes come from that model; no weights are used.
  ``qwen2.5-7b-layer-set-x<L>`` is the same with L layers (profiling).
* ``small-swarm-4096``: 2048 gradients 128 x 512 and 2048 gradients
  256 x 1024, N(0, 1) times a per-matrix scale 10**U(-4, -1), bf16.
* ``large-dense-24``: 16 gradients 8192 x 8192 and 8 of 8192 x 28672,
  noise N(0, 1e-3) plus a rank-32 spike as above, bf16.

Weights are N(0, 0.02^2) in the gradient dtype; momentum starts at zero.
Every matrix i of workload w is drawn from its own generator seeded with
``seed_w * 2**20 + i`` (weights: ``+ 2**19``), so any subset of matrices can
be regenerated on its own.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional, Sequence, Tuple

import torch

QWEN7B_LAYER: Tuple[Tuple[str, int, int], ...] = (
    ("q", 3584, 3584),
    ("k", 512, 3584),
    ("v", 512, 3584),
    ("o", 3584, 3584),
    ("gate", 18944, 3584),
    ("up", 18944, 3584),
    ("down", 3584, 18944),
)


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    dtype: str                      # "bf16" or "f32"
    shapes: Tuple[Tuple[int, int], ...]
    dist: str                       # "normal" | "spiked" | "logscaled"
    var: float = 1.0
    rank: int = 0
    beta: float = 0.95
    lr: float = 0.02
    labels: Tuple[str, ...] = field(default=())

    @property
    def count(self) -> int:
        return len(self.shapes)

    def elements(self) -> int:
        return sum(r * c for r, c in self.shapes)


def _qwen_shapes(layers: int):
    shapes, labels = [], []
    for layer in range(layers):
        for tag, r, c in QWEN7B_LAYER:
            shapes.append((r, c))
            labels.append(f"L{layer}.{tag}")
    return tuple(shapes), tuple(labels)


def workload(name: str) -> Workload:
    if name == "single-64x256-fp32":
        return Workload(name, 1, "f32", ((64, 256),), "normal", 1.0)
    if name == "uniform-64x512x2048":
        return Workload(name, 2, "bf16", ((512, 2048),) * 64, "spiked", 1e-3, 8)
    if name == "qwen2.5-7b-layer-set-x28":
        s, l = _qwen_shapes(28)
        return Workload(name, 3, "bf16", s, "spiked", 1e-3, 8, labels=l)
    if name.startswith("qwen2.5-7b-layer-set-x") and name != "qwen2.5-7b-layer-set-x28":
        layers = int(name.rsplit("x", 1)[1])
        s, l = _qwen_shapes(layers)
        return Workload(name, 3, "bf16", s, "spiked", 1e-3, 8, labels=l)
    if name == "small-swarm-4096":
        return Workload(name, 4, "bf16", ((128, 512),) * 2048 + ((256, 1024),) * 2048,
                        "logscaled", 1.0)
    if name == "large-dense-24":
        return Workload(name, 5, "bf16", ((8192, 8192),) * 16 + ((8192, 28672),) * 8,
                        "spiked", 1e-3, 32)
    raise KeyError(name)


WORKLOADS = (
    "single-64x256-fp32",
    "uniform-64x512x2048",
    "qwen2.5-7b-layer-set-x28",
    "small-swarm-4096",
    "large-dense-24",
)


def custom(name: str, shapes: Sequence[Tuple[int, int]], *, seed: int, dtype: str = "bf16",
           dist: str = "spiked", var: float = 1e-3, rank: int = 8) -> Workload:
    """A workload with caller-chosen shapes, drawn with one of the recipes."""
    return Workload(name, seed, dtype, tuple((int(r), int(c)) for r, c in shapes), dist, var, rank)


def _torch_dtype(dtype: str):
    return {"bf16": torch.bfloat16, "f32": torch.float32}[dtype]


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def gradient(w: Workload, i: int, device="cpu") -> torch.Tensor:
    """Gradient i of workload ``w`` in the workload dtype, on ``device``."""
    rows, cols = w.shapes[i]
    g = _gen(device, w.seed * 2**20 + i)
    x = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
    if w.dist == "normal":
        x.mul_(math.sqrt(w.var))
    elif w.dist == "spiked":
        std = math.sqrt(w.var)
        x.mul_(std)
        u = torch.randn(rows, w.rank, generator=g, device=device, dtype=torch.float32)
        v = torch.randn(cols, w.rank, generator=g, device=device, dtype=torch.float32)
        x.addmm_(u, v.t(), alpha=10.0 * std / math.sqrt(w.rank))
    elif w.dist == "logscaled":
        e = torch.rand(1, generator=g, device=device, dtype=torch.float64).item()
        x.mul_(10.0 ** (-4.0 + 3.0 * e))
    else:
        raise ValueError(w.dist)
    return x.to(_torch_dtype(w.dtype))


def weight(w: Workload, i: int, device="cpu") -> torch.Tensor:
    rows, cols = w.shapes[i]
    g = _gen(device, w.seed * 2**20 + 2**19 + i)
    x = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32).mul_(0.02)
    return x.to(_torch_dtype(w.dtype))


def gradients(w: Workload, device="cpu", indices: Optional[Sequence[int]] = None) -> List[torch.Tensor]:
    idx = range(w.count) if indices is None else indices
    return [gradient(w, i, device) for i in idx]


def weights(w: Workload, device="cpu", indices: Optional[Sequence[int]] = None) -> List[torch.Tensor]:
    idx = range(w.count) if indices is None else indices
    return [weight(w, i, device) for i in idx]


def sample_indices(w: Workload, seed: int = 0) -> List[int]:
    """First, last and one seeded random matrix of every shape bucket."""
    by_shape = {}
    for i, s in enumerate(w.shapes):
        by_shape.setdefault(s, []).append(i)
    rnd = _gen("cpu", 7919 + seed)
    out = []
    for s in sorted(by_shape):
        ids = by_shape[s]
        pick = {ids[0], ids[-1], ids[int(torch.randint(len(ids), (1,), generator=rnd).item())]}
        out.extend(sorted(pick))
    return sorted(out)

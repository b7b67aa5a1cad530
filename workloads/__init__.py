"""Seeded synthetic inputs for the Muon / NorMuon step.

This module is shared by the CUDA path's tests and bench and by the fp64
oracle.  It holds shapes, hyperparameters and seeded random draws only; it
computes nothing of the optimizer itself (no momentum, no normalization, no
Newton-Schulz, no update scale).

Workloads follow the shapes the source pages discuss:

* ``single_256``: one 256x256 fp32 gradient, as in the kernel-isolation
  experiment of the DeepSpeed issue "Muon under AutoTP orthogonalizes each
  shard" (section "Measurement"), one Muon step.
* ``conv_megabatch``: sixteen stacked Conv2d weights [16, 64, 64, 3, 3], the
  megabatch geometry of the dion PR "Fix convolution flattening in megabatches
  and NorMuon normalization" (section "Problem and fix"), flattened to
  [16, 64, 576]; NorMuon.
* ``per_head``: a 4096x4096 q_proj split into 32 heads of 128 rows (the
  per-head option of the DeepSpeed issue, section "What could be done"),
  plus a 512x1024 and a 1024x512 matrix (the shape of that issue's
  follow-up table), three consecutive steps, plain Muon.
* ``llama8b``: a Llama-8B-shaped model, 32 layers of q, k, v, o, gate, up,
  down; bf16 gradients and momentum, fp32 master weights with a bf16 copy;
  NorMuon.
* ``moe``: 64 experts with w1 [2048, 7168] and w2 [7168, 2048]; per-expert
  gradient scale log-uniform in [1e-2, 1]; Gram Newton-Schulz; NorMuon; two
  consecutive steps.

Seeds: gradient ``i`` of step ``t`` of workload number ``k`` is drawn from a
generator seeded with ``1000*k + 100*t + i``; the initial weights of matrix
``i`` from ``1000*k + 90 + i`` (the 256x256 case draws its weights as the
second draw of the same generator as its gradient, seed 0).
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence, Tuple

import torch

QUINTIC = (3.4445, -4.7750, 2.0315)


@dataclasses.dataclass(frozen=True)
class Group:
    """A batch of same-shape parameter slices.

    ``param_shape`` is the shape of ONE parameter as the model holds it (for
    a convolution [out, in, kh, kw]); the optimizer sees it flattened to
    [out, prod(rest)].  ``heads`` > 1 splits each parameter along dim 0 into
    that many head blocks, and each block is one Newton-Schulz slice.
    """

    name: str
    param_shape: Tuple[int, ...]
    count: int                      # parameters in the group
    heads: int = 1
    first_index: int = 0            # matrix index of the first parameter (seeding)

    @property
    def rows(self) -> int:
        return self.param_shape[0]

    @property
    def cols(self) -> int:
        return int(math.prod(self.param_shape[1:]))

    @property
    def slice_rows(self) -> int:
        return self.rows // self.heads

    @property
    def slices(self) -> int:
        return self.count * self.heads


@dataclasses.dataclass(frozen=True)
class Workload:
    key: str
    number: int
    groups: Tuple[Group, ...]
    grad_dtype: torch.dtype
    mom_dtype: torch.dtype
    weight_dtype: torch.dtype
    weight_copy_bf16: bool
    steps: int
    grad_std: float
    weight_std: float
    lr: float
    weight_decay: float
    momentum: float = 0.95
    nesterov: bool = True
    ns_eps: float = 1e-7
    ns_steps: int = 5
    normuon: bool = False
    beta2: float = 0.95
    nor_eps: float = 1e-8
    variants: Tuple[str, ...] = ("standard",)
    expert_scale_seed: Optional[int] = None   # per-parameter log-uniform grad scale
    expert_scale_range: Tuple[float, float] = (1e-2, 1.0)

    @property
    def slices(self) -> int:
        return sum(g.slices for g in self.groups)

    @property
    def elements(self) -> int:
        return sum(g.count * g.rows * g.cols for g in self.groups)


def _llama_groups(layers: int = 32) -> Tuple[Group, ...]:
    specs = [("q_proj", (4096, 4096)), ("k_proj", (1024, 4096)), ("v_proj", (1024, 4096)),
             ("o_proj", (4096, 4096)), ("gate_proj", (14336, 4096)), ("up_proj", (14336, 4096)),
             ("down_proj", (4096, 14336))]
    out = []
    idx = 0
    for name, shp in specs:
        out.append(Group(name, shp, layers, 1, idx))
        idx += layers
    return tuple(out)


WORKLOADS = {
    "single_256": Workload(
        key="single_256", number=1,
        groups=(Group("w", (256, 256), 1),),
        grad_dtype=torch.float32, mom_dtype=torch.float32, weight_dtype=torch.float32,
        weight_copy_bf16=False, steps=1, grad_std=1.0, weight_std=0.02,
        lr=0.05, weight_decay=0.0, normuon=False, variants=("standard", "gram")),
    "conv_megabatch": Workload(
        key="conv_megabatch", number=2,
        groups=(Group("conv", (64, 64, 3, 3), 16),),
        grad_dtype=torch.bfloat16, mom_dtype=torch.bfloat16, weight_dtype=torch.bfloat16,
        weight_copy_bf16=False, steps=1, grad_std=1.0, weight_std=0.02,
        lr=0.02, weight_decay=0.01, normuon=True, variants=("standard", "gram")),
    "per_head": Workload(
        key="per_head", number=3,
        groups=(Group("q_proj_heads", (4096, 4096), 1, heads=32, first_index=0),
                Group("w512x1024", (512, 1024), 1, first_index=1),
                Group("w1024x512", (1024, 512), 1, first_index=2)),
        grad_dtype=torch.bfloat16, mom_dtype=torch.bfloat16, weight_dtype=torch.bfloat16,
        weight_copy_bf16=False, steps=3, grad_std=1.0, weight_std=0.02,
        lr=0.02, weight_decay=0.0, normuon=False, variants=("standard", "gram")),
    "llama8b": Workload(
        key="llama8b", number=4,
        groups=_llama_groups(32),
        grad_dtype=torch.bfloat16, mom_dtype=torch.bfloat16, weight_dtype=torch.float32,
        weight_copy_bf16=True, steps=1, grad_std=1e-3, weight_std=0.02,
        lr=0.02, weight_decay=0.0, normuon=True, variants=("standard", "gram")),
    "moe": Workload(
        key="moe", number=5,
        groups=(Group("w1", (2048, 7168), 64, 1, 0), Group("w2", (7168, 2048), 64, 1, 64)),
        grad_dtype=torch.bfloat16, mom_dtype=torch.bfloat16, weight_dtype=torch.bfloat16,
        weight_copy_bf16=False, steps=2, grad_std=1e-3, weight_std=0.02,
        lr=0.02, weight_decay=0.0, normuon=True, variants=("gram",),
        expert_scale_seed=5000),
}


def grad_seed(w: Workload, step: int, index: int) -> int:
    return 1000 * w.number + 100 * step + index


def weight_seed(w: Workload, index: int) -> int:
    return 1000 * w.number + 90 + index


def expert_scales(w: Workload) -> Optional[torch.Tensor]:
    """Per-parameter gradient scale 10**U(log10 lo, log10 hi), one per expert.

    Experts are numbered by parameter index modulo the expert count of the
    first group, so w1 and w2 of the same expert share a scale.
    """
    if w.expert_scale_seed is None:
        return None
    n_exp = w.groups[0].count
    g = torch.Generator().manual_seed(w.expert_scale_seed)
    lo, hi = (math.log10(v) for v in w.expert_scale_range)
    u = torch.rand(n_exp, generator=g, dtype=torch.float64)
    return torch.pow(10.0, lo + (hi - lo) * u)


def _randn(shape: Sequence[int], seed: int, device: str) -> torch.Tensor:
    g = torch.Generator(device=device).manual_seed(seed)
    return torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)


def gradient(w: Workload, group: Group, param: int, step: int, device: str = "cpu") -> torch.Tensor:
    """Gradient of parameter ``param`` of ``group`` at ``step`` (param_shape, grad dtype)."""
    idx = group.first_index + param
    if w.key == "single_256":
        x = _randn(group.param_shape, 0, device)        # first draw of generator(0)
    else:
        x = _randn(group.param_shape, grad_seed(w, step, idx), device)
    x = x * w.grad_std
    sc = expert_scales(w)
    if sc is not None:
        x = x * float(sc[param % sc.numel()])
    return x.to(w.grad_dtype)


def initial_weight(w: Workload, group: Group, param: int, device: str = "cpu") -> torch.Tensor:
    idx = group.first_index + param
    if w.key == "single_256":
        g = torch.Generator(device=device).manual_seed(0)
        torch.randn(group.param_shape, generator=g, device=device)       # first draw: the gradient
        x = torch.randn(group.param_shape, generator=g, device=device, dtype=torch.float32)
    else:
        x = _randn(group.param_shape, weight_seed(w, idx), device)
    return (x * w.weight_std).to(w.weight_dtype)


def scaled(w: Workload, factor: int) -> Workload:
    """The same workload with every parameter count divided by ``factor`` (>=1)."""
    gs = tuple(dataclasses.replace(g, count=max(1, g.count // factor)) for g in w.groups)
    return dataclasses.replace(w, groups=gs)


def small_shapes() -> List[Tuple[int, int]]:
    """Ragged shapes used by parity tests: several tiles plus ragged tails."""
    return [(64, 576), (200, 300), (300, 200), (256, 256), (384, 520), (130, 1000)]

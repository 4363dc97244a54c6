"""Seeded synthetic inputs for the QLoRA NF4 linear layer.

This module holds no arithmetic of the method: it only draws random tensors
with fixed seeds and the shapes and value distributions of the workloads, so
that the CUDA path and the CPU oracle can be fed the same bytes.  Every draw
is made in fp32 from a ``torch.Generator`` and rounded to bf16 by torch
(round to nearest even).

Seeds follow ``seed = 1000 * workload + 10 * tensor_index + role`` with roles
W=0, X=1, A=2, B=3, dY=4, outlier mask=5, mixture choice=6, t(4) draw=7.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

ROLE_W, ROLE_X, ROLE_A, ROLE_B, ROLE_DY, ROLE_OUTLIER, ROLE_MIX, ROLE_T4 = range(8)


def seed_of(workload: int, tensor_index: int, role: int) -> int:
    return 1000 * workload + 10 * tensor_index + role


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal(seed: int, shape, std: float, device="cpu") -> torch.Tensor:
    """bf16 tensor ~ N(0, std^2)."""
    t = torch.randn(shape, generator=_gen(seed, device), device=device, dtype=torch.float32)
    return (t * std).to(torch.bfloat16)


def uniform(seed: int, shape, bound: float, device="cpu") -> torch.Tensor:
    """bf16 tensor ~ U(-bound, bound)."""
    t = torch.rand(shape, generator=_gen(seed, device), device=device, dtype=torch.float32)
    return ((t * 2.0 - 1.0) * bound).to(torch.bfloat16)


def weight(workload: int, idx: int, N: int, K: int, std: float, outlier_frac: float = 0.0,
           outlier_mult: float = 10.0, t4_mix: float = 0.0, device="cpu") -> torch.Tensor:
    """Frozen base weight W [N, K] in bf16.

    * ``outlier_frac``: that fraction of entries (a seeded uniform choice) is
      multiplied by ``outlier_mult``.
    * ``t4_mix``: with that probability an entry is drawn from a Student t(4)
      scaled by std / sqrt(2) (so both components have variance std^2)
      instead of N(0, std^2).
    """
    w = torch.randn((N, K), generator=_gen(seed_of(workload, idx, ROLE_W), device), device=device,
                    dtype=torch.float32) * std
    if t4_mix > 0.0:
        g = _gen(seed_of(workload, idx, ROLE_T4), device)
        z = torch.randn((N, K), generator=g, device=device, dtype=torch.float32)
        chi = torch.randn((4, N, K), generator=g, device=device, dtype=torch.float32).square_().sum(0)
        t4 = z / torch.sqrt(chi / 4.0)
        del chi, z
        pick = torch.rand((N, K), generator=_gen(seed_of(workload, idx, ROLE_MIX), device), device=device) < t4_mix
        w = torch.where(pick, t4 * (std / math.sqrt(2.0)), w)
        del t4, pick
    if outlier_frac > 0.0:
        sel = torch.rand((N, K), generator=_gen(seed_of(workload, idx, ROLE_OUTLIER), device),
                         device=device) < outlier_frac
        w = torch.where(sel, w * outlier_mult, w)
    return w.to(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw bf16 bit patterns of a tensor as a numpy uint16 array (CPU copy)."""
    assert t.dtype == torch.bfloat16
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact fp64 values of a bf16 tensor."""
    return t.detach().cpu().to(torch.float64).numpy()


# --------------------------------------------------------------------------
# the five workloads
# --------------------------------------------------------------------------
@dataclass
class Projection:
    name: str
    N: int          # out features
    K: int          # in features


@dataclass
class Workload:
    index: int
    name: str
    projections: list
    Ms: list
    r: int
    alpha: float
    w_std: float
    backward: bool
    outlier_frac: float = 0.0
    t4_mix: float = 0.0
    repeat: int = 1          # how many copies of the projection set (bulk workload)
    notes: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def scaling(self) -> float:
        return self.alpha / self.r


LLAMA7B = [Projection("q_proj", 4096, 4096), Projection("k_proj", 4096, 4096),
           Projection("v_proj", 4096, 4096), Projection("o_proj", 4096, 4096),
           Projection("gate_proj", 11008, 4096), Projection("up_proj", 11008, 4096),
           Projection("down_proj", 4096, 11008)]

WORKLOADS = {
    1: Workload(1, "single-linear-4096x4096-M16", [Projection("linear", 4096, 4096)], [16], 16, 32.0, 0.02, True),
    2: Workload(2, "decode-gemv-llama7b-mlp", [Projection("up_proj", 11008, 4096), Projection("down_proj", 4096, 11008)],
                [1, 4, 8, 32], 16, 32.0, 0.02, False),
    3: Workload(3, "llama7b-block-train-M2048", LLAMA7B, [2048], 16, 32.0, 0.02, True, outlier_frac=0.001),
    4: Workload(4, "llama70b-projections", [Projection("o_proj", 8192, 8192), Projection("up_proj", 28672, 8192),
                                          Projection("down_proj", 8192, 28672)],
                [1, 512, 4096], 64, 16.0, 0.015, True),
    5: Workload(5, "bulk-quantize-llama7b-32-layers", LLAMA7B, [], 16, 32.0, 0.02, False, t4_mix=0.1, repeat=32),
}


def layer_inputs(wl: Workload, proj_index: int, M: int, device="cpu", with_dy: bool = True):
    """X, A, B (and dY) for one projection of a workload."""
    p = wl.projections[proj_index]
    X = normal(seed_of(wl.index, proj_index, ROLE_X) + 100 * M, (M, p.K), 1.0, device)
    A = uniform(seed_of(wl.index, proj_index, ROLE_A), (wl.r, p.K), 1.0 / math.sqrt(p.K), device)
    B = normal(seed_of(wl.index, proj_index, ROLE_B), (p.N, wl.r), 0.01, device)
    dY = normal(seed_of(wl.index, proj_index, ROLE_DY) + 100 * M, (M, p.N), 1.0, device) if with_dy else None
    return X, A, B, dY


def layer_weight(wl: Workload, proj_index: int, device="cpu", copy: int = 0) -> torch.Tensor:
    p = wl.projections[proj_index]
    return weight(wl.index, proj_index + 7 * copy, p.N, p.K, wl.w_std, wl.outlier_frac, 10.0, wl.t4_mix,
                  device)

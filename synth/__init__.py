"""Seeded synthetic inputs for the 2:4-sparse + low-rank linear layer.

This module only draws random numbers and rounds them to bf16; it holds none
of the layer's arithmetic, so both the CPU oracle checks and the CUDA path may
use it.  Everything is returned as numpy ``uint16`` bf16 bit patterns.

Recipe (the workloads of the five benchmark configurations):

* Gaussian draws in fp32 from numpy's PCG64 generator, one generator per
  tensor, seeded with ``1000*cfg + 10*sub + tensor_id`` where ``tensor_id`` is
  X=1, W=2, U=3, V=4, outlier-permutation=5.  ``sub`` numbers the layers
  inside a configuration (0 when there is only one); W and X use the number
  of the layer *shape* instead, so the rank variants of one shape share them.
* Scale by the stated standard deviation, then round to bf16
  (round-to-nearest-even).  W is projected to 2:4 only after this rounding.
* Outlier channels: ``round(0.01 * d_in)`` columns of X, chosen by a seeded
  permutation, are multiplied by 20 before rounding.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

TENSOR_X, TENSOR_W, TENSOR_U, TENSOR_V, TENSOR_OUTLIER = 1, 2, 3, 4, 5


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return the bits.

    Inputs must be finite (the generators never produce NaN or Inf).
    """
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def seed_for(cfg: int, tensor_id: int, sub: int = 0) -> int:
    return 1000 * cfg + 10 * sub + tensor_id


def gaussian_bf16(shape, std: float, seed: int) -> np.ndarray:
    g = np.random.Generator(np.random.PCG64(seed))
    a = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return f32_to_bf16_bits(a)


def activations_bf16(M: int, d_in: int, seed: int, outlier_seed: int | None) -> np.ndarray:
    """X ~ N(0, 1); with ``outlier_seed`` set, 1% of the channels scaled by 20."""
    g = np.random.Generator(np.random.PCG64(seed))
    a = g.standard_normal(size=(M, d_in), dtype=np.float32)
    if outlier_seed is not None:
        k = int(round(0.01 * d_in))
        cols = np.random.Generator(np.random.PCG64(outlier_seed)).permutation(d_in)[:k]
        a[:, cols] *= np.float32(20.0)
    return f32_to_bf16_bits(a)


@dataclass(frozen=True)
class Layer:
    """One decomposed linear layer: dense W (d_out x d_in) and rank-r factors."""
    name: str
    d_out: int
    d_in: int
    r: int
    cfg: int
    sub: int = 0
    shape_sub: int | None = None   # seeds of W and X; defaults to sub
    x_outliers: bool = False
    w_std: float = 0.02
    # "lowrank" selects the factor distributions:
    #   "v_unit"  : U ~ N(0, 0.02^2/r), V ~ N(0, 1/r)        (the tiny configuration)
    #   "both_small": U, V ~ N(0, 0.02^2/r)                   (the decode/70B configurations)
    lowrank: str = "v_unit"

    def u_std(self) -> float:
        return 0.02 / math.sqrt(self.r) if self.r else 0.0

    def v_std(self) -> float:
        if self.r == 0:
            return 0.0
        return 1.0 / math.sqrt(self.r) if self.lowrank == "v_unit" else 0.02 / math.sqrt(self.r)

    @property
    def wsub(self) -> int:
        return self.sub if self.shape_sub is None else self.shape_sub

    def weight(self) -> np.ndarray:
        return gaussian_bf16((self.d_out, self.d_in), self.w_std, seed_for(self.cfg, TENSOR_W, self.wsub))

    def factors(self) -> tuple[np.ndarray, np.ndarray]:
        U = gaussian_bf16((self.d_out, self.r), self.u_std(), seed_for(self.cfg, TENSOR_U, self.sub))
        V = gaussian_bf16((self.r, self.d_in), self.v_std(), seed_for(self.cfg, TENSOR_V, self.sub))
        return U, V

    def activations(self, M: int) -> np.ndarray:
        out = seed_for(self.cfg, TENSOR_OUTLIER, self.wsub) if self.x_outliers else None
        return activations_bf16(M, self.d_in, seed_for(self.cfg, TENSOR_X, self.wsub), out)


@dataclass(frozen=True)
class Config:
    cfg: int
    title: str
    layers: tuple
    Ms: tuple = field(default_factory=tuple)


def _cfg4_layers():
    shapes = [("q_proj", 4096, 4096), ("k_proj", 1024, 4096), ("v_proj", 1024, 4096),
              ("o_proj", 4096, 4096), ("gate_proj", 14336, 4096), ("up_proj", 14336, 4096),
              ("down_proj", 4096, 14336)]
    return tuple(Layer(n, do, di, 64, cfg=4, sub=i) for i, (n, do, di) in enumerate(shapes))


def _cfg5_layers():
    out = []
    sub = 0
    for shape, (name, do, di) in enumerate((("up_proj_70b", 28672, 8192), ("down_proj_70b", 8192, 28672))):
        for r in (64, 128, 256):
            out.append(Layer(f"{name}_r{r}", do, di, r, cfg=5, sub=sub, shape_sub=shape, x_outliers=True,
                             lowrank="both_small"))
            sub += 1
    return tuple(out)


CONFIGS = {
    1: Config(1, "tiny decomposed linear 256x256, r=8, M=8",
              (Layer("tiny", 256, 256, 8, cfg=1),), (8,)),
    2: Config(2, "Llama-3-8B q_proj decode 4096x4096, r=64, M in {1,4,16}",
              (Layer("q_proj", 4096, 4096, 64, cfg=2, x_outliers=True, lowrank="both_small"),),
              (1, 4, 16)),
    3: Config(3, "Llama-3-8B gate/up prefill 14336x4096, r=64, M=2048",
              (Layer("gate_up", 14336, 4096, 64, cfg=3),), (2048,)),
    4: Config(4, "Llama-3-8B block linear set (7 layers), r=64, M=4096",
              _cfg4_layers(), (4096,)),
    5: Config(5, "70B MLP up/down 28672x8192 / 8192x28672, r in {64,128,256}, M sweep",
              _cfg5_layers(), (1, 16, 128, 1024, 8192)),
}

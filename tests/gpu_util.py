"""Helpers for the GPU parity tests: device transfer of bf16 bit patterns,
seeded sampling of (token, output) pairs, and the acceptance check against
the fp64 oracle."""
from __future__ import annotations

import functools

import numpy as np
import torch

import oracle
import synth

REL_FRO_TOL = 5e-3       # relative Frobenius error bound
ELEM_REL_TOL = 1e-2      # per-element bound: |err| <= 1e-2 * (|X||W'|^T) + 1e-3
ELEM_ABS_TOL = 1e-3


def to_dev(bits: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns -> CUDA bf16 tensor (bit copy)."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def to_dev_u8(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def from_dev(t: torch.Tensor) -> np.ndarray:
    """CUDA bf16 tensor -> uint16 bit patterns."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bits_to_f64(b: np.ndarray) -> np.ndarray:
    return synth.bf16_bits_to_f32(b).astype(np.float64)


def sample_indices(n: int, k: int, seed: int, tile: int = 128) -> np.ndarray:
    """All of range(n) when n <= k; otherwise k seeded indices that always
    include both ends and the first/last rows of the final (ragged) tile."""
    if n <= k:
        return np.arange(n, dtype=np.int64)
    rng = np.random.Generator(np.random.PCG64(seed))
    fixed = {0, 1, n - 1, n - 2, (n - 1) // tile * tile, min(n - 1, tile), tile - 1 if tile < n else 0}
    rest = rng.choice(n, size=k, replace=False)
    out = sorted(fixed | set(int(x) for x in rest))
    return np.array(out[:max(k, len(fixed))], dtype=np.int64)


def check_forward(Y_bits: np.ndarray, Y_ref: np.ndarray, B_ref: np.ndarray, what: str):
    """The acceptance test on the sampled block: relative Frobenius error and
    the per-element bound, both in fp64 on the bf16 GPU output."""
    Y = bits_to_f64(Y_bits)
    assert np.all(np.isfinite(Y)), f"{what}: non-finite output"
    diff = Y - Y_ref
    denom = np.linalg.norm(Y_ref)
    rel = np.linalg.norm(diff) / denom if denom > 0 else np.linalg.norm(diff)
    assert rel <= REL_FRO_TOL, f"{what}: relative Frobenius error {rel:.3e}"
    bound = ELEM_REL_TOL * B_ref + ELEM_ABS_TOL
    bad = np.abs(diff) > bound
    if bad.any():
        i, j = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} elements out of bound; first at {i},{j}: "
                             f"gpu {Y[i, j]:.6g} ref {Y_ref[i, j]:.6g} bound {bound[i, j]:.3g}")
    return rel


@functools.lru_cache(maxsize=2)
def layer_weights(cfg: int, name: str):
    """(W, vals, meta, U, V) of a configuration layer; vals/meta from the oracle."""
    layer = next(l for l in synth.CONFIGS[cfg].layers if l.name == name)
    W = layer.weight()
    vals, meta = oracle.pack_2to4(W)
    U, V = layer.factors()
    return layer, W, vals, meta, U, V


@functools.lru_cache(maxsize=2)
def layer_activations(cfg: int, name: str, M: int):
    layer = next(l for l in synth.CONFIGS[cfg].layers if l.name == name)
    return layer.activations(M)

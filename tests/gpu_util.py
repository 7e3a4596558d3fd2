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
    """All of range(n) when n <= k; otherwise the sorted union of fixed indices
    (both ends, the first and last rows of the first and of the final, ragged
    tile) and k seeded draws spread over the whole range, so the sample holds
    at least k indices and always reaches the top of the range."""
    if n <= k:
        return np.arange(n, dtype=np.int64)
    rng = np.random.Generator(np.random.PCG64(seed))
    last_tile = (n - 1) // tile * tile
    fixed = {0, 1, n - 2, n - 1, last_tile, max(0, last_tile - 1), min(n - 1, tile - 1), min(n - 1, tile)}
    rest = rng.choice(n, size=k, replace=False)
    return np.array(sorted(fixed | set(int(x) for x in rest)), dtype=np.int64)


def stratified_indices(n: int, block: int, seed: int) -> np.ndarray:
    """One seeded index inside every aligned block of ``block`` indices (the
    last, ragged block included), plus n - 1: a sample that meets every
    16-token unit or 128-row tile a kernel's work partition can produce."""
    rng = np.random.Generator(np.random.PCG64(seed))
    starts = np.arange(0, n, block, dtype=np.int64)
    widths = np.minimum(block, n - starts)
    picks = starts + (rng.random(starts.shape[0]) * widths).astype(np.int64)
    return np.unique(np.concatenate([picks, [n - 1]]))


def check_forward(Y_bits: np.ndarray, Y_ref: np.ndarray, B_ref: np.ndarray, what: str,
                  rows=None, outs=None):
    """The acceptance test on the sampled block: relative Frobenius error and
    the per-element bound, both in fp64 on the bf16 GPU output.  ``rows`` and
    ``outs`` (the token and output indices of the block) name the failing
    cell in the message."""
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
        tok = int(rows[i]) if rows is not None else int(i)
        out = int(outs[j]) if outs is not None else int(j)
        raise AssertionError(f"{what}: {bad.sum()} elements out of bound; first at token {tok}, output {out}: "
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

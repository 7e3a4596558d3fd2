"""Data-free alternating minimisation for W ~ S + L (2:4 sparse S, rank-r L).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py): used by the tests, the
smoke check and the benchmark's CPU-baseline leg, never by the product path.

What it computes, from the pages (fp64 throughout, numpy for the SVD):

* C_r(Z): the rank-r truncation of Z from its top r singular triplets
  (HASSLE-free, section 3, notation; by the Eckart-Young theorem the best
  approximation of rank at most r in the Frobenius norm).
* P1, data-free (identity Hessian): with L fixed, the best 2:4 matrix S for
  ||W - L - S||_F is the hard-thresholding of W - L (HASSLE-free, section
  4.1.1): in every aligned group of four along d_in keep the two entries of
  largest magnitude, values unchanged.  Ties go to the lower index (the
  reading taken for the 2:4 projection everywhere in this repository).
* P2, data-free: with S fixed, the best L of rank at most r is C_r(W - S)
  (HASSLE-free, section 4.2.1).
* Initialisation as in LoSparse, section 3.2: the low-rank part starts from
  the top-r singular components of the pretrained weight, L0 = C_r(W), then
  S0 = P1(W - L0).
* The alternation (HASSLE-free, section 4): each iteration solves P2 then P1
  with the other block fixed.  Both steps are exact block minimisers, so the
  objective ||W - S - L||_F never increases.

``objective`` is recorded after the initialisation and after every iteration.
"""
from __future__ import annotations

import numpy as np


def truncated_svd(Z: np.ndarray, r: int) -> np.ndarray:
    """C_r(Z) in fp64 from numpy's SVD (a library primitive)."""
    if r <= 0:
        return np.zeros_like(Z, dtype=np.float64)
    Uz, sz, Vz = np.linalg.svd(np.asarray(Z, dtype=np.float64), full_matrices=False)
    r = min(r, sz.shape[0])
    return (Uz[:, :r] * sz[:r]) @ Vz[:r, :]


def hard_threshold_2to4(R: np.ndarray) -> np.ndarray:
    """P1 for an identity Hessian: keep the two largest |R| of each aligned
    group of four along the last axis (ties to the lower index), zero the rest."""
    R = np.asarray(R, dtype=np.float64)
    return np.where(keep_mask_2to4(R), R, 0.0)


def keep_mask_2to4(R: np.ndarray) -> np.ndarray:
    """The positions P1 keeps (boolean, the shape of R): in every aligned group
    of four along the last axis, the two of largest |R|, ties to the lower
    index."""
    R = np.asarray(R, dtype=np.float64)
    d_out, d_in = R.shape
    if d_in % 4:
        raise ValueError("d_in must be a multiple of 4")
    g = np.abs(R).reshape(d_out, d_in // 4, 4)
    # rank of position p = number of q that beat it (larger, or equal and q < p)
    beaten = np.zeros(g.shape, dtype=np.int64)
    for p in range(4):
        for q in range(4):
            if q == p:
                continue
            beats = g[..., q] > g[..., p]
            if q < p:
                beats |= g[..., q] == g[..., p]
            beaten[..., p] += beats
    return (beaten < 2).reshape(d_out, d_in)


def objective(W: np.ndarray, S: np.ndarray, L: np.ndarray) -> float:
    return float(np.linalg.norm(np.asarray(W, dtype=np.float64) - S - L))


def alternating_minimisation(W: np.ndarray, r: int, iters: int):
    """Returns (S, L, objectives) with objectives[0] after the initialisation
    and objectives[t] after iteration t (t = 1 .. iters)."""
    Wf = np.asarray(W, dtype=np.float64)
    L = truncated_svd(Wf, r)
    S = hard_threshold_2to4(Wf - L)
    objs = [objective(Wf, S, L)]
    for _ in range(iters):
        L = truncated_svd(Wf - S, r)
        S = hard_threshold_2to4(Wf - L)
        objs.append(objective(Wf, S, L))
    return S, L, objs

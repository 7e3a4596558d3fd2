"""Backward of the layer with respect to its low-rank factors (S frozen).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py): used by the tests, the
smoke check and the benchmark's CPU-baseline leg, never by the product path.

The layer computes Y = X S^T + (X V^T) U^T (LoSparse, section 3.2, in the
d_out x d_in convention of this repository); its low-rank factors are what
LoRA fine-tuning trains (3BASiL summary page: the low-rank components
initialise LoRA, S stays fixed).  For an upstream gradient dY = dL/dY
(M x d_out), the chain rule on Y = T U^T with T = X V^T gives

    dU = dY^T T          (d_out x r)
    dV = (dY U)^T X      (r x d_in)

evaluated here in fp64 from the bf16 inputs, with the element-wise bounds
B_dU = |dY|^T (|X| |V|^T) and B_dV = (|dY| |U|)^T |X| used by the
acceptance test.
"""
from __future__ import annotations

import numpy as np


def _f64(bits) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def lora_backward(X, dY, U, V):
    """(dU, dV, B_dU, B_dV) in fp64 from bf16 bit patterns X [M, d_in],
    dY [M, d_out], U [d_out, r], V [r, d_in]."""
    Xf, dYf, Uf, Vf = _f64(X), _f64(dY), _f64(U), _f64(V)
    T = Xf @ Vf.T
    G = dYf @ Uf
    dU = dYf.T @ T
    dV = G.T @ Xf
    B_dU = np.abs(dYf).T @ (np.abs(Xf) @ np.abs(Vf).T)
    B_dV = (np.abs(dYf) @ np.abs(Uf)).T @ np.abs(Xf)
    return dU, dV, B_dU, B_dV

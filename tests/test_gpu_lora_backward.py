"""GPU parity of the backward with respect to U and V (S frozen) against the
fp64 oracle (oracle/lora_backward.py): dU = dY^T (X V^T), dV = (dY U)^T X.
Acceptance: relative Frobenius error <= 5e-3 and |err| <= 1e-2 B + 1e-6 max(B)
per element (B the element-wise bound of the oracle), at full size on the
gate/up shape and on ragged shapes, every rank tile (64, 128, 256), with T
given by the caller or recomputed."""
import numpy as np
import pytest
import torch

import oracle.lora_backward as lb
import synth
from gpu_util import to_dev

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sparse_rank_linear_02_b200 as slr


def _check(got: torch.Tensor, ref: np.ndarray, bound: np.ndarray, what: str):
    g = got.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(g)), f"{what}: non-finite"
    diff = g - ref
    rel = np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300)
    assert rel <= 5e-3, f"{what}: relative Frobenius error {rel:.3e}"
    tol = 1e-2 * bound + 1e-6 * bound.max()
    bad = np.abs(diff) > tol
    assert not bad.any(), f"{what}: {bad.sum()} elements out of bound, first {np.argwhere(bad)[0]}"
    return rel


def _problem(M, d_out, d_in, r, seed):
    X = synth.activations_bf16(M, d_in, seed, seed + 1)
    dY = synth.gaussian_bf16((M, d_out), 1.0, seed + 2)
    U = synth.gaussian_bf16((d_out, r), 0.02, seed + 3)
    V = synth.gaussian_bf16((r, d_in), 1.0 / np.sqrt(d_in), seed + 4)
    return X, dY, U, V


@pytest.mark.parametrize("M,d_out,d_in,r", [(64, 256, 256, 8), (300, 520, 384, 64), (200, 136, 192, 96),
                                            (130, 264, 128, 128), (96, 128, 320, 256), (2048, 14336, 4096, 64)])
def test_lora_backward(M, d_out, d_in, r):
    X, dY, U, V = _problem(M, d_out, d_in, r, M + d_out + r)
    dU, dV = slr.lora_backward(to_dev(X), to_dev(dY), to_dev(U), to_dev(V))
    torch.cuda.synchronize()
    slr.check_kernel_error()
    rdU, rdV, BU, BV = lb.lora_backward(X, dY, U, V)
    _check(dU, rdU, BU, f"dU {M}x{d_out}x{d_in} r={r}")
    _check(dV, rdV, BV, f"dV {M}x{d_out}x{d_in} r={r}")


def test_lora_backward_with_forward_T_and_zero_tokens():
    M, d_out, d_in, r = 192, 512, 256, 64
    X, dY, U, V = _problem(M, d_out, d_in, r, 5)
    Xd, Ud, Vd = to_dev(X), to_dev(U), to_dev(V)
    T = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(max(slr.workspace_size(M, d_out, d_in, r), 256), dtype=torch.uint8, device="cuda")
    slr.forward_project(Xd, Vd, d_out, ws, path="tensor")   # the forward's T (bf16) in the workspace
    T.copy_(ws[: M * r * 2].view(torch.bfloat16).view(M, r))
    dU, dV = slr.lora_backward(Xd, to_dev(dY), Ud, Vd, T=T)
    rdU, rdV, BU, BV = lb.lora_backward(X, dY, U, V)
    _check(dU, rdU, BU, "dU with T")
    _check(dV, rdV, BV, "dV with T")
    e = torch.empty((0, d_in), dtype=torch.bfloat16, device="cuda")
    dU0, dV0 = slr.lora_backward(e, torch.empty((0, d_out), dtype=torch.bfloat16, device="cuda"), Ud, Vd)
    assert torch.count_nonzero(dU0) == 0 and torch.count_nonzero(dV0) == 0

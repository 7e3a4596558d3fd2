"""GPU parity of the data-free alternating minimisation W ~ S + U V (HASSLE-free
section 4, identity Hessian; LoSparse section 3.2 start) against the fp64
oracle (oracle/datafree_am.py: exact SVD, exact hard threshold).

The GPU computes C_r by subspace iteration in fp32 and rounds S, U, V to bf16
for storage, so trajectories are compared through what is unique: the
objective ||W - S - U V||_F after the start and after every iteration
(relative 2e-3 once the subspace iteration has converged), its monotone
decrease, the 2:4 structure of S, and the consistency of the returned
factors with the reported objective.
"""
import numpy as np
import pytest
import torch

import oracle.datafree_am as am
import synth
from gpu_util import bits_to_f64, from_dev, to_dev

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sparse_rank_linear_02_b200 as slr


def _q0(d_in, r, seed):
    return torch.from_numpy(np.random.Generator(np.random.PCG64(seed)).standard_normal((d_in, r))
                            .astype(np.float32)).cuda()


def _dense_S(vals, meta, d_in):
    import oracle
    return bits_to_f64(oracle.unpack_2to4(from_dev(vals), meta.cpu().numpy(), d_in))


def _check_structure(vals, meta, d_out, d_in):
    m = meta.cpu().numpy().astype(np.int64)
    nib = np.stack([m & 0xF, m >> 4], axis=-1).reshape(d_out, -1)[:, : d_in // 4]
    lo, hi = nib & 3, nib >> 2
    assert np.all(lo < hi), "metadata nibbles must name two ascending positions"


def _gapped(d_out, d_in, r, seed, top=40.0):
    """A rank-r part with singular values top .. top/2 plus a 2:4 part and noise,
    so the spectrum has a clear gap after the r-th value (the subspace iteration
    converges in a few dozen steps and the trajectories are comparable)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    Uo, _ = np.linalg.qr(rng.normal(size=(d_out, r)))
    Vo, _ = np.linalg.qr(rng.normal(size=(d_in, r)))
    L = (Uo * np.linspace(top, top / 2, r)) @ Vo.T
    S0 = am.hard_threshold_2to4(rng.normal(size=(d_out, d_in))) * 0.5
    return synth.f32_to_bf16_bits((L + S0 + 0.05 * rng.normal(size=(d_out, d_in))).astype(np.float32))


def _run_and_compare(W, r, iters, power_first, power, rtol, seed):
    d_out, d_in = W.shape
    vals, meta, U, V, obj = slr.decompose_datafree(to_dev(W), r, iters, power_first=power_first, power=power,
                                                    Q0=_q0(d_in, r, seed))
    torch.cuda.synchronize()
    obj = obj.cpu().numpy()
    _, _, ref = am.alternating_minimisation(bits_to_f64(W), r, iters)
    np.testing.assert_allclose(obj, ref, rtol=rtol)
    assert all(b <= a * (1 + 1e-5) for a, b in zip(obj, obj[1:])), obj
    _check_structure(vals, meta, d_out, d_in)
    S = _dense_S(vals, meta, d_in)
    L = bits_to_f64(from_dev(U)) @ bits_to_f64(from_dev(V))
    recon = np.linalg.norm(bits_to_f64(W) - S - L)
    assert abs(recon - obj[-1]) <= 1e-2 * obj[-1], (recon, obj[-1])


@pytest.mark.parametrize("d_out,d_in,r,iters", [(256, 128, 8, 4), (192, 320, 16, 3), (520, 264, 32, 3)])
def test_decompose_matches_oracle_gapped(d_out, d_in, r, iters):
    """Spectral gap after r: every objective within 1e-3 of the exact oracle's."""
    _run_and_compare(_gapped(d_out, d_in, r, d_out + r), r, iters, 40, 10, 1e-3, 5)


def test_decompose_matches_oracle_gaussian():
    """A Gaussian W has almost no gap after r, so the fp32 subspace iteration and
    the exact SVD may settle on slightly different (equally good) subspaces and
    the trajectories drift apart: objectives within 1e-2."""
    W = synth.gaussian_bf16((256, 128), 0.02, 384)
    _run_and_compare(W, 8, 4, 80, 30, 1e-2, 5)


def test_decompose_start_is_eckart_young():
    """iters = 0: U V is C_r(W) (the truncation error equals the sum of the
    trailing squared singular values) and S the hard threshold of W - U V."""
    d_out, d_in, r = 300, 160, 24
    W = _gapped(d_out, d_in, r, 7)
    Wf = bits_to_f64(W)
    vals, meta, U, V, obj = slr.decompose_datafree(to_dev(W), r, 0, power_first=60, Q0=_q0(d_in, r, 8))
    L = bits_to_f64(from_dev(U)) @ bits_to_f64(from_dev(V))
    sv = np.linalg.svd(Wf, compute_uv=False)
    ey = np.sqrt(np.sum(sv[r:] ** 2))
    assert abs(np.linalg.norm(Wf - L) - ey) <= 2e-3 * ey
    _, _, ref = am.alternating_minimisation(Wf, r, 0)
    np.testing.assert_allclose(obj.cpu().numpy(), ref, rtol=1e-3)


def test_decompose_recovers_planted_structure():
    """W = S0 + L0 (2:4 with large entries plus rank 8), r = 8: the alternation
    all but recovers the planted pair, on the GPU as in the oracle."""
    rng = np.random.Generator(np.random.PCG64(11))
    d_out, d_in, r = 384, 256, 8
    S0 = am.hard_threshold_2to4(rng.normal(size=(d_out, d_in)) * 3.0)
    L0 = rng.normal(size=(d_out, r)) @ rng.normal(size=(r, d_in)) * 0.3
    W = synth.f32_to_bf16_bits((S0 + L0).astype(np.float32))
    Wn = np.linalg.norm(bits_to_f64(W))
    _, _, _, _, obj = slr.decompose_datafree(to_dev(W), r, 16, power_first=60, power=6, Q0=_q0(d_in, r, 12))
    obj = obj.cpu().numpy()
    _, _, ref = am.alternating_minimisation(bits_to_f64(W), r, 16)
    assert ref[-1] < 0.01 * ref[0], ref           # the oracle recovers it ...
    assert obj[-1] < 0.01 * obj[0], obj           # ... and so does the GPU
    assert obj[-1] <= 1.1 * ref[-1] + 2e-3 * Wn, (obj[-1], ref[-1])


def test_decompose_deterministic():
    W = to_dev(synth.gaussian_bf16((128, 96), 0.02, 13))
    a = slr.decompose_datafree(W, 8, 2, Q0=_q0(96, 8, 1))
    b = slr.decompose_datafree(W, 8, 2, Q0=_q0(96, 8, 1))
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.uint8) if x.dtype != torch.float64 else x,
                           y.view(torch.uint8) if y.dtype != torch.float64 else y)


def test_decompose_config_layer():
    """The Llama-3-8B gate/up shape (14336 x 4096, r = 64), three iterations of
    two warm-started power steps: monotone objective, valid 2:4 metadata,
    finite factors."""
    layer = next(l for l in synth.CONFIGS[3].layers if l.name == "gate_up")
    W = layer.weight()
    vals, meta, U, V, obj = slr.decompose_datafree(to_dev(W), 64, 3, power_first=8, power=2,
                                                    Q0=_q0(layer.d_in, 64, 3))
    torch.cuda.synchronize()
    obj = obj.cpu().numpy()
    assert np.all(np.isfinite(obj)) and obj[0] < np.linalg.norm(bits_to_f64(W))
    assert all(b <= a * (1 + 1e-4) for a, b in zip(obj, obj[1:])), obj
    _check_structure(vals, meta, layer.d_out, layer.d_in)
    assert torch.isfinite(U.float()).all() and torch.isfinite(V.float()).all()


# ----------------------------------------------------------------------------- element-wise P1 / P2

def _gpu_mask(meta, d_out, d_in):
    """Kept positions named by the packed metadata (boolean [d_out, d_in])."""
    m = meta.cpu().numpy().astype(np.int64)
    nib = np.stack([m & 0xF, m >> 4], axis=-1).reshape(d_out, -1)[:, : d_in // 4]
    mask = np.zeros((d_out, d_in // 4, 4), dtype=bool)
    rows, groups = np.indices(nib.shape)
    mask[rows, groups, nib & 3] = True
    mask[rows, groups, nib >> 2] = True
    return mask.reshape(d_out, d_in)


def _check_p1(W, vals, meta, U32, V32, what, max_ambiguous=1e-2):
    """S must be the 2:4 hard threshold (HASSLE-free section 4.1.1) of W - L with
    L = U32 V32, the GPU's own unrounded low-rank part: identical kept positions
    in every group except those where the second and third largest |W - L|
    lie within the GPU's rounding of each other, and kept values equal to
    W - L rounded to bf16.  The GPU forms L from bf16 hi/lo planes of the two
    factors (|error| <= 2^-16 (|U32||V32|)_ij per product, three products) and
    W - L in fp32; the tolerance per entry is four times that estimate."""
    d_out, d_in = W.shape
    Wf = bits_to_f64(W)
    Uf = U32.double().cpu().numpy()
    Vf = V32.double().cpu().numpy()
    L = Uf @ Vf
    R = Wf - L
    tol = 4.0 * (3 * 2.0 ** -16 * (np.abs(Uf) @ np.abs(Vf)) + 2.0 ** -23 * (np.abs(Wf) + np.abs(L)))
    keep_ref = am.keep_mask_2to4(R)
    keep_gpu = _gpu_mask(meta, d_out, d_in)
    # ambiguous groups: the two entries either side of the cut are within tolerance
    a = np.abs(R).reshape(d_out, -1, 4)
    t = tol.reshape(d_out, -1, 4)
    order = np.argsort(-a, axis=-1, kind="stable")
    a2 = np.take_along_axis(a, order[..., 1:2], -1)[..., 0]
    a3 = np.take_along_axis(a, order[..., 2:3], -1)[..., 0]
    t2 = np.take_along_axis(t, order[..., 1:2], -1)[..., 0]
    t3 = np.take_along_axis(t, order[..., 2:3], -1)[..., 0]
    ambiguous = (a2 - a3) <= (t2 + t3)
    differs = np.any(keep_ref.reshape(d_out, -1, 4) != keep_gpu.reshape(d_out, -1, 4), axis=-1)
    n_groups = differs.size
    assert not np.any(differs & ~ambiguous), \
        f"{what}: {int(np.sum(differs & ~ambiguous))} groups keep other positions than the hard threshold " \
        f"of W - U32 V32 outside rounding ties (first at row, group {np.argwhere(differs & ~ambiguous)[0]})"
    assert ambiguous.sum() <= max_ambiguous * n_groups, (what, int(ambiguous.sum()), n_groups)
    # kept values: bf16 of W - L (half an ulp of bf16, plus the tolerance)
    S = bits_to_f64(oracle_unpack(vals, meta, d_in))
    ok = np.repeat(~ambiguous, 4, axis=-1).reshape(d_out, d_in) & keep_gpu
    err = np.abs(S - R)
    bound = 2.0 ** -8 * np.abs(R) + tol + 1e-30
    assert np.all(err[ok] <= bound[ok]), f"{what}: kept value off W - L by {float(np.max(err[ok] - bound[ok])):.3g}"
    assert np.all(S[~keep_gpu] == 0.0)
    return int(differs.sum()), int(ambiguous.sum()), n_groups


def oracle_unpack(vals, meta, d_in):
    import oracle
    return oracle.unpack_2to4(from_dev(vals), meta.cpu().numpy(), d_in)


@pytest.mark.parametrize("d_out,d_in,r,iters", [(256, 128, 8, 3), (192, 320, 16, 2), (520, 264, 32, 2)])
def test_decompose_p1_and_p2_element_wise_gapped(d_out, d_in, r, iters):
    """After `iters` iterations:
    P1 -- S is the hard threshold of W - U32 V32 (see _check_p1);
    P2 -- U32 V32 is C_r(W - S_prev) (HASSLE-free section 4.2.1) element by
    element, S_prev being the GPU's S after iters - 1 iterations (the run is
    deterministic and warm-started, so the shorter run is a prefix of the
    longer one): |L_gpu - C_r|_ij <= 2e-4 max|C_r| (fp32 subspace iteration
    on hi/lo planes of W - S_prev, converged on a matrix with a spectral gap),
    and the bf16 factors U V within their rounding, 2^-7 (|U||V|)_ij, of it."""
    W = _gapped(d_out, d_in, r, d_out + r)
    q0 = _q0(d_in, r, 5)
    vp, mp, _, _, _ = slr.decompose_datafree(to_dev(W), r, iters - 1, power_first=40, power=10, Q0=q0)
    vals, meta, U, V, obj, U32, V32 = slr.decompose_datafree(to_dev(W), r, iters, power_first=40, power=10, Q0=q0,
                                                             factors_f32=True)
    torch.cuda.synchronize()
    _check_p1(W, vals, meta, U32, V32, f"P1 {d_out}x{d_in} r={r}")
    Wf = bits_to_f64(W)
    S_prev = bits_to_f64(oracle_unpack(vp, mp, d_in))
    L_ref = am.truncated_svd(Wf - S_prev, r)
    L_gpu = U32.double().cpu().numpy() @ V32.double().cpu().numpy()
    scale = np.max(np.abs(L_ref))
    err = np.abs(L_gpu - L_ref)
    assert np.max(err) <= 2e-4 * scale, f"P2: max |U32 V32 - C_r(W - S_prev)| = {np.max(err) / scale:.3g} of max|C_r|"
    Ub, Vb = bits_to_f64(from_dev(U)), bits_to_f64(from_dev(V))
    errb = np.abs(Ub @ Vb - L_ref)
    assert np.all(errb <= 2.0 ** -7 * (np.abs(Ub) @ np.abs(Vb)) + 2e-4 * scale), "P2: bf16 factors"


def test_decompose_config_layer_start_and_threshold():
    """The gate/up layer (14336 x 4096, r = 64), iters = 0: the start's U32 V32
    captures the top-r energy of W up to the subspace iteration's convergence
    (||W - U32 V32||_F between the Eckart-Young error, from the eigenvalues of
    W^T W, and 1.002 times it), and S is the hard threshold of W - U32 V32
    element by element (P1 check above)."""
    layer = next(l for l in synth.CONFIGS[3].layers if l.name == "gate_up")
    W = layer.weight()
    vals, meta, U, V, obj, U32, V32 = slr.decompose_datafree(to_dev(W), 64, 0, power_first=8, power=2,
                                                             Q0=_q0(layer.d_in, 64, 3), factors_f32=True)
    torch.cuda.synchronize()
    Wf = bits_to_f64(W)
    ev = np.linalg.eigvalsh(Wf.T @ Wf)
    ey = np.sqrt(max(np.sum(Wf * Wf) - np.sum(ev[-64:]), 0.0))
    L = U32.double().cpu().numpy() @ V32.double().cpu().numpy()
    fit = np.linalg.norm(Wf - L)
    assert ey * (1 - 1e-6) <= fit <= ey * 1.002, (fit, ey)
    del L
    _check_p1(W, vals, meta, U32, V32, "P1 gate/up start")

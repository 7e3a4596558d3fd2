"""GPU parity of the activation-aware 2:4 projection (HASSLE-free, section
4.1.2: diagonal Hessian, Wanda's score |w_ij| * ||X_:,j||) and of the column
norms that feed it, through the C ABI, against the fp64 oracle.

Projection: bit-exact, given the same fp32 scales, on the configuration
shapes (scales = the oracle's column norms of the layer's synthetic
activations, outlier channels included, rounded to fp32) and on adversarial
weights and scales (ties, NaN, Inf, zero and negative scales), on both the
vectorised and the general kernel.

Column norms: the fp64 running sum of squares within 80 * 2^-24 relative of
the oracle's fp64 sum (the fp32 partial sums are at most 64 + 8 terms deep),
norms within 41 * 2^-24; accumulation over batches; deterministic bits.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import check_forward, from_dev, layer_weights, sample_indices, to_dev, to_dev_u8

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sparse_rank_linear_02_b200 as slr

SUMSQ_REL_TOL = 80 * 2.0 ** -24
NORM_REL_TOL = 41 * 2.0 ** -24


def _scale_dev(s: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(s, dtype=np.float32)).cuda()


def _shapes():
    seen, out = set(), []
    for c in synth.CONFIGS.values():
        for l in c.layers:
            if (l.d_out, l.d_in) not in seen:
                seen.add((l.d_out, l.d_in))
                out.append((c.cfg, l.name))
    return out


def _check_pack_rows(W, scale, vals, meta, rows):
    """Oracle on a row subset (the projection is row-local)."""
    vref, mref = oracle.pack_2to4_scaled(np.ascontiguousarray(W[rows]), scale)
    np.testing.assert_array_equal(from_dev(vals)[rows], vref)
    np.testing.assert_array_equal(meta.cpu().numpy()[rows], mref)


# ----------------------------------------------------------------------------- projection

@pytest.mark.parametrize("cfg,name", _shapes(), ids=lambda x: str(x))
def test_pack_scaled_config_bit_exact(cfg, name):
    """Full-size layers, scales from the oracle's norms of 256 calibration
    tokens; every row on layers up to 2^24 weights, 512 sampled rows above."""
    layer = next(l for l in synth.CONFIGS[cfg].layers if l.name == name)
    W = layer.weight()
    X = layer.activations(256)
    scale = oracle.column_norms(X).astype(np.float32)
    vals, meta = slr.pack_2to4_scaled(to_dev(W), _scale_dev(scale))
    torch.cuda.synchronize()
    rows = np.arange(layer.d_out) if layer.d_out * layer.d_in <= (1 << 24) else \
        sample_indices(layer.d_out, 512, seed=cfg * 13 + layer.d_out)
    _check_pack_rows(W, scale, vals, meta, rows)
    # The outlier channels change the choice somewhere (else the test proves little).
    plain, _ = oracle.pack_2to4(np.ascontiguousarray(W[rows[:64]]))
    if layer.x_outliers:
        assert not np.array_equal(from_dev(vals)[rows[:64]], plain)


def _adversarial(seed, rows, cols):
    rng = np.random.Generator(np.random.PCG64(seed))
    W = rng.integers(0, 1 << 16, size=(rows, cols), dtype=np.uint32).astype(np.uint16)
    W[:, : cols // 4] &= 0x8000 | 0x3F80          # +-1.0 / +-0: ties under equal scales
    W[rows // 2:, cols // 2:] = rng.choice(np.array([0, 0x8000, 0x3F80, 0xBF80, 0x7F80, 0xFF80, 0x7FC0],
                                                    dtype=np.uint16), size=(rows - rows // 2, cols - cols // 2))
    scale = np.ldexp(1.0, rng.integers(-3, 4, size=cols)).astype(np.float32)
    scale *= rng.choice(np.array([1, -1], dtype=np.float32), size=cols)
    special = slice(cols // 3, min(cols, cols // 3 + 16))
    n_special = special.stop - special.start
    scale[special] = rng.choice(np.array([0, np.inf, -np.inf, np.nan, 1e-45, 3e38], dtype=np.float32),
                                size=n_special)
    if cols >= 64:
        scale[-8:] = rng.uniform(0.1, 10, size=8).astype(np.float32)   # rounded products
    return W, scale


@pytest.mark.parametrize("rows,cols", [(64, 256), (33, 72), (5, 12), (7, 4), (128, 4100), (3, 2048 + 8)])
def test_pack_scaled_adversarial_bit_exact(rows, cols):
    W, scale = _adversarial(rows * 1000 + cols + 1, rows, cols)
    vals, meta = slr.pack_2to4_scaled(to_dev(W), _scale_dev(scale))
    _check_pack_rows(W, scale, vals, meta, np.arange(rows))


def test_pack_scaled_rounded_products_bit_exact():
    """Log-normal scales: products round in fp32, near-ties decided by rounding."""
    rng = np.random.Generator(np.random.PCG64(31))
    W = synth.gaussian_bf16((300, 1024), 0.02, 32)
    scale = np.exp(rng.normal(0.0, 2.0, size=1024)).astype(np.float32)
    vals, meta = slr.pack_2to4_scaled(to_dev(W), _scale_dev(scale))
    _check_pack_rows(W, scale, vals, meta, np.arange(300))


def test_pack_scaled_strided_and_unaligned():
    """ldw > d_in, and W / scale pointers that are not 16-byte aligned (the
    general kernel), against the same oracle."""
    big, scale_big = _adversarial(77, 40, 264)
    Wd, Sd = to_dev(big), _scale_dev(scale_big)
    for lo, hi in [(0, 256), (8, 264), (4, 260), (1, 253)]:
        scale = np.ascontiguousarray(scale_big[lo:hi])
        vals, meta = slr.pack_2to4_scaled(Wd[:, lo:hi], Sd[lo:hi])
        vref, mref = oracle.pack_2to4_scaled(np.ascontiguousarray(big[:, lo:hi]), scale)
        np.testing.assert_array_equal(from_dev(vals), vref)
        np.testing.assert_array_equal(meta.cpu().numpy(), mref)


def test_pack_scaled_uniform_matches_plain_kernel():
    """Uniform power-of-two scales reduce to the plain projection on finite weights."""
    W = synth.gaussian_bf16((96, 512), 0.02, 33)
    Wd = to_dev(W)
    v0, m0 = slr.pack_2to4(Wd)
    v1, m1 = slr.pack_2to4_scaled(Wd, torch.full((512,), -4.0, device="cuda"))
    assert torch.equal(v0.view(torch.int16), v1.view(torch.int16)) and torch.equal(m0, m1)


def test_pack_scaled_empty_and_errors():
    empty = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    vals, meta = slr.pack_2to4_scaled(empty, torch.ones(64, device="cuda"))
    assert vals.shape == (0, 32) and meta.shape == (0, 8)
    st = slr.lib().slr_pack_2to4_scaled(None, 4, 8, 8, None, None, None, None)
    assert st == 1                                   # SLR_ERR_NULL
    st = slr.lib().slr_pack_2to4_scaled(None, 4, 6, 8, None, None, None, None)
    assert st == 2                                   # SLR_ERR_SHAPE (d_in % 4)


# ----------------------------------------------------------------------------- column norms

def _check_norms(norms, sumsq, ref_sumsq, what):
    s = sumsq.cpu().numpy()
    rel = np.abs(s - ref_sumsq) / np.maximum(ref_sumsq, 1e-300)
    assert np.all((rel <= SUMSQ_REL_TOL) | (ref_sumsq == 0)), f"{what}: sumsq rel err {rel.max():.3e}"
    assert np.all(s[ref_sumsq == 0] == 0)
    if norms is not None:
        n = norms.cpu().numpy().astype(np.float64)
        ref = np.sqrt(ref_sumsq)
        nrel = np.abs(n - ref) / np.maximum(ref, 1e-300)
        assert np.all((nrel <= NORM_REL_TOL) | (ref == 0)), f"{what}: norm rel err {nrel.max():.3e}"


@pytest.mark.parametrize("M,d_in", [(1, 8), (77, 264), (256, 4096), (2048, 4096), (1000, 14336), (5000, 72)])
def test_column_norms(M, d_in):
    """Ragged strips (d_in not a multiple of 256), ragged row splits, outlier
    channels (1% of the columns scaled by 20)."""
    X = synth.activations_bf16(M, d_in, seed=M + d_in, outlier_seed=M * 3 + 1)
    norms, sumsq = slr.column_norms(to_dev(X))
    ref = oracle.column_norms(X) ** 2
    _check_norms(norms, sumsq, ref, f"M={M} d_in={d_in}")


def test_column_norms_accumulate_and_strided():
    """Three batches (one empty, one a column slice with ldx > d_in) add up to
    the oracle's norms of the stacked tokens; M == 0 rewrites the norms only."""
    X1 = synth.activations_bf16(300, 512, seed=41, outlier_seed=42)
    wide = synth.activations_bf16(129, 520, seed=43, outlier_seed=None)
    X2 = np.ascontiguousarray(wide[:, 8:])
    _, sumsq = slr.column_norms(to_dev(X1), want_norms=False)
    norms, sumsq = slr.column_norms(to_dev(np.zeros((0, 512), dtype=np.uint16)), sumsq)
    _check_norms(norms, sumsq, oracle.column_norms(X1) ** 2, "batch 1")
    norms, sumsq = slr.column_norms(to_dev(wide)[:, 8:], sumsq)
    _check_norms(norms, sumsq, oracle.column_norms(np.vstack([X1, X2])) ** 2, "batches 1+2")


def test_column_norms_deterministic_and_exact_cases():
    X = synth.activations_bf16(4096, 1024, seed=51, outlier_seed=52)
    Xd = to_dev(X)
    a, sa = slr.column_norms(Xd)
    b, sb = slr.column_norms(Xd)
    assert torch.equal(a, b) and torch.equal(sa, sb)
    # Integer-valued squares sum exactly: constant columns c over 4096 rows.
    C = np.zeros((4096, 16), dtype=np.uint16)
    C[:] = synth.f32_to_bf16_bits(np.array([1, -2, 3, 0.5, 0, -0.25, 8, 1.5] * 2, dtype=np.float32))
    n, s = slr.column_norms(to_dev(C))
    np.testing.assert_array_equal(n.cpu().numpy(), 64 * np.abs(np.array([1, -2, 3, 0.5, 0, -0.25, 8, 1.5] * 2,
                                                                           dtype=np.float32)))


def test_column_norms_errors():
    lib = slr.lib()
    assert lib.slr_column_norms(None, 4, 12, 12, None, None, None, 0, None) == 2   # d_in % 8
    assert lib.slr_column_norms(None, 4, 8, 8, None, None, None, 0, None) == 1     # sumsq NULL
    assert lib.slr_column_norms(None, 4, 0, 0, None, None, None, 0, None) == 0     # nothing to do
    X = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    s = torch.zeros(64, dtype=torch.float64, device="cuda")
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    need = slr.column_norms_workspace_size(64, 64)
    assert need > 16
    st = lib.slr_column_norms(X.data_ptr(), 64, 64, 64, s.data_ptr(), None, ws.data_ptr(), 16, None)
    assert st == 4                                                                  # SLR_ERR_WORKSPACE


# ----------------------------------------------------------------------------- calibrate, project, run

def test_calibrated_layer_forward():
    """Norms from calibration tokens (GPU) within tolerance of the oracle's; the
    projection with the oracle's fp32 norms is bit-exact; the forward of that
    packed layer meets the acceptance bounds against the oracle."""
    layer, W, _, _, U, V = layer_weights(2, "q_proj")
    Xcal = layer.activations(512)
    norms, sumsq = slr.column_norms(to_dev(Xcal))
    ref = oracle.column_norms(Xcal)
    _check_norms(norms, sumsq, ref ** 2, "calibration")
    scale = ref.astype(np.float32)
    vals, meta = slr.pack_2to4_scaled(to_dev(W), _scale_dev(scale))
    vref, mref = oracle.pack_2to4_scaled(W, scale)
    np.testing.assert_array_equal(from_dev(vals), vref)
    np.testing.assert_array_equal(meta.cpu().numpy(), mref)
    X = layer.activations(64)
    Y = slr.forward(to_dev(X), to_dev(vref), to_dev_u8(mref), to_dev(U), to_dev(V))
    rows = sample_indices(64, 64, 3)
    outs = sample_indices(layer.d_out, 512, 4)
    Yref, Bref = oracle.forward(X, vref, mref, U, V, rows=rows, outs=outs)
    check_forward(from_dev(Y)[np.ix_(rows, outs)], Yref, Bref, "calibrated q_proj", rows, outs)

"""Pins for the CPU oracle: checks against facts fixed by the pages and by
mathematics, never against the oracle itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError
when the oracle disagrees.  ``tests/test_oracle.py`` runs them on the real
oracle; ``tests/test_oracle_mutants.py`` runs them on deliberately broken
copies to show that each plausible mistake is caught by at least one pin.
"""
from __future__ import annotations

import itertools
import os

import numpy as np

import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "worked_example.txt")

# bf16 bit patterns of the small alphabet {0, -0, +-1, +-2, +-3, +-4}.
_ALPHABET = np.array([0x0000, 0x8000, 0x3F80, 0xBF80, 0x4000, 0xC000,
                      0x4040, 0xC040, 0x4080, 0xC080], dtype=np.uint16)


def _bf16(x) -> np.ndarray:
    return synth.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def _f64(bits) -> np.ndarray:
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def brute_force_pair(group_abs) -> tuple[int, int]:
    """Frobenius-optimal 2:4 choice by enumeration of all six index pairs.

    A pair is optimal when every kept magnitude is >= every dropped one (the
    hard-thresholding optimum of HASSLE-free section 4.1.1); among optimal
    pairs take the lexicographically smallest (the lower-index tie rule).
    """
    best = None
    for a, b in itertools.combinations(range(4), 2):
        dropped = [group_abs[p] for p in range(4) if p not in (a, b)]
        if min(group_abs[a], group_abs[b]) >= max(dropped):
            if best is None or (a, b) < best:
                best = (a, b)
    return best


def decode_meta(meta_row: np.ndarray, groups: int):
    out = []
    for g in range(groups):
        nib = (int(meta_row[g // 2]) >> (4 * (g % 2))) & 0xF
        out.append((nib & 3, nib >> 2))
    return out


def read_golden(path: str = GOLDEN):
    rows = {}
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            rows.setdefault(key, []).append(vals)
    hexrows = lambda k: np.array([[int(v, 16) for v in r] for r in rows[k]], dtype=np.uint16)
    return {
        "W": hexrows("W"), "VALS": hexrows("VALS"),
        "META": np.array([[int(v, 16) for v in r] for r in rows["META"]], dtype=np.uint8),
        "X": hexrows("X"), "U": hexrows("U"), "V": hexrows("V"),
        "Y": np.array([[float(v) for v in r] for r in rows["Y"]]),
        "B": np.array([[float(v) for v in r] for r in rows["B"]]),
    }


# --------------------------------------------------------------------------- pack pins

def pin_pack_golden(o):
    g = read_golden()
    vals, meta = o.pack_2to4(g["W"])
    np.testing.assert_array_equal(vals, g["VALS"])
    np.testing.assert_array_equal(meta, g["META"])


def pin_pack_exhaustive_alphabet(o):
    """Every group of four over the 10-letter alphabet (10^4 groups)."""
    groups = np.array(list(itertools.product(range(len(_ALPHABET)), repeat=4)))
    W = _ALPHABET[groups].reshape(-1, 4)        # one group per row, d_in = 4
    vals, meta = o.pack_2to4(W)
    absf = np.abs(_f64(W))
    for i in range(W.shape[0]):
        a, b = brute_force_pair(absf[i])
        nib = int(meta[i, 0]) & 0xF
        assert (nib & 3, nib >> 2) == (a, b), (i, W[i], (nib & 3, nib >> 2), (a, b))
        assert vals[i, 0] == W[i, a] and vals[i, 1] == W[i, b], (i, W[i], vals[i])
        assert int(meta[i, 0]) >> 4 == 0


def pin_pack_random_bruteforce(o, seed: int = 7):
    """Random bf16 groups with a narrow exponent range (many exact ties)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    sign = rng.integers(0, 2, size=(300, 24)).astype(np.uint16) << 15
    expo = rng.integers(125, 129, size=(300, 24)).astype(np.uint16) << 7
    mant = rng.integers(0, 4, size=(300, 24)).astype(np.uint16) << 5
    W = (sign | expo | mant).astype(np.uint16)
    vals, meta = o.pack_2to4(W)
    absf = np.abs(_f64(W))
    for i in range(W.shape[0]):
        pairs = decode_meta(meta[i], 6)
        for g in range(6):
            a, b = brute_force_pair(absf[i, 4 * g:4 * g + 4])
            assert pairs[g] == (a, b), (i, g)
            assert vals[i, 2 * g] == W[i, 4 * g + a] and vals[i, 2 * g + 1] == W[i, 4 * g + b]


def pin_pack_invariants(o):
    layer = synth.CONFIGS[1].layers[0]
    W = layer.weight()
    vals, meta = o.pack_2to4(W)
    d_out, d_in = W.shape
    S = o.unpack_2to4(vals, meta, d_in)
    Wf = np.abs(_f64(W))
    for i in range(0, d_out, 7):
        pairs = decode_meta(meta[i], d_in // 4)
        for g, (a, b) in enumerate(pairs):
            assert 0 <= a < b <= 3
            grp = Wf[i, 4 * g:4 * g + 4]
            dropped = [grp[p] for p in range(4) if p not in (a, b)]
            assert min(grp[a], grp[b]) >= max(dropped)
            assert np.count_nonzero(S[i, 4 * g:4 * g + 4] & 0x7FFF) <= 2
            for p in range(4):
                if p not in (a, b):
                    assert S[i, 4 * g + p] == 0
                else:
                    assert S[i, 4 * g + p] == W[i, 4 * g + p]


def pin_pack_roundtrip(o):
    W = synth.gaussian_bf16((64, 96), 0.02, 11)
    vals, meta = o.pack_2to4(W)
    S = o.unpack_2to4(vals, meta, 96)
    vals2, meta2 = o.pack_2to4(S)          # idempotent on an already-projected matrix
    np.testing.assert_array_equal(vals2, vals)
    np.testing.assert_array_equal(meta2, meta)
    # A matrix that is 2:4 by construction packs losslessly.
    rng = np.random.Generator(np.random.PCG64(12))
    dense = np.zeros((32, 64), dtype=np.uint16)
    for i in range(32):
        for g in range(16):
            a, b = sorted(rng.choice(4, size=2, replace=False))
            dense[i, 4 * g + a] = _bf16([rng.uniform(0.5, 2.0) * rng.choice([-1, 1])])[0]
            dense[i, 4 * g + b] = _bf16([rng.uniform(0.5, 2.0) * rng.choice([-1, 1])])[0]
    v3, m3 = o.pack_2to4(dense)
    np.testing.assert_array_equal(o.unpack_2to4(v3, m3, 64), dense)


def pin_pack_specials(o):
    """NaN/Inf/-0 follow the integer magnitude key (a stated reading)."""
    W = np.array([[0x3F80, 0x7FC0, 0x7F80, 0xFF80,      # 1, NaN, +Inf, -Inf -> keep NaN, +Inf
                   0x8000, 0x0000, 0x8000, 0x0000]],     # -0, +0, -0, +0     -> keep idx 0, 1
                 dtype=np.uint16)
    vals, meta = o.pack_2to4(W)
    np.testing.assert_array_equal(vals, [[0x7FC0, 0x7F80, 0x8000, 0x0000]])
    assert int(meta[0, 0]) == ((1 | 2 << 2) | ((0 | 1 << 2) << 4))


def pin_pack_odd_groups(o):
    """d_in = 12: three groups, the last meta byte holds one nibble."""
    W = _bf16([[1, 2, 3, 4, 4, 3, 2, 1, 0, 5, 0, 5]])
    vals, meta = o.pack_2to4(W)
    assert meta.shape == (1, 2)
    np.testing.assert_array_equal(vals, _bf16([[3, 4, 4, 3, 5, 5]]))
    assert int(meta[0, 0]) == ((2 | 3 << 2) | ((0 | 1 << 2) << 4))
    assert int(meta[0, 1]) == (1 | 3 << 2)


# --------------------------------------------------------------------------- forward pins

def pin_forward_golden(o):
    g = read_golden()
    Y, B = o.forward(g["X"], g["VALS"], g["META"], g["U"], g["V"])
    np.testing.assert_array_equal(Y, g["Y"])
    np.testing.assert_array_equal(B, g["B"])


def _small_int_problem(seed, M, d_out, d_in, r):
    rng = np.random.Generator(np.random.PCG64(seed))
    X = _bf16(rng.integers(-3, 4, size=(M, d_in)))
    W = _bf16(rng.integers(-4, 5, size=(d_out, d_in)))
    U = _bf16(rng.integers(-2, 3, size=(d_out, r)))
    V = _bf16(rng.integers(-2, 3, size=(r, d_in)))
    return X, W, U, V


def pin_forward_identity_exact(o):
    """X (S + U V)^T == X S^T + (X V^T) U^T, exactly, with small integers
    (every partial sum is an integer well inside fp64's exact range)."""
    for seed, (M, d_out, d_in, r) in enumerate([(5, 12, 16, 3), (3, 8, 24, 1), (7, 20, 8, 6)]):
        X, W, U, V = _small_int_problem(100 + seed, M, d_out, d_in, r)
        vals, meta = o.pack_2to4(W)
        S = _f64(o.unpack_2to4(vals, meta, d_in))
        Xf, Uf, Vf = _f64(X), _f64(U), _f64(V)
        rhs = Xf @ S.T + (Xf @ Vf.T) @ Uf.T
        Y, B = o.forward(X, vals, meta, U, V)
        np.testing.assert_array_equal(Y, rhs)
        np.testing.assert_array_equal(B, np.abs(Xf) @ np.abs(S + Uf @ Vf).T)


def pin_forward_numpy(o):
    """fp64 library GEMM cross-check on non-square shapes (catches transposes)."""
    for (M, d_out, d_in, r, seed) in [(8, 256, 256, 8, 1), (6, 40, 72, 5, 2), (9, 24, 64, 16, 3)]:
        X = synth.gaussian_bf16((M, d_in), 1.0, seed * 10 + 1)
        W = synth.gaussian_bf16((d_out, d_in), 0.02, seed * 10 + 2)
        U = synth.gaussian_bf16((d_out, r), 0.3, seed * 10 + 3)
        V = synth.gaussian_bf16((r, d_in), 0.3, seed * 10 + 4)
        vals, meta = o.pack_2to4(W)
        S = _f64(o.unpack_2to4(vals, meta, d_in))
        Wp = S + _f64(U) @ _f64(V)
        ref = _f64(X) @ Wp.T
        Y, B = o.forward(X, vals, meta, U, V)
        scale = np.abs(_f64(X)) @ np.abs(Wp).T
        assert np.all(np.abs(Y - ref) <= 1e-12 * scale + 1e-300)
        assert np.all(np.abs(B - scale) <= 1e-12 * scale + 1e-300)
        assert np.all(np.abs(Y) <= B * (1 + 1e-12))


def pin_forward_one_hot(o):
    """X = e_j picks column j of W' = S + U V."""
    d_out, d_in, r = 16, 32, 4
    _, W, U, V = _small_int_problem(5, 1, d_out, d_in, r)
    vals, meta = o.pack_2to4(W)
    S = _f64(o.unpack_2to4(vals, meta, d_in))
    Wp = S + _f64(U) @ _f64(V)
    X = np.zeros((d_in, d_in), dtype=np.uint16)
    X[np.arange(d_in), np.arange(d_in)] = 0x3F80
    Y, _ = o.forward(X, vals, meta, U, V)
    np.testing.assert_array_equal(Y, Wp.T)


def pin_forward_sparse_only(o):
    """r = 0 (and U = 0) leaves X S^T."""
    X, W, U, V = _small_int_problem(6, 4, 12, 16, 3)
    vals, meta = o.pack_2to4(W)
    S = _f64(o.unpack_2to4(vals, meta, 16))
    Y0, _ = o.forward(X, vals, meta, None, None)
    np.testing.assert_array_equal(Y0, _f64(X) @ S.T)
    Yz, _ = o.forward(X, vals, meta, np.zeros_like(U), V)
    np.testing.assert_array_equal(Yz, _f64(X) @ S.T)


def pin_forward_row_subset(o):
    X, W, U, V = _small_int_problem(8, 10, 12, 16, 2)
    vals, meta = o.pack_2to4(W)
    Yall, Ball = o.forward(X, vals, meta, U, V)
    rows = [7, 0, 3, 3]
    Ys, Bs = o.forward(X, vals, meta, U, V, rows=rows)
    np.testing.assert_array_equal(Ys, Yall[rows])
    np.testing.assert_array_equal(Bs, Ball[rows])
    outs = [11, 2, 2, 5]
    Yo, Bo = o.forward(X, vals, meta, U, V, rows=rows, outs=outs)
    np.testing.assert_array_equal(Yo, Yall[np.ix_(rows, outs)])
    np.testing.assert_array_equal(Bo, Ball[np.ix_(rows, outs)])
    # The subset entries also match the numpy definition directly.
    S = _f64(o.unpack_2to4(vals, meta, 16))
    Wp = S + _f64(U) @ _f64(V)
    np.testing.assert_array_equal(Yo, (_f64(X) @ Wp.T)[np.ix_(rows, outs)])


def pin_lowrank_project(o):
    X, _, _, V = _small_int_problem(9, 6, 4, 24, 5)
    np.testing.assert_array_equal(o.lowrank_project(X, V), _f64(X) @ _f64(V).T)


# --------------------------------------------------------------------------- activation-aware pack pins
#
# HASSLE-free, section 4.1.2: with the diagonal Hessian D^2 (D = diag of the
# input column norms) the sparse step hard-thresholds W D, i.e. weight w_ij is
# ranked by |w_ij| * s_j.  The pins below check the oracle's fp32 score against
# exact arithmetic where the product is exact, against the weighted objective,
# and against the unscaled projection where the scale is uniform.

def _pow2_scales(rng, n, lo=-6, hi=7):
    return np.ldexp(1.0, rng.integers(lo, hi, size=n)).astype(np.float32)


def _bf16_scales(rng, n):
    """Positive scales with 8-bit significands, so |w| * s (bf16 w) is exact in fp32."""
    return synth.bf16_bits_to_f32(_bf16(rng.uniform(0.25, 4.0, size=n))).astype(np.float32)


def pin_scaled_uniform_equals_unscaled(o):
    """scale == c (any power of two, either sign) reduces to the plain 2:4 projection."""
    W = synth.gaussian_bf16((48, 128), 0.02, 21)
    v0, m0 = o.pack_2to4(W)
    for c in (1.0, 0.5, -8.0, 2.0 ** -20):
        v1, m1 = o.pack_2to4_scaled(W, np.full(128, c, dtype=np.float32))
        np.testing.assert_array_equal(v1, v0)
        np.testing.assert_array_equal(m1, m0)


def pin_scaled_bruteforce_exact(o, seed: int = 22):
    """Exact products (bf16 weights times 8-bit-significand scales) ranked by
    enumeration of the six pairs; the narrow weight alphabet makes many ties."""
    rng = np.random.Generator(np.random.PCG64(seed))
    d_in = 32
    sign = rng.integers(0, 2, size=(200, d_in)).astype(np.uint16) << 15
    expo = rng.integers(125, 129, size=(200, d_in)).astype(np.uint16) << 7
    mant = rng.integers(0, 4, size=(200, d_in)).astype(np.uint16) << 5
    W = (sign | expo | mant).astype(np.uint16)
    for scale in (_pow2_scales(rng, d_in), _bf16_scales(rng, d_in), -_pow2_scales(rng, d_in, -2, 3)):
        vals, meta = o.pack_2to4_scaled(W, scale)
        score = np.abs(_f64(W)) * np.abs(scale.astype(np.float64))
        for i in range(W.shape[0]):
            pairs = decode_meta(meta[i], d_in // 4)
            for g in range(d_in // 4):
                a, b = brute_force_pair(score[i, 4 * g:4 * g + 4])
                assert pairs[g] == (a, b), (i, g, pairs[g], (a, b))
                assert vals[i, 2 * g] == W[i, 4 * g + a] and vals[i, 2 * g + 1] == W[i, 4 * g + b]


def pin_scaled_minimises_weighted_error(o, seed: int = 23):
    """The kept pair minimises the diagonal-Hessian error sum_j s_j^2 w_j^2 over
    the dropped positions of each group, among all six 2-of-4 masks (fp64,
    with slack for the fp32 rounding of the score)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    W = synth.gaussian_bf16((64, 64), 0.02, seed)
    scale = np.exp(rng.normal(0.0, 1.5, size=64)).astype(np.float32)
    vals, meta = o.pack_2to4_scaled(W, scale)
    S = _f64(o.unpack_2to4(vals, meta, 64))
    Wf, s2 = _f64(W), scale.astype(np.float64) ** 2
    for i in range(64):
        for g in range(16):
            w, ss = Wf[i, 4 * g:4 * g + 4], s2[4 * g:4 * g + 4]
            err = np.sum(ss * (w - S[i, 4 * g:4 * g + 4]) ** 2)
            best = min(np.sum([ss[p] * w[p] ** 2 for p in range(4) if p not in pair])
                       for pair in itertools.combinations(range(4), 2))
            assert err <= best * (1 + 2.0 ** -20) + 1e-300, (i, g, err, best)


def pin_scaled_hand_examples(o):
    """Worked by hand: weights 1,2,3,4 with scales 4,2,1,1/2 score 4,4,3,2
    (keep 0 and 1); scores 1,3,2,3 keep 1 and 3; an all-equal score keeps 0, 1."""
    W = _bf16([[1, 2, 3, 4, 1, 1, 1, 1, 2, 1, 1, 2, -3, 0.5, 2, -1]])
    scale = np.array([4, 2, 1, 0.5, 1, 3, 2, 3, 1, 2, 2, 1, -1, 8, -0.75, 2], dtype=np.float32)
    vals, meta = o.pack_2to4_scaled(W, scale)
    # group 3 scores 3, 4, 1.5, 2 -> keep 0, 1
    np.testing.assert_array_equal(vals, _bf16([[1, 2, 1, 1, 2, 1, -3, 0.5]]))
    assert int(meta[0, 0]) == ((0 | 1 << 2) | ((1 | 3 << 2) << 4))
    assert int(meta[0, 1]) == ((0 | 1 << 2) | ((0 | 1 << 2) << 4))
    # The unscaled projection of the same row differs in groups 0 and 3.
    v0, _ = o.pack_2to4(W)
    np.testing.assert_array_equal(v0[0, [0, 1, 6, 7]], _bf16([3, 4, -3, 2]))


def pin_scaled_specials(o):
    """Stated readings: a NaN score (NaN weight, or 0 times an infinite scale)
    ranks above every number; an infinite score ranks above every finite one;
    a zero scale makes all four scores +0, so the lower index wins."""
    W = np.array([[0x3F80, 0x7FC0, 0x4000, 0x4040,      # NaN weight kept with the 3
                   0x0000, 0x3F80, 0x4000, 0x4040,      # 0 * Inf = NaN, kept with the 3 (Inf)
                   0x4040, 0x4000, 0x3F80, 0xC080]],    # zero scales: keep positions 0, 1
                 dtype=np.uint16)
    scale = np.array([1, 1, 1, 1, np.inf, 1, 1, np.inf, 0, 0, 0, 0], dtype=np.float32)
    vals, meta = o.pack_2to4_scaled(W, scale)
    np.testing.assert_array_equal(vals, [[0x7FC0, 0x4040, 0x0000, 0x4040, 0x4040, 0x4000]])
    assert int(meta[0, 0]) == ((1 | 3 << 2) | ((0 | 3 << 2) << 4))
    assert int(meta[0, 1]) == (0 | 1 << 2)


def pin_scaled_group_locality(o, seed: int = 24):
    """A group's choice depends on its own four scales only, and on their ratios:
    multiplying one group's scales by a power of two changes nothing, and
    permuting groups (weights and scales together) permutes the output."""
    rng = np.random.Generator(np.random.PCG64(seed))
    W = synth.gaussian_bf16((16, 48), 0.02, seed)
    scale = np.exp(rng.normal(0.0, 1.0, size=48)).astype(np.float32)
    vals, meta = o.pack_2to4_scaled(W, scale)
    s2 = scale.copy()
    s2[8:12] *= 64.0
    s2[20:24] *= 2.0 ** -9
    v2, m2 = o.pack_2to4_scaled(W, s2)
    np.testing.assert_array_equal(v2, vals)
    np.testing.assert_array_equal(m2, meta)
    perm = rng.permutation(12)
    cols = (4 * perm[:, None] + np.arange(4)).reshape(-1)
    vp, mp = o.pack_2to4_scaled(W[:, cols], scale[cols])
    pv = (2 * perm[:, None] + np.arange(2)).reshape(-1)
    np.testing.assert_array_equal(vp, vals[:, pv])
    for i in range(16):
        assert decode_meta(mp[i], 12) == [decode_meta(meta[i], 12)[k] for k in perm]


def pin_column_norms(o):
    """Closed forms: a constant column c over M = 16 rows has norm 4|c|; a
    one-hot column has norm |x|; a 3-4-5 column has norm 5; random columns
    agree with the library 2-norm."""
    M = 16
    X = np.zeros((M, 8), dtype=np.uint16)
    X[:, 0] = _bf16([-1.5] * M)
    X[:, 1] = _bf16([2.0 ** -10] * M)
    X[5, 2] = _bf16([-7.0])[0]
    X[0, 3], X[9, 3] = _bf16([3.0, -4.0])
    X[:, 5] = _bf16(np.arange(M) - 7.5)
    X[:, 6] = 0x8000                                     # -0 everywhere
    X[:, 7] = _bf16(np.where(np.arange(M) % 2 == 0, 1.0, -1.0))
    n = o.column_norms(X)
    assert n[0] == 6.0 and n[1] == 4 * 2.0 ** -10 and n[2] == 7.0 and n[3] == 5.0
    assert n[4] == 0.0 and n[6] == 0.0 and n[7] == 4.0
    assert abs(n[5] - np.sqrt(np.sum((np.arange(M) - 7.5) ** 2))) <= 1e-15 * n[5]
    Xr = synth.gaussian_bf16((37, 24), 1.0, 25)
    np.testing.assert_allclose(o.column_norms(Xr), np.linalg.norm(_f64(Xr), axis=0), rtol=1e-14)
    assert o.column_norms(np.zeros((0, 5), dtype=np.uint16)).tolist() == [0.0] * 5


# --------------------------------------------------------------------------- 2:8 pins
#
# The 2:8 projection keeps the two largest magnitudes of each aligned group of
# eight (ties to the lower index); a 2:8 matrix is also a 2:4 matrix.

_PAIRS8 = list(itertools.combinations(range(8), 2))


def brute_force_pairs8(absg: np.ndarray) -> np.ndarray:
    """For each row of ``absg`` [G, 8], the lexicographically first pair (a, b)
    whose kept magnitudes are all >= every dropped one (enumeration of the 28
    pairs, vectorised over the groups).  Returns [G, 2]."""
    G = absg.shape[0]
    best = np.full((G, 2), -1, dtype=np.int64)
    for a, b in _PAIRS8:
        dropped = np.delete(absg, [a, b], axis=1).max(axis=1)
        ok = (np.minimum(absg[:, a], absg[:, b]) >= dropped) & (best[:, 0] < 0)
        best[ok] = (a, b)
    assert np.all(best >= 0)
    return best


def _check_pack28(W, vals, meta):
    d_out, d_in = W.shape
    G = d_in // 8
    absg = np.abs(_f64(W)).reshape(d_out * G, 8)
    want = brute_force_pairs8(absg)
    got = np.stack([meta.reshape(-1) & 7, meta.reshape(-1) >> 3], axis=1).astype(np.int64)
    np.testing.assert_array_equal(got, want)
    Wg = W.reshape(d_out * G, 8)
    idx = np.arange(d_out * G)
    np.testing.assert_array_equal(vals.reshape(-1, 2)[:, 0], Wg[idx, want[:, 0]])
    np.testing.assert_array_equal(vals.reshape(-1, 2)[:, 1], Wg[idx, want[:, 1]])


def pin_pack28_exhaustive_alphabet(o):
    """Every group of eight over {+0, -1, 1, 2} (4^8 groups, many ties)."""
    alpha = _bf16([0.0, -1.0, 1.0, 2.0])
    groups = np.array(list(itertools.product(range(4), repeat=8)), dtype=np.int64)
    W = alpha[groups].reshape(-1, 64)               # eight groups per row
    vals, meta = o.pack_2to8(W)
    _check_pack28(W, vals, meta)


def pin_pack28_random_bruteforce(o, seed: int = 61):
    rng = np.random.Generator(np.random.PCG64(seed))
    sign = rng.integers(0, 2, size=(200, 48)).astype(np.uint16) << 15
    expo = rng.integers(125, 129, size=(200, 48)).astype(np.uint16) << 7
    mant = rng.integers(0, 4, size=(200, 48)).astype(np.uint16) << 5
    W = (sign | expo | mant).astype(np.uint16)
    vals, meta = o.pack_2to8(W)
    _check_pack28(W, vals, meta)
    Wg = synth.gaussian_bf16((64, 256), 0.02, seed)
    v2, m2 = o.pack_2to8(Wg)
    _check_pack28(Wg, v2, m2)


def pin_pack28_hand_and_specials(o):
    """Worked by hand: |1 5 3 -7 2 0 6 4| keeps -7 (3) and 6 (6); all zeros keep
    positions 0 and 1; NaN above Inf above finite; equal magnitudes of either
    sign tie and go to the lower index."""
    W = np.concatenate([_bf16([[1, 5, 3, -7, 2, 0, 6, 4, 0, 0, 0, 0, 0, 0, 0, 0]]),
                        np.array([[0x3F80, 0x7F80, 0x4000, 0x7FC0, 0, 0, 0, 0,
                                   0xBF80, 0x3F80, 0x3F80, 0xBF80, 0x3F80, 0, 0, 0]], dtype=np.uint16)], axis=1)
    vals, meta = o.pack_2to8(W)
    np.testing.assert_array_equal(meta, [[3 | 6 << 3, 0 | 1 << 3, 1 | 3 << 3, 0 | 1 << 3]])
    np.testing.assert_array_equal(vals, np.concatenate([_bf16([[-7, 6, 0, 0]]),
                                                       [[0x7F80, 0x7FC0, 0xBF80, 0x3F80]]], axis=1))


def pin_pack28_is_2to4(o):
    """A 2:8 matrix packs losslessly as 2:4, and the kept positions of each
    group of eight are among the 2:4 choices of their half-groups."""
    W = synth.gaussian_bf16((48, 192), 0.02, 62)
    v8, m8 = o.pack_2to8(W)
    S8 = o.unpack_2to8(v8, m8, 192)
    assert np.all(np.count_nonzero(S8.reshape(48, -1, 4) & 0x7FFF, axis=2) <= 2)
    v4, m4 = o.as_2to4(v8, m8, 192)
    np.testing.assert_array_equal(o.unpack_2to4(v4, m4, 192), S8)
    _, mw = o.pack_2to4(W)
    for i in range(48):
        pairs4 = decode_meta(mw[i], 48)
        for g in range(24):
            a, b = int(m8[i, g]) & 7, int(m8[i, g]) >> 3
            for p in (a, b):
                assert p % 4 in pairs4[2 * g + p // 4], (i, g, p)
    # Idempotent on its own output.
    v8b, m8b = o.pack_2to8(S8)
    np.testing.assert_array_equal(v8b, v8)
    np.testing.assert_array_equal(m8b, m8)


def pin_forward_2to8_identity(o):
    """X S8^T + (X V^T) U^T with small integers, exactly, through the 2:4 packing."""
    X, W, U, V = _small_int_problem(63, 6, 10, 32, 3)
    v8, m8 = o.pack_2to8(W)
    S = _f64(o.unpack_2to8(v8, m8, 32))
    Xf = _f64(X)
    Y, B = o.forward_2to8(X, v8, m8, U, V)
    np.testing.assert_array_equal(Y, Xf @ S.T + (Xf @ _f64(V).T) @ _f64(U).T)
    np.testing.assert_array_equal(B, np.abs(Xf) @ np.abs(S + _f64(U) @ _f64(V)).T)


ALL_PINS = [
    pin_pack_golden, pin_pack_exhaustive_alphabet, pin_pack_random_bruteforce,
    pin_pack_invariants, pin_pack_roundtrip, pin_pack_specials, pin_pack_odd_groups,
    pin_forward_golden, pin_forward_identity_exact, pin_forward_numpy, pin_forward_one_hot,
    pin_forward_sparse_only, pin_forward_row_subset, pin_lowrank_project,
    pin_scaled_uniform_equals_unscaled, pin_scaled_bruteforce_exact, pin_scaled_minimises_weighted_error,
    pin_scaled_hand_examples, pin_scaled_specials, pin_scaled_group_locality, pin_column_norms,
    pin_pack28_exhaustive_alphabet, pin_pack28_random_bruteforce, pin_pack28_hand_and_specials,
    pin_pack28_is_2to4, pin_forward_2to8_identity,
]


# --------------------------------------------------------------------------- alternating-minimisation pins
#
# These take the module oracle.datafree_am (or a planted-mistake copy of it).
# Pinned against: exact low-rank and diagonal cases of the truncation,
# brute force over random rank-r competitors (Eckart-Young), the C oracle's
# 2:4 projection on bf16-exact values and a brute-force pair choice, the
# monotone objective of exact block minimisation, and the degenerate cases
# r = 0, W of rank r, W already 2:4.

def pin_am_truncation_exact_cases(am):
    rng = np.random.Generator(np.random.PCG64(91))
    A = rng.integers(-3, 4, size=(30, 3)).astype(np.float64)
    B = rng.integers(-3, 4, size=(3, 20)).astype(np.float64)
    Z = A @ B                                       # rank <= 3
    np.testing.assert_allclose(am.truncated_svd(Z, 3), Z, atol=1e-10)
    np.testing.assert_allclose(am.truncated_svd(Z, 5), Z, atol=1e-10)
    D = np.zeros((6, 8))
    D[np.arange(6), np.arange(6)] = [1.0, -7.0, 3.0, 0.5, -4.0, 2.0]
    want = np.zeros_like(D)
    want[1, 1], want[4, 4] = -7.0, -4.0             # the two largest |singular values|
    np.testing.assert_allclose(am.truncated_svd(D, 2), want, atol=1e-12)
    assert np.all(am.truncated_svd(Z, 0) == 0)


def pin_am_truncation_beats_random(am):
    """Eckart-Young by brute force: no random rank-r matrix of the forms
    Z P (P a rank-r orthogonal projector) or A B (A, B least-squares fitted on
    random subspaces) comes closer to Z than C_r(Z)."""
    rng = np.random.Generator(np.random.PCG64(92))
    Z = rng.normal(size=(24, 16))
    for r in (1, 3, 6):
        best = np.linalg.norm(Z - am.truncated_svd(Z, r))
        assert np.linalg.matrix_rank(am.truncated_svd(Z, r), tol=1e-9) == r
        for _ in range(200):
            Q, _ = np.linalg.qr(rng.normal(size=(16, r)))
            assert np.linalg.norm(Z - Z @ Q @ Q.T) >= best - 1e-12
            P, _ = np.linalg.qr(rng.normal(size=(24, r)))
            assert np.linalg.norm(Z - P @ P.T @ Z) >= best - 1e-12


def pin_am_hard_threshold(am, seed: int = 93):
    """On bf16-exact values the 2:4 hard threshold keeps exactly the positions
    the C oracle's 2:4 projection keeps (ties included); on fp64 values the
    pair agrees with enumeration of the six pairs."""
    import oracle
    rng = np.random.Generator(np.random.PCG64(seed))
    sign = rng.integers(0, 2, size=(40, 32)).astype(np.uint16) << 15
    expo = rng.integers(125, 129, size=(40, 32)).astype(np.uint16) << 7
    mant = rng.integers(0, 4, size=(40, 32)).astype(np.uint16) << 5
    W = (sign | expo | mant).astype(np.uint16)
    vals, meta = oracle.pack_2to4(W)
    S_c = _f64(oracle.unpack_2to4(vals, meta, 32))
    np.testing.assert_array_equal(am.hard_threshold_2to4(_f64(W)), S_c)
    R = rng.normal(size=(30, 16))
    R[:, 4:8] = np.round(R[:, 4:8])                 # ties
    S = am.hard_threshold_2to4(R)
    for i in range(30):
        for g in range(4):
            a, b = brute_force_pair(np.abs(R[i, 4 * g:4 * g + 4]))
            kept = [p for p in range(4) if p in (a, b)]
            for p in range(4):
                assert S[i, 4 * g + p] == (R[i, 4 * g + p] if p in kept else 0.0)


def pin_am_monotone_objective(am):
    """Exact block minimisation: the objective never increases, and each P1
    and P2 step is optimal for its block (checked against perturbed blocks)."""
    rng = np.random.Generator(np.random.PCG64(94))
    W = rng.normal(size=(32, 24))
    S, L, objs = am.alternating_minimisation(W, 3, 6)
    assert len(objs) == 7
    assert all(b <= a + 1e-12 for a, b in zip(objs, objs[1:])), objs
    # Alternating improves on the initialisation (8.17 -> 5.59 here): the low-rank
    # block really is refitted to W - S.
    assert objs[-1] < 0.8 * objs[0], objs
    assert abs(objs[-1] - np.linalg.norm(W - S - L)) < 1e-12
    assert np.linalg.matrix_rank(L, tol=1e-9) <= 3
    assert np.all(np.count_nonzero(S.reshape(32, 6, 4), axis=2) <= 2)
    # P1 optimality: moving one kept position elsewhere in its group is worse.
    R = W - L
    base = np.linalg.norm(R - S)
    for (i, g) in [(0, 0), (5, 3), (31, 5)]:
        kept = [p for p in range(4) if S[i, 4 * g + p] != 0]
        drop = [p for p in range(4) if p not in kept]
        S2 = S.copy()
        S2[i, 4 * g + kept[0]] = 0.0
        S2[i, 4 * g + drop[0]] = R[i, 4 * g + drop[0]]
        assert np.linalg.norm(R - S2) >= base - 1e-12


def pin_am_degenerate_cases(am):
    rng = np.random.Generator(np.random.PCG64(95))
    W = rng.normal(size=(16, 12))
    S, L, objs = am.alternating_minimisation(W, 0, 3)           # r = 0: S = P1(W)
    assert np.all(L == 0)
    np.testing.assert_array_equal(S, am.hard_threshold_2to4(W))
    assert max(objs) - min(objs) < 1e-12
    A, B = rng.normal(size=(16, 2)), rng.normal(size=(2, 12))   # W of rank 2
    S, L, objs = am.alternating_minimisation(A @ B, 2, 2)
    assert objs[0] < 1e-10 and np.abs(S).max() < 1e-10
    S0 = am.hard_threshold_2to4(rng.normal(size=(16, 12)) * 10)  # W already 2:4, r = 1
    S, L, objs = am.alternating_minimisation(S0, 1, 8)
    assert all(b <= a + 1e-12 for a, b in zip(objs, objs[1:]))


AM_PINS = [pin_am_truncation_exact_cases, pin_am_truncation_beats_random, pin_am_hard_threshold,
           pin_am_monotone_objective, pin_am_degenerate_cases]


# --------------------------------------------------------------------------- LoRA backward pins
#
# These take the module oracle.lora_backward (or a planted-mistake copy).  The
# gradient is pinned by its definition: the loss <dY, Y> with Y from the C
# forward oracle is linear in U (and in V), so a central difference with
# small integer data is exact; plus independence from S and the bound.

def _lora_problem(seed, M=5, d_out=8, d_in=12, r=3):
    rng = np.random.Generator(np.random.PCG64(seed))
    X = _bf16(rng.integers(-3, 4, size=(M, d_in)))
    dY = _bf16(rng.integers(-3, 4, size=(M, d_out)))
    W = _bf16(rng.integers(-4, 5, size=(d_out, d_in)))
    U = _bf16(rng.integers(-2, 3, size=(d_out, r)))
    V = _bf16(rng.integers(-2, 3, size=(r, d_in)))
    return X, dY, W, U, V


def _loss(o, X, dY, vals, meta, U, V):
    Y, _ = o.forward(X, vals, meta, U, V)
    return float(np.sum(_f64(dY) * Y))


def pin_lora_finite_difference(lb):
    import oracle
    o = oracle.default()
    for seed, shape in [(101, (5, 8, 12, 3)), (102, (3, 16, 8, 2)), (103, (7, 4, 16, 5))]:
        X, dY, W, U, V = _lora_problem(seed, *shape)
        vals, meta = o.pack_2to4(W)
        dU, dV, _, _ = lb.lora_backward(X, dY, U, V)
        for (i, k) in [(0, 0), (shape[1] - 1, shape[3] - 1), (shape[1] // 2, 1 % shape[3])]:
            Up, Um = U.copy(), U.copy()
            Up[i, k] = _bf16([_f64(U[i:i + 1, k:k + 1])[0, 0] + 1.0])[0]
            Um[i, k] = _bf16([_f64(U[i:i + 1, k:k + 1])[0, 0] - 1.0])[0]
            fd = (_loss(o, X, dY, vals, meta, Up, V) - _loss(o, X, dY, vals, meta, Um, V)) / 2.0
            assert dU[i, k] == fd, (seed, i, k, dU[i, k], fd)
        for (k, j) in [(0, 0), (shape[3] - 1, shape[2] - 1), (1 % shape[3], shape[2] // 2)]:
            Vp, Vm = V.copy(), V.copy()
            Vp[k, j] = _bf16([_f64(V[k:k + 1, j:j + 1])[0, 0] + 1.0])[0]
            Vm[k, j] = _bf16([_f64(V[k:k + 1, j:j + 1])[0, 0] - 1.0])[0]
            fd = (_loss(o, X, dY, vals, meta, U, Vp) - _loss(o, X, dY, vals, meta, U, Vm)) / 2.0
            assert dV[k, j] == fd, (seed, k, j, dV[k, j], fd)


def pin_lora_shapes_bounds_and_s_independence(lb):
    import oracle
    o = oracle.default()
    X, dY, W, U, V = _lora_problem(104, 6, 8, 16, 4)
    dU, dV, BU, BV = lb.lora_backward(X, dY, U, V)
    assert dU.shape == (8, 4) and dV.shape == (4, 16)
    assert np.all(np.abs(dU) <= BU) and np.all(np.abs(dV) <= BV)
    # The gradient does not depend on S: the loss difference between two S is
    # constant in U, so finite differences through either S agree.
    v1, m1 = o.pack_2to4(W)
    v2, m2 = o.pack_2to4(_bf16(np.zeros((8, 16))))
    Up = U.copy()
    Up[3, 2] = _bf16([_f64(U[3:4, 2:3])[0, 0] + 1.0])[0]
    d1 = _loss(o, X, dY, v1, m1, Up, V) - _loss(o, X, dY, v1, m1, U, V)
    d2 = _loss(o, X, dY, v2, m2, Up, V) - _loss(o, X, dY, v2, m2, U, V)
    assert d1 == d2 == dU[3, 2]
    # Non-negative inputs: the bound is the gradient itself.
    Xa, dYa, Ua, Va = (_bf16(np.abs(_f64(a))) for a in (X, dY, U, V))
    dU2, dV2, BU2, BV2 = lb.lora_backward(Xa, dYa, Ua, Va)
    np.testing.assert_array_equal(dU2, BU2)
    np.testing.assert_array_equal(dV2, BV2)


LORA_PINS = [pin_lora_finite_difference, pin_lora_shapes_bounds_and_s_independence]

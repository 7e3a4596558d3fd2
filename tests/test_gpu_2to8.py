"""GPU parity of the 2:8 + low-rank layer (the 3BASiL summary page's 2:8 plus
rank-64 configuration) through the C ABI, against the fp64 oracle.

Projection: both packings (dense 2:8 and the 2:4 packing of the projected
matrix) bit-exact on configuration weights and adversarial bits, strided and
unaligned W.  Forward: the 2:8 streaming kernel and the 2:4 tensor-core path
on the 2:4 packing, under the same acceptance bounds as the 2:4 layer
(relative Frobenius <= 5e-3, per element <= 1e-2 (|X||W'|^T) + 1e-3), on
seeded samples at full size, for every token-block and rows-per-warp variant.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import check_forward, from_dev, sample_indices, to_dev, to_dev_u8

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sparse_rank_linear_02_b200 as slr


def _layer(cfg, name):
    return next(l for l in synth.CONFIGS[cfg].layers if l.name == name)


def _check_pack28(W, outs, rows):
    vals8, meta8, vals4, meta4 = outs
    Wr = np.ascontiguousarray(W[rows])
    v8, m8 = oracle.pack_2to8(Wr)
    np.testing.assert_array_equal(from_dev(vals8)[rows], v8)
    np.testing.assert_array_equal(meta8.cpu().numpy()[rows], m8)
    v4, m4 = oracle.as_2to4(v8, m8, W.shape[1])
    np.testing.assert_array_equal(from_dev(vals4)[rows], v4)
    np.testing.assert_array_equal(meta4.cpu().numpy()[rows], m4)


@pytest.mark.parametrize("cfg,name", [(1, "tiny"), (2, "q_proj"), (3, "gate_up"), (5, "up_proj_70b_r64"),
                                      (5, "down_proj_70b_r64")], ids=lambda x: str(x))
def test_pack_2to8_config_bit_exact(cfg, name):
    layer = _layer(cfg, name)
    W = layer.weight()
    outs = slr.pack_2to8(to_dev(W))
    torch.cuda.synchronize()
    rows = np.arange(layer.d_out) if layer.d_out * layer.d_in <= (1 << 24) else \
        sample_indices(layer.d_out, 384, seed=layer.d_out + 28)
    _check_pack28(W, outs, rows)


def _adversarial(seed, rows, cols):
    rng = np.random.Generator(np.random.PCG64(seed))
    W = rng.integers(0, 1 << 16, size=(rows, cols), dtype=np.uint32).astype(np.uint16)
    W[:, : cols // 4] &= 0x8000 | 0x3F80
    W[rows // 2:, cols // 2:] = rng.choice(np.array([0, 0x8000, 0x3F80, 0xBF80, 0x7F80, 0xFF80, 0x7FC0],
                                                    dtype=np.uint16), size=(rows - rows // 2, cols - cols // 2))
    W[0, :] = 0                      # all-zero groups keep positions 0 and 1
    return W


@pytest.mark.parametrize("rows,cols", [(64, 256), (33, 72), (5, 8), (128, 4104)])
def test_pack_2to8_adversarial_bit_exact(rows, cols):
    W = _adversarial(rows * 100 + cols, rows, cols)
    _check_pack28(W, slr.pack_2to8(to_dev(W)), np.arange(rows))


def test_pack_2to8_single_format_and_strided():
    big = _adversarial(5, 40, 272)
    Wd = to_dev(big)
    for lo, hi in [(0, 256), (8, 264), (4, 268), (1, 265)]:   # 16-byte aligned, 8-byte, 2-byte offsets
        W = np.ascontiguousarray(big[:, lo:hi])
        v8, m8, n4, n4m = slr.pack_2to8(Wd[:, lo:hi], as_2to4=False)
        assert n4 is None and n4m is None
        rv8, rm8 = oracle.pack_2to8(W)
        np.testing.assert_array_equal(from_dev(v8), rv8)
        np.testing.assert_array_equal(m8.cpu().numpy(), rm8)
        n8, n8m, v4, m4 = slr.pack_2to8(Wd[:, lo:hi], dense=False)
        assert n8 is None and n8m is None
        rv4, rm4 = oracle.as_2to4(rv8, rm8, hi - lo)
        np.testing.assert_array_equal(from_dev(v4), rv4)
        np.testing.assert_array_equal(m4.cpu().numpy(), rm4)


def _forward_case(layer, M, seed, k_rows=16, k_outs=384):
    """Pack on the GPU, run the 2:8 forward, and check sampled outputs against
    the oracle evaluated on the sampled output rows only (the oracle packs
    those rows of W itself; the GPU packing of them must match bit for bit)."""
    W = layer.weight()
    U, V = layer.factors()
    X = layer.activations(M)
    v8, m8, v4, m4 = slr.pack_2to8(to_dev(W))
    Y = slr.forward_2to8(to_dev(X), v8, m8, to_dev(U), to_dev(V))
    torch.cuda.synchronize()
    rows = sample_indices(M, k_rows, seed)
    outs = sample_indices(layer.d_out, k_outs, seed + 1)
    rv, rm = oracle.pack_2to8(np.ascontiguousarray(W[outs]))
    np.testing.assert_array_equal(from_dev(v8)[outs], rv)
    np.testing.assert_array_equal(m8.cpu().numpy()[outs], rm)
    Yref, Bref = oracle.forward_2to8(X, rv, rm, np.ascontiguousarray(U[outs]), V, rows=rows)
    check_forward(from_dev(Y)[np.ix_(rows, outs)], Yref, Bref, f"{layer.name} 2:8 M={M}", rows, outs)
    return W, U, V, v4, m4


@pytest.mark.parametrize("cfg,name,M", [(2, "q_proj", 1), (2, "q_proj", 2), (2, "q_proj", 3), (2, "q_proj", 16),
                                        (3, "gate_up", 1), (3, "gate_up", 2), (3, "gate_up", 5),
                                        (5, "up_proj_70b_r64", 1), (5, "down_proj_70b_r64", 2),
                                        (5, "up_proj_70b_r256", 1), (1, "tiny", 9)],
                         ids=lambda x: str(x))
def test_forward_2to8(cfg, name, M):
    _forward_case(_layer(cfg, name), M, seed=M * 31 + cfg)


@pytest.mark.parametrize("kernel", ["ring", "regs"])
@pytest.mark.parametrize("rw", ["1", "2", "4"])
def test_forward_2to8_rows_per_warp_variants(kernel, rw, monkeypatch):
    """Both kernels (shared-memory ring, registers), every rows-per-thread
    instantiation, on a shape with a ragged last row block (d_out = 4100) and
    every token-block size."""
    monkeypatch.setenv("SLR_DECODE28_RW", rw)
    monkeypatch.setenv("SLR_DECODE28_KERNEL", kernel)
    d_out, d_in, r = 4100, 1024, 64
    W = synth.gaussian_bf16((d_out, d_in), 0.02, 71)
    U = synth.gaussian_bf16((d_out, r), 0.5, 72)
    V = synth.gaussian_bf16((r, d_in), 0.5 / np.sqrt(d_in), 73)
    rv8, rm8 = oracle.pack_2to8(W)
    for M in (1, 2, 4, 7):
        X = synth.activations_bf16(M, d_in, 74 + M, None)
        Y = slr.forward_2to8(to_dev(X), to_dev(rv8), to_dev_u8(rm8), to_dev(U), to_dev(V))
        outs = sample_indices(d_out, 512, 75)
        Yref, Bref = oracle.forward_2to8(X, rv8, rm8, U, V, outs=outs)
        check_forward(from_dev(Y)[:, outs], Yref, Bref, f"rw={rw} M={M}", None, outs)


def test_forward_2to8_rank_variants_and_edges():
    """r = 0 (sparse term alone, exact small integers), r = 128 with 32 threads
    per row slot (ranks past 64 take the loop), d_in = 32 (register kernel: one
    chunk, most lanes idle), d_in = 1152 and 128 (ring, partial thread use),
    d_in = 16640 (ring, five segments of 3328 columns), M = 0."""
    rng = np.random.Generator(np.random.PCG64(81))
    d_out, d_in = 96, 64
    Wi = synth.f32_to_bf16_bits(rng.integers(-4, 5, size=(d_out, d_in)).astype(np.float32))
    Xi = synth.f32_to_bf16_bits(rng.integers(-3, 4, size=(3, d_in)).astype(np.float32))
    v8, m8 = oracle.pack_2to8(Wi)
    Y = slr.forward_2to8(to_dev(Xi), to_dev(v8), to_dev_u8(m8), None, None)
    S = synth.bf16_bits_to_f32(oracle.unpack_2to8(v8, m8, d_in)).astype(np.float64)
    exact = synth.bf16_bits_to_f32(Xi).astype(np.float64) @ S.T      # integers, exact in fp32
    np.testing.assert_array_equal(from_dev(Y), synth.f32_to_bf16_bits(exact.astype(np.float32)))
    for (d_out, d_in, r, M) in [(200, 256, 128, 2), (64, 32, 8, 1), (300, 32, 16, 4), (300, 1152, 64, 3),
                                (40, 128, 64, 1), (260, 16640, 64, 2)]:
        W = synth.gaussian_bf16((d_out, d_in), 0.05, d_out + d_in)
        U = synth.gaussian_bf16((d_out, r), 0.5, r + 1)
        V = synth.gaussian_bf16((r, d_in), 0.5 / np.sqrt(d_in), r + 2)
        X = synth.activations_bf16(M, d_in, M + 3, None)
        v8, m8 = oracle.pack_2to8(W)
        Y = slr.forward_2to8(to_dev(X), to_dev(v8), to_dev_u8(m8), to_dev(U), to_dev(V))
        Yref, Bref = oracle.forward_2to8(X, v8, m8, U, V)
        check_forward(from_dev(Y), Yref, Bref, f"{d_out}x{d_in} r={r} M={M}")
    empty = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    Y0 = slr.forward_2to8(empty, torch.zeros((8, 16), dtype=torch.bfloat16, device="cuda"),
                          torch.zeros((8, 8), dtype=torch.uint8, device="cuda"), None, None)
    assert Y0.shape == (0, 8)


def test_2to8_matrix_on_tensor_path():
    """The 2:4 packing of a 2:8 matrix runs on the 2:4 tensor-core forward
    (prefill, M = 2048) within the same bounds."""
    layer = _layer(3, "gate_up")
    W, U, V, v4, m4 = _forward_case(layer, 2, seed=5)
    M = 2048
    Xp = layer.activations(M)
    Y = slr.forward(to_dev(Xp), v4, m4, to_dev(U), to_dev(V), path="tensor")
    torch.cuda.synchronize()
    slr.check_kernel_error()
    rows = sample_indices(M, 24, 6)
    outs = sample_indices(layer.d_out, 256, 7)
    rv, rm = oracle.pack_2to8(np.ascontiguousarray(W[outs]))
    Yref, Bref = oracle.forward_2to8(Xp, rv, rm, np.ascontiguousarray(U[outs]), V, rows=rows)
    check_forward(from_dev(Y)[np.ix_(rows, outs)], Yref, Bref, "2:8 gate_up on the tensor path", rows, outs)


@pytest.mark.parametrize("M", [1, 4, 300])
def test_forward_2to8_routes_multi_token_calls_to_2to4(M):
    """Given both packings, forward_2to8 keeps one token on the 2:8 streaming
    kernel and sends more tokens to slr_forward on the 2:4 packing: the result
    is bit-identical to the matching direct call and within the oracle's
    bounds."""
    layer = _layer(2, "q_proj")
    W = layer.weight()
    U, V = layer.factors()
    X = layer.activations(M)
    v8, m8, v4, m4 = slr.pack_2to8(to_dev(W))
    args = (to_dev(X),)
    Y = slr.forward_2to8(args[0], v8, m8, to_dev(U), to_dev(V), vals4=v4, meta4=m4)
    if M == 1:
        direct = slr.forward_2to8(args[0], v8, m8, to_dev(U), to_dev(V))
    else:
        direct = slr.forward(args[0], v4, m4, to_dev(U), to_dev(V))
    torch.cuda.synchronize()
    slr.check_kernel_error()
    np.testing.assert_array_equal(from_dev(Y), from_dev(direct))
    rows = sample_indices(M, 16, 31)
    outs = sample_indices(layer.d_out, 256, 32)
    rv, rm = oracle.pack_2to8(np.ascontiguousarray(W[outs]))
    Yref, Bref = oracle.forward_2to8(X, rv, rm, np.ascontiguousarray(U[outs]), V, rows=rows)
    check_forward(from_dev(Y)[np.ix_(rows, outs)], Yref, Bref, f"2:8 routed M={M}", rows, outs)

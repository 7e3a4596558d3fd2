"""GPU parity: the CUDA library (through the C ABI) against the fp64 oracle.

Pack: bit-exact on every configuration shape and on adversarial inputs.
Forward: the acceptance bounds (relative Frobenius <= 5e-3, per element
|err| <= 1e-2 (|X||W'|^T) + 1e-3) on every configuration, on both execution
paths, on seeded samples of (token, output) pairs at full size (all pairs for
the small shapes), plus cases that isolate each term and the edge cases.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import (bits_to_f64, check_forward, from_dev, layer_activations, layer_weights,
                      sample_indices, to_dev, to_dev_u8)

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sparse_rank_linear_02_b200 as slr


def _shapes():
    seen, out = set(), []
    for c in synth.CONFIGS.values():
        for l in c.layers:
            if (l.d_out, l.d_in) not in seen:
                seen.add((l.d_out, l.d_in))
                out.append((c.cfg, l.name))
    return out


# ----------------------------------------------------------------------------- pack

@pytest.mark.parametrize("cfg,name", _shapes(), ids=lambda x: str(x))
def test_pack_config_bit_exact(cfg, name):
    layer, W, vals_ref, meta_ref, _, _ = layer_weights(cfg, name)
    vals, meta = slr.pack_2to4(to_dev(W))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(from_dev(vals), vals_ref)
    np.testing.assert_array_equal(meta.cpu().numpy(), meta_ref)


def _adversarial(seed, rows, cols):
    rng = np.random.Generator(np.random.PCG64(seed))
    W = rng.integers(0, 1 << 16, size=(rows, cols), dtype=np.uint32).astype(np.uint16)  # any bits, NaN too
    W[:, : cols // 4] &= 0x8000 | 0x3F80          # many +-1.0 / +-0 ties
    W[rows // 2:, cols // 2:] = rng.choice(np.array([0, 0x8000, 0x3F80, 0xBF80, 0x7F80, 0xFF80, 0x7FC0],
                                                    dtype=np.uint16), size=(rows - rows // 2, cols - cols // 2))
    return W


@pytest.mark.parametrize("rows,cols", [(64, 256), (33, 72), (5, 12), (7, 4), (128, 4100)])
def test_pack_adversarial_bit_exact(rows, cols):
    W = _adversarial(rows * 1000 + cols, rows, cols)
    vals_ref, meta_ref = oracle.pack_2to4(W)
    vals, meta = slr.pack_2to4(to_dev(W))
    np.testing.assert_array_equal(from_dev(vals), vals_ref)
    np.testing.assert_array_equal(meta.cpu().numpy(), meta_ref)


def test_pack_strided_and_unaligned():
    """ldw > d_in (a column slice of a wider matrix) and W pointers that are not
    16-byte aligned (8- and 2-byte offsets take the general kernel)."""
    big = _adversarial(99, 40, 264)
    Wd = to_dev(big)
    for lo, hi in [(0, 256), (4, 260), (1, 253)]:
        vals_ref, meta_ref = oracle.pack_2to4(np.ascontiguousarray(big[:, lo:hi]))
        vals, meta = slr.pack_2to4(Wd[:, lo:hi])
        np.testing.assert_array_equal(from_dev(vals), vals_ref)
        np.testing.assert_array_equal(meta.cpu().numpy(), meta_ref)


# ----------------------------------------------------------------------------- forward

def _forward_case(cfg, name, M, path, k_rows=48, k_outs=384):
    layer, W, vals, meta, U, V = layer_weights(cfg, name)
    X = layer_activations(cfg, name, M)
    Y = slr.forward(to_dev(X), to_dev(vals), to_dev_u8(meta), to_dev(U), to_dev(V), path=path)
    torch.cuda.synchronize()
    slr.check_kernel_error()
    rows = sample_indices(M, k_rows, seed=cfg * 7 + M)
    outs = sample_indices(layer.d_out, k_outs, seed=cfg * 11 + layer.d_out)
    Yref, Bref = oracle.forward(X, vals, meta, U, V, rows=rows, outs=outs)
    Yg = from_dev(Y)[np.ix_(rows, outs)]
    return check_forward(Yg, Yref, Bref, f"cfg{cfg} {name} M={M} path={path}", rows, outs)


def _cases():
    out = []
    for c in synth.CONFIGS.values():
        for l in c.layers:
            for M in c.Ms:
                out.append((c.cfg, l.name, M, "auto"))
    # the other path on the decode and prefill shapes
    for M in (1, 4, 16):
        out.append((2, "q_proj", M, "tensor"))
    out.append((1, "tiny", 8, "tensor"))
    out.append((3, "gate_up", 2048, "decode"))
    out.append((5, "up_proj_70b_r256", 128, "decode"))
    return out


@pytest.mark.parametrize("cfg,name,M,path", _cases(), ids=lambda x: str(x))
def test_forward_config(cfg, name, M, path):
    _forward_case(cfg, name, M, path)


def _lowrank_only(d_out, d_in, r, M, path, seed):
    """S = 0 and factors of unit scale: Y = (X V^T) U^T alone must meet the bounds
    (the configured factor scales make the low-rank term too small to see)."""
    X = synth.gaussian_bf16((M, d_in), 1.0, seed + 1)
    U = synth.gaussian_bf16((d_out, r), 1.0, seed + 2)
    V = synth.gaussian_bf16((r, d_in), 1.0 / np.sqrt(d_in), seed + 3)
    vals = np.zeros((d_out, d_in // 2), dtype=np.uint16)
    meta = np.full((d_out, d_in // 8), 0x44, dtype=np.uint8)
    Y = slr.forward(to_dev(X), to_dev(vals), to_dev_u8(meta), to_dev(U), to_dev(V), path=path)
    rows = sample_indices(M, 40, seed)
    outs = sample_indices(d_out, 300, seed + 5)
    Yref, Bref = oracle.forward(X, vals, meta, U, V, rows=rows, outs=outs)
    check_forward(from_dev(Y)[np.ix_(rows, outs)], Yref, Bref, f"lowrank-only {d_out}x{d_in} r={r} M={M} {path}",
                  rows, outs)


@pytest.mark.parametrize("path", ["decode", "tensor"])
@pytest.mark.parametrize("d_out,d_in,r,M", [(4096, 4096, 64, 16), (14336, 4096, 64, 300), (256, 256, 8, 8),
                                            (1024, 8192, 256, 130), (512, 1024, 128, 1)])
def test_forward_lowrank_only(d_out, d_in, r, M, path):
    _lowrank_only(d_out, d_in, r, M, path, seed=d_out + d_in + r + M)


@pytest.mark.parametrize("path", ["decode", "tensor"])
def test_forward_one_hot_exact(path):
    """U = 0 and X rows e_j: Y[m, :] = S[:, j] exactly (decodes the metadata of
    every column of every row; any index, order or layout slip changes bits)."""
    d_out, d_in = 384, 512
    W = synth.gaussian_bf16((d_out, d_in), 0.02, 5151)
    vals, meta = oracle.pack_2to4(W)
    S = oracle.unpack_2to4(vals, meta, d_in)
    X = np.zeros((d_in, d_in), dtype=np.uint16)
    X[np.arange(d_in), np.arange(d_in)] = 0x3F80
    U = np.zeros((d_out, 8), dtype=np.uint16)
    V = synth.gaussian_bf16((8, d_in), 1.0, 5152)
    Y = slr.forward(to_dev(X), to_dev(vals), to_dev_u8(meta), to_dev(U), to_dev(V), path=path)
    np.testing.assert_array_equal(bits_to_f64(from_dev(Y)), bits_to_f64(np.ascontiguousarray(S.T)))


@pytest.mark.parametrize("path", ["decode", "tensor"])
@pytest.mark.parametrize("d_out,d_in,r,M", [
    (200, 256, 16, 37),      # ragged output tile, ragged token tile
    (128, 128, 0, 1),        # one stage, no low-rank term
    (136, 384, 8, 129),      # r = 8 pads to the MMA K step; M just over a tile
    (256, 640, 128, 255),    # two rank steps on the tensor path
    (264, 1024, 256, 20),    # four rank steps; decode with several token blocks
    (256, 512, 264, 40),     # r > 256: the projection's persistent fallback, five rank steps
])
def test_forward_edges(d_out, d_in, r, M, path):
    seed = d_out * 31 + d_in + r + M
    X = synth.activations_bf16(M, d_in, seed, seed + 9)
    W = synth.gaussian_bf16((d_out, d_in), 0.02, seed + 1)
    vals, meta = oracle.pack_2to4(W)
    U = synth.gaussian_bf16((d_out, r), 0.5, seed + 2)
    V = synth.gaussian_bf16((r, d_in), 0.5 / np.sqrt(max(r, 1)), seed + 3)
    Y = slr.forward(to_dev(X), to_dev(vals), to_dev_u8(meta), to_dev(U) if r else None,
                    to_dev(V) if r else None, path=path)
    Yref, Bref = oracle.forward(X, vals, meta, U if r else None, V if r else None)
    check_forward(from_dev(Y), Yref, Bref, f"edge {d_out}x{d_in} r={r} M={M} {path}")


@pytest.mark.parametrize("d_out,d_in,r,M", [
    (4096, 4096, 64, 256),    # mid M: 256-row tiles, chunk cap below the kernel's maximum
    (4096, 4096, 64, 512),
    (1024, 4096, 64, 4096),   # few row tiles, many tokens
    (2048, 8192, 64, 1000),   # 512-row tiles, ragged token count
    (3072, 4096, 128, 700),   # d_out not a multiple of 512
    (4096, 14336, 64, 160),   # split-K kernel on two 128-token tiles, K split two ways (56 stages each)
    (1024, 8192, 128, 200),   # split-K kernel, four-way K split, two rank stages
    (8192, 4096, 64, 160),    # below 192 tokens: every pair-kernel kind is a candidate
    (4096, 4096, 64, 96),     # 65..128 tokens on 32 row tiles: split-K kernel, four-way split
])
def test_forward_plan_shapes(d_out, d_in, r, M):
    """Default dispatch on shapes where the pair-kernel plan choice matters
    (kernel kind, chunk-width cap, split or whole last round)."""
    seed = d_out + 3 * d_in + 5 * r + 7 * M
    X = synth.activations_bf16(M, d_in, seed, seed + 9)
    W = synth.gaussian_bf16((d_out, d_in), 0.02, seed + 1)
    vals, meta = oracle.pack_2to4(W)
    U = synth.gaussian_bf16((d_out, r), 0.5, seed + 2)
    V = synth.gaussian_bf16((r, d_in), 0.5 / np.sqrt(r), seed + 3)
    Y = slr.forward(to_dev(X), to_dev(vals), to_dev_u8(meta), to_dev(U), to_dev(V), path="tensor")
    torch.cuda.synchronize()
    slr.check_kernel_error()
    rows = sample_indices(M, 48, seed)
    outs = sample_indices(d_out, 512, seed + 1)
    Yref, Bref = oracle.forward(X, vals, meta, U, V, rows=rows, outs=outs)
    check_forward(from_dev(Y)[np.ix_(rows, outs)], Yref, Bref, f"plan {d_out}x{d_in} r={r} M={M}", rows, outs)


def test_forward_matches_between_paths():
    """The two paths agree with each other as well as with the oracle."""
    layer, W, vals, meta, U, V = layer_weights(2, "q_proj")
    X = layer_activations(2, "q_proj", 16)
    args = (to_dev(X), to_dev(vals), to_dev_u8(meta), to_dev(U), to_dev(V))
    Yd = bits_to_f64(from_dev(slr.forward(*args, path="decode")))
    Yt = bits_to_f64(from_dev(slr.forward(*args, path="tensor")))
    assert np.linalg.norm(Yd - Yt) / np.linalg.norm(Yd) < 5e-3


def test_no_kernel_timeouts():
    slr.check_kernel_error()


VARIANTS = ["1sm", "2sm128", "2sm240", "2sm256", "2smtall", "2smtallw", "2smtallk", "small"]


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("d_out,d_in,r,M", [
    (200, 256, 16, 37),      # ragged output rows (the pair's second CTA is partly outside d_out)
    (136, 384, 8, 129),      # r = 8; M just over a 128-token tile
    (512, 640, 128, 300),    # several pair tiles, two rank stages, ragged token tile
    (1024, 1024, 256, 513),  # four rank stages; more tiles than one wave of pairs
    (384, 512, 64, 5),       # small M: split K over a cluster, ragged token tile
    (1024, 2048, 128, 16),   # small M, 16-token tile, two rank stages
    (256, 4096, 64, 33),     # small M, 64-token tile
    (4096, 4096, 64, 1),     # one token, 32 row tiles x 4-CTA clusters
    (296, 1024, 64, 100),    # 65..128 tokens: one 128-token tile (split-K kernel), ragged rows
])
def test_forward_tensor_variants(variant, d_out, d_in, r, M, monkeypatch):
    """Every tensor-core kernel variant (1-SM; 2-SM pairs on 256-row tiles with
    chunks of up to 128 or 240 tokens; 2-SM pairs on 512-row tiles; the split-K
    small-M kernel) against the oracle, selected through SLR_TC_KERNEL."""
    monkeypatch.setenv("SLR_TC_KERNEL", variant)
    seed = d_out * 7 + d_in + r + M
    X = synth.activations_bf16(M, d_in, seed, seed + 9)
    W = synth.gaussian_bf16((d_out, d_in), 0.02, seed + 1)
    vals, meta = oracle.pack_2to4(W)
    U = synth.gaussian_bf16((d_out, r), 0.5, seed + 2)
    V = synth.gaussian_bf16((r, d_in), 0.5 / np.sqrt(r), seed + 3)
    Y = slr.forward(to_dev(X), to_dev(vals), to_dev_u8(meta), to_dev(U), to_dev(V), path="tensor")
    torch.cuda.synchronize()
    slr.check_kernel_error()
    rows = sample_indices(M, 64, seed)
    Yref, Bref = oracle.forward(X, vals, meta, U, V, rows=rows)
    check_forward(from_dev(Y)[rows], Yref, Bref, f"{variant} {d_out}x{d_in} r={r} M={M}", rows)


@pytest.mark.parametrize("variant", VARIANTS)
def test_forward_tensor_variants_prefill(variant, monkeypatch):
    """The gate/up prefill shape (14336 x 4096, r = 64, M = 2048) on each variant."""
    monkeypatch.setenv("SLR_TC_KERNEL", variant)
    _forward_case(3, "gate_up", 2048, "tensor")


@pytest.mark.parametrize("variant", VARIANTS)
def test_forward_tensor_variants_one_hot(variant, monkeypatch):
    """Exact metadata decoding on each variant (U = 0, X = identity rows)."""
    monkeypatch.setenv("SLR_TC_KERNEL", variant)
    d_out, d_in = 640, 256
    W = synth.gaussian_bf16((d_out, d_in), 0.02, 6161)
    vals, meta = oracle.pack_2to4(W)
    S = oracle.unpack_2to4(vals, meta, d_in)
    X = np.zeros((d_in, d_in), dtype=np.uint16)
    X[np.arange(d_in), np.arange(d_in)] = 0x3F80
    U = np.zeros((d_out, 8), dtype=np.uint16)
    V = synth.gaussian_bf16((8, d_in), 1.0, 6162)
    Y = slr.forward(to_dev(X), to_dev(vals), to_dev_u8(meta), to_dev(U), to_dev(V), path="tensor")
    np.testing.assert_array_equal(bits_to_f64(from_dev(Y)), bits_to_f64(np.ascontiguousarray(S.T)))


@pytest.mark.parametrize("d_out,d_in,r,M", [
    (1000, 8192, 64, 250),    # 4 tiles over 32 pairs: 8 K slices of 8 stages, ragged rows and tokens
    (1024, 8192, 128, 256),   # two rank stages in slice 0, projection phase at r = 128
    (2048, 4096, 256, 700),   # r > 128: T from the projection kernel, then the K-split kernel
    (14336, 4096, 8, 2048),   # the gate/up shape: whole rounds, then 2-3 slices per tail tile
    (2048, 28672, 64, 512),   # long K: 12 tiles, 6-7 slices of 32-37 stages each
])
def test_forward_ksplit_tail(d_out, d_in, r, M, monkeypatch):
    """The 512-row kernel with its last round split along K (SLR_TC_KERNEL=
    2smtallk): each slice's fp32 partial tile, the fixed-order reduction and
    the direct bf16 store, every element (or every output of sampled tokens)
    against the oracle, and the output bit-identical on a second call."""
    monkeypatch.setenv("SLR_TC_KERNEL", "2smtallk")
    seed = d_out + d_in + r + M + 77
    X, vals, meta, U, V = _layer_case(d_out, d_in, r, M, seed)
    args = (to_dev(X), to_dev(vals), to_dev_u8(meta), to_dev(U), to_dev(V))
    Y1 = slr.forward(*args, path="tensor")
    Y2 = slr.forward(*args, path="tensor")
    torch.cuda.synchronize()
    slr.check_kernel_error()
    b1, b2 = from_dev(Y1), from_dev(Y2)
    np.testing.assert_array_equal(b1, b2)
    rows = np.arange(M) if M * d_out <= 2_000_000 else sample_indices(M, 48, seed)
    Yref, Bref = oracle.forward(X, vals, meta, U, V, rows=rows)
    check_forward(b1[rows], Yref, Bref, f"K-split {d_out}x{d_in} r={r} M={M}", rows)


# ----------------------------------------------------------------------------- chained launches

def _layer_case(d_out, d_in, r, M, seed, outliers=True):
    X = synth.activations_bf16(M, d_in, seed, seed + 9 if outliers else None)
    W = synth.gaussian_bf16((d_out, d_in), 0.02, seed + 1)
    vals, meta = oracle.pack_2to4(W)
    U = synth.gaussian_bf16((d_out, r), 0.5, seed + 2)
    V = synth.gaussian_bf16((r, d_in), 0.5 / np.sqrt(max(r, 1)), seed + 3)
    return X, vals, meta, U, V


@pytest.mark.parametrize("path", ["decode", "tensor"])
@pytest.mark.parametrize("d_out,d_in,r,M", [
    (4096, 4096, 64, 1), (4096, 4096, 64, 4), (4096, 4096, 64, 16),   # q_proj decode
    (1024, 4096, 64, 16),     # 8 row tiles, K split four ways
    (3000, 2048, 128, 33),    # BN = 64, ragged last row tile
    (2048, 1024, 256, 64),    # four rank stages
    (1024, 2048, 0, 7),       # no projection: the combine itself is chained
    (28672, 8192, 64, 2),     # 224 row tiles, two CTAs per SM
])
def test_forward_chained_matches_unchained(path, d_out, d_in, r, M):
    """SLR_FWD_OVERLAP_PRECEDING changes when the kernels may start, not what
    they compute: bit-identical Y, and within the oracle's bounds."""
    seed = d_out + 7 * d_in + 11 * r + M
    X, vals, meta, U, V = _layer_case(d_out, d_in, r, M, seed)
    args = (to_dev(X), to_dev(vals), to_dev_u8(meta), to_dev(U) if r else None, to_dev(V) if r else None)
    Y0 = slr.forward(*args, path=path)
    Y1 = slr.forward(*args, path=path, overlap_preceding=True)
    torch.cuda.synchronize()
    slr.check_kernel_error()
    assert torch.equal(Y0.view(torch.int16), Y1.view(torch.int16))
    rows = sample_indices(M, 16, seed)
    outs = sample_indices(d_out, 512, seed + 1)
    Yref, Bref = oracle.forward(X, vals, meta, U if r else None, V if r else None, rows=rows, outs=outs)
    check_forward(from_dev(Y1)[np.ix_(rows, outs)], Yref, Bref, f"chained {d_out}x{d_in} r={r} M={M} {path}",
                  rows, outs)


@pytest.mark.parametrize("path", ["decode", "tensor"])
@pytest.mark.parametrize("M", [1, 16])
def test_forward_chained_dependent_layers(path, M):
    """Eight square layers back to back, each reading the previous layer's Y as
    its X and sharing one workspace, all queued as chained calls: identical
    bits to the same sequence without the flag (a kernel that read X or the
    workspace before the previous layer finished would differ)."""
    d = 4096
    layers = []
    for l in range(8):
        W = synth.gaussian_bf16((d, d), 0.05, 900 + l)
        vals, meta = oracle.pack_2to4(W)
        U = synth.gaussian_bf16((d, 64), 0.05, 950 + l)
        V = synth.gaussian_bf16((64, d), 0.05, 970 + l)
        layers.append((to_dev(vals), to_dev_u8(meta), to_dev(U), to_dev(V)))
    X0 = to_dev(synth.activations_bf16(M, d, 990, None))
    ws = torch.empty(max(slr.workspace_size(M, d, d, 64), 256), dtype=torch.uint8, device="cuda")

    def run(chained):
        x = X0
        outs = []
        for vals, meta, U, V in layers:
            y = torch.empty((M, d), dtype=torch.bfloat16, device="cuda")
            slr.forward(x, vals, meta, U, V, path=path, out=y, workspace=ws, overlap_preceding=chained)
            outs.append(y)
            x = y
        torch.cuda.synchronize()
        return outs

    ref = run(False)
    for rep in range(3):
        got = run(True)
        for l, (a, b) in enumerate(zip(ref, got)):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16)), f"layer {l} differs (repeat {rep})"
    slr.check_kernel_error()

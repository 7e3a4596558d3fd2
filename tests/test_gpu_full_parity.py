"""Full-size forward parity on the configurations the benchmark times.

The acceptance bounds (relative Frobenius <= 5e-3; per element
|err| <= 1e-2 (|X||W'|^T) + 1e-3, with W' = S + U V in fp64: LoSparse,
section 3.2) are checked

* on every element of the dispatched gate/up prefill forward
  (14336 x 4096, r = 64, M = 2048 tokens), and
* on two slices of every layer of the seven-layer block (M = 4096) and of
  the 70B up/down layers for each rank (M = 128, 1024, 8192): all tokens
  against one output row drawn from every 128-row block, and all outputs
  against one token drawn from every 16-token unit.  Together the slices meet
  every (row tile, token unit) pair the kernels' work partitions produce,
  the ragged last ones included.
"""
import functools

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import check_forward, from_dev, stratified_indices, to_dev, to_dev_u8

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sparse_rank_linear_02_b200 as slr


@functools.lru_cache(maxsize=1)
def _packed(d_out, d_in, cfg, wsub):
    """Oracle-packed S of a layer shape (the rank variants of a shape share W)."""
    layer = next(l for l in synth.CONFIGS[cfg].layers if (l.d_out, l.d_in, l.wsub) == (d_out, d_in, wsub))
    return oracle.pack_2to4(layer.weight())


def _layer(cfg, name):
    return next(l for l in synth.CONFIGS[cfg].layers if l.name == name)


def _run(layer, M):
    vals, meta = _packed(layer.d_out, layer.d_in, layer.cfg, layer.wsub)
    U, V = layer.factors()
    X = layer.activations(M)
    Y = slr.forward(to_dev(X), to_dev(vals), to_dev_u8(meta), to_dev(U), to_dev(V))
    torch.cuda.synchronize()
    slr.check_kernel_error()
    return X, vals, meta, U, V, from_dev(Y)


def test_forward_gate_up_prefill_every_element():
    layer = _layer(3, "gate_up")
    X, vals, meta, U, V, Y = _run(layer, 2048)
    Yref, Bref = oracle.forward(X, vals, meta, U, V)
    check_forward(Y, Yref, Bref, "gate/up M=2048, every element")


def _slice_cases():
    out = [(4, l.name, 4096) for l in synth.CONFIGS[4].layers]
    for l in synth.CONFIGS[5].layers:
        for M in (128, 1024, 8192):
            out.append((5, l.name, M))
    return out


@pytest.mark.parametrize("cfg,name,M", _slice_cases(), ids=lambda x: str(x))
def test_forward_full_size_slices(cfg, name, M):
    layer = _layer(cfg, name)
    X, vals, meta, U, V, Y = _run(layer, M)
    seed = 97 * cfg + M + layer.d_out
    # every token against one output row of every 128-row block
    outs = stratified_indices(layer.d_out, 128, seed)
    Yref, Bref = oracle.forward(X, vals, meta, U, V, outs=outs)
    check_forward(Y[:, outs], Yref, Bref, f"cfg{cfg} {name} M={M}: all tokens", None, outs)
    # every output against one token of every 16-token unit
    rows = stratified_indices(M, 16, seed + 1)
    Yref, Bref = oracle.forward(X, vals, meta, U, V, rows=rows)
    check_forward(Y[rows], Yref, Bref, f"cfg{cfg} {name} M={M}: all outputs", rows, None)

"""The no-allocation small-M forward (slr_forward_decode_noalloc).

It serves callers that cannot allocate device memory where they run the layer
(an engine that owns the whole device heap, a decode loop that may not call
cudaMalloc): the rank-projection scratch lives in a fixed array inside the
library.  This file is named so that pytest collects it last; it must pass
both on its own in a fresh process and after the other tests.

Checks, through the C ABI, over a sequence of calls that share the array:
each call's Y is bit-identical to slr_forward_with_path on the decode path
(the same kernels, with the scratch in a caller workspace) and meets the
oracle's acceptance bounds.  The sequence starts with a call that fills the
whole array with large values, then alternates small and large problems
(one token, r = 0, M * r at the array's capacity), so a call that read
entries it had not written would see another call's values.  A problem
larger than the array is rejected without a launch.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import check_forward, from_dev, to_dev, to_dev_u8

pytestmark = pytest.mark.gpu

SLR_OK, SLR_ERR_WORKSPACE = 0, 4
MAX_T_ELEMS = 16384
P = ctypes.c_void_p


def _lib():
    import sparse_rank_linear_02_b200 as slr
    lib = slr.lib()
    f = lib.slr_forward_decode_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [P, ctypes.c_int64, P, P, ctypes.c_int64, ctypes.c_int64, P, P, ctypes.c_int64, P, P]
    return slr, lib


def _problem(d_out, d_in, r, M, seed, x_scale=1.0):
    X = synth.activations_bf16(M, d_in, seed, seed + 1)
    if x_scale != 1.0:
        X = synth.f32_to_bf16_bits(synth.bf16_bits_to_f32(X) * np.float32(x_scale))
    W = synth.gaussian_bf16((d_out, d_in), 0.02, seed + 2)
    U = synth.gaussian_bf16((d_out, r), 0.5, seed + 3)
    V = synth.gaussian_bf16((r, d_in), 0.5 / np.sqrt(max(r, 1)), seed + 4)
    vals, meta = oracle.pack_2to4(W)
    return X, vals, meta, U, V


def _ptr(t):
    return P(t.data_ptr()) if t is not None else None


def _call_pair(slr, lib, d_out, d_in, r, M, seed, x_scale=1.0):
    """Runs the no-allocation entry point and the workspace entry point on one
    problem; returns the host inputs and both outputs (bf16 bits)."""
    stream = torch.cuda.current_stream().cuda_stream
    X, vals, meta, U, V = _problem(d_out, d_in, r, M, seed, x_scale)
    Xd, vd, md = to_dev(X), to_dev(vals), to_dev_u8(meta)
    Ud, Vd = (to_dev(U), to_dev(V)) if r else (None, None)
    Y = torch.full((M, d_out), float("nan"), dtype=torch.bfloat16, device="cuda")
    st = lib.slr_forward_decode_noalloc(_ptr(Xd), M, _ptr(vd), _ptr(md), d_out, d_in, _ptr(Ud), _ptr(Vd), r,
                                        _ptr(Y), stream)
    assert st == SLR_OK
    ws_bytes = max(slr.workspace_size(M, d_out, d_in, r), 256)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    Y_ref = torch.full((M, d_out), float("nan"), dtype=torch.bfloat16, device="cuda")
    st = lib.slr_forward_with_path(_ptr(Xd), M, _ptr(vd), _ptr(md), d_out, d_in, _ptr(Ud), _ptr(Vd), r,
                                   _ptr(Y_ref), _ptr(ws), ws_bytes, 1, stream)
    assert st == SLR_OK
    torch.cuda.synchronize()
    return (X, vals, meta, U if r else None, V if r else None), from_dev(Y), from_dev(Y_ref)


def test_noalloc_matches_workspace_forward_and_oracle_on_consecutive_calls():
    slr, lib = _lib()
    # fills all MAX_T_ELEMS entries of the array with values ~1e3 times the
    # later problems' (X scaled by 1024)
    _call_pair(slr, lib, 512, 1024, 128, MAX_T_ELEMS // 128, 300, x_scale=1024.0)
    sequence = [
        (1024, 2048, 64, 1, 301),                    # one token
        (4096, 4096, 64, MAX_T_ELEMS // 64, 302),    # M * r at the capacity of the array
        (768, 1024, 0, 7, 303),                      # no low-rank term: the array is not used
        (2048, 1024, 128, 5, 304),                   # fewer entries than the previous call wrote
        (1024, 2048, 256, MAX_T_ELEMS // 256, 305),  # at capacity with the largest rank tile
        (640, 512, 8, 3, 306),
    ]
    for d_out, d_in, r, M, seed in sequence:
        (X, vals, meta, U, V), y, y_ref = _call_pair(slr, lib, d_out, d_in, r, M, seed)
        what = f"noalloc {d_out}x{d_in} r={r} M={M}"
        assert np.array_equal(y, y_ref), f"{what}: differs from slr_forward_with_path (decode path) in " \
                                         f"{int(np.sum(y != y_ref))} elements"
        Yref, Bref = oracle.forward(X, vals, meta, U, V)
        check_forward(y, Yref, Bref, what)


def test_noalloc_rejects_problems_larger_than_its_scratch():
    _, lib = _lib()
    fake = P(0x10000)
    for r in (8, 64, 256):
        M = MAX_T_ELEMS // r + 1
        # validation fails before the pointers are used or anything is launched
        st = lib.slr_forward_decode_noalloc(fake, M, fake, fake, 512, 512, fake, fake, r, fake, None)
        assert st == SLR_ERR_WORKSPACE

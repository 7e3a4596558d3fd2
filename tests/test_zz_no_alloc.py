"""The no-allocation small-M forward (slr_forward_decode_noalloc).

It serves callers that cannot allocate device memory where they run the layer
(an engine that owns the whole device heap, a decode loop that may not call
cudaMalloc): the rank-projection scratch lives in a fixed array inside the
library.  This file is named so that pytest collects it last; it must pass
both on its own in a fresh process and after the other tests.

Checks, through the C ABI: two calls in a row (different shapes, so stale
scratch from the first call would show) match slr_forward_with_path on the
decode path, within the same bounds the other forward tests use; and a
problem larger than the built-in scratch is rejected without a launch.
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


def _problem(d_out, d_in, r, M, seed):
    X = synth.activations_bf16(M, d_in, seed, seed + 1)
    W = synth.gaussian_bf16((d_out, d_in), 0.02, seed + 2)
    U = synth.gaussian_bf16((d_out, r), 0.5, seed + 3)
    V = synth.gaussian_bf16((r, d_in), 0.5 / np.sqrt(r), seed + 4)
    vals, meta = oracle.pack_2to4(W)
    return X, vals, meta, U, V


def _ptr(t):
    return P(t.data_ptr())


def test_noalloc_matches_workspace_forward_on_consecutive_calls():
    slr, lib = _lib()
    stream = torch.cuda.current_stream().cuda_stream
    for d_out, d_in, r, M, seed in [(1024, 2048, 64, 16, 301), (2048, 1024, 128, 5, 302)]:
        X, vals, meta, U, V = _problem(d_out, d_in, r, M, seed)
        Xd, vd, md, Ud, Vd = to_dev(X), to_dev(vals), to_dev_u8(meta), to_dev(U), to_dev(V)
        # existing entry point, decode path, with a caller workspace
        ws_bytes = slr.workspace_size(M, d_out, d_in, r)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        Y_ref = torch.empty((M, d_out), dtype=torch.bfloat16, device="cuda")
        st = lib.slr_forward_with_path(_ptr(Xd), M, _ptr(vd), _ptr(md), d_out, d_in, _ptr(Ud), _ptr(Vd), r,
                                       _ptr(Y_ref), _ptr(ws), ws_bytes, 1, stream)
        assert st == SLR_OK
        # the no-allocation entry point
        Y = torch.full((M, d_out), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = lib.slr_forward_decode_noalloc(_ptr(Xd), M, _ptr(vd), _ptr(md), d_out, d_in, _ptr(Ud), _ptr(Vd), r,
                                            _ptr(Y), stream)
        assert st == SLR_OK
        torch.cuda.synchronize()
        y_ref, y = from_dev(Y_ref), from_dev(Y)
        # same bounds as the other forward tests, with the oracle's |X||W'|^T
        _, B = oracle.forward(X, vals, meta, U, V)
        ref = synth.bf16_bits_to_f32(y_ref).astype(np.float64)
        check_forward(y, ref, B, f"noalloc vs slr_forward {d_out}x{d_in} r={r} M={M}")


def test_noalloc_rejects_problems_larger_than_its_scratch():
    _, lib = _lib()
    r = 256
    M = MAX_T_ELEMS // r + 1
    # validation fails before the pointers are used or anything is launched
    fake = P(0x10000)
    st = lib.slr_forward_decode_noalloc(fake, M, fake, fake, 512, 512, fake, fake, r, fake, None)
    assert st == SLR_ERR_WORKSPACE

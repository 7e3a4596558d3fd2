"""Failure detection on the GPU without a fault.

Every wait in the tensor-core kernels is bounded: when it expires the kernel
records a timeout in the library's error word, leaves its loops, frees what it
holds and returns, and slr_check_kernel_error() reports SLR_ERR_TIMEOUT.  The
self-test entry point makes such a wait run out on purpose (a barrier that
nothing completes, a limit of about a millisecond); these tests check that the
status reaches the host, that it is cleared once read, and that the context
still computes correct results afterwards.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import check_forward, from_dev, to_dev, to_dev_u8

pytestmark = pytest.mark.gpu

SLR_ERR_TIMEOUT = 7


def test_expired_wait_is_reported_then_cleared():
    import sparse_rank_linear_02_b200 as slr
    slr.check_kernel_error()                       # nothing pending before
    slr.selftest_wait_timeout(2_000_000)
    with pytest.raises(slr.SlrError) as info:
        slr.check_kernel_error()
    assert info.value.status == SLR_ERR_TIMEOUT
    slr.check_kernel_error()                       # read once, then clear


def test_context_usable_after_expired_wait():
    import sparse_rank_linear_02_b200 as slr
    slr.selftest_wait_timeout(1_000_000)
    with pytest.raises(slr.SlrError):
        slr.check_kernel_error()
    d_out, d_in, r, M = 512, 1024, 16, 40
    X = synth.activations_bf16(M, d_in, 411, 412)
    W = synth.gaussian_bf16((d_out, d_in), 0.02, 413)
    U = synth.gaussian_bf16((d_out, r), 0.5, 414)
    V = synth.gaussian_bf16((r, d_in), 0.5 / np.sqrt(r), 415)
    vals, meta = oracle.pack_2to4(W)
    Y = slr.forward(to_dev(X), to_dev(vals), to_dev_u8(meta), to_dev(U), to_dev(V), path="tensor")
    torch.cuda.synchronize()
    slr.check_kernel_error()
    Y_ref, B = oracle.forward(X, vals, meta, U, V)
    check_forward(from_dev(Y), Y_ref, B, "forward after an expired self-test wait")


def test_selftest_rejects_bad_limits():
    import sparse_rank_linear_02_b200 as slr
    for bad in (0, -5, 1 << 31):
        with pytest.raises(slr.SlrError) as info:
            slr.selftest_wait_timeout(bad)
        assert info.value.status == 8            # SLR_ERR_ARG

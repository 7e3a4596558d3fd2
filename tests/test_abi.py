"""C-ABI checks that need no GPU: the library loads, exports every function
that include/slr.h declares, and rejects bad arguments on the host before any
launch.  Fake pointer values are used only where validation fails before the
device is touched."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "slr.h")

import sparse_rank_linear_02_b200 as slr  # noqa: E402

OK, NULL, SHAPE, ALIGN, WORKSPACE, DEVICE, CUDA, TIMEOUT, ARG = range(9)
P = ctypes.c_void_p


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SLR_API\s+[\w\s\*]+?\b(slr_\w+)\s*\(", text)))


def test_header_declares_api():
    names = declared_functions()
    for n in ["slr_pack_2to4", "slr_forward", "slr_forward_workspace_size", "slr_status_string"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(slr.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings():
    for s in range(9):
        assert slr.lib().slr_status_string(s).decode().startswith("SLR_")
    assert slr.lib().slr_status_string(99) == b"SLR_ERR_UNKNOWN"


def test_meta_row_bytes_and_workspace():
    lib = slr.lib()
    assert lib.slr_meta_row_bytes(4096) == 512
    assert lib.slr_meta_row_bytes(12) == 2
    assert lib.slr_meta_row_bytes(4) == 1
    assert slr.workspace_size(16, 4096, 4096, 64) == 16 * 64 * 4
    # above 64 tokens: bf16 T, 1 KB of counters, the projection phase's partials
    # (r <= 128) and the K-split slots (one per pair of the device, 74 pairs on
    # 148 SMs, the size assumed without a GPU: 2 CTAs x 2 halves x 240 x 128 fp32)
    pairs = 74
    if torch.cuda.is_available():
        pairs = min(128, torch.cuda.get_device_properties(0).multi_processor_count // 2)
    ks = pairs * 2 * 2 * 240 * 128 * 4
    assert slr.workspace_size(2048, 14336, 4096, 64) == 2048 * 64 * 2 + 1024 + 128 * 256 * 64 * 4 + ks
    assert slr.workspace_size(2048, 14336, 4096, 128) == 2048 * 128 * 2 + 1024 + 128 * 256 * 128 * 4 + ks
    assert slr.workspace_size(2048, 14336, 4096, 256) == 2048 * 256 * 2 + 1024 + ks
    assert slr.workspace_size(8, 256, 256, 0) == 0
    assert slr.workspace_size(0, 256, 256, 8) == 0


def test_path_selection():
    assert slr.select_path(1, 4096, 4096, 64) == "decode"
    assert slr.select_path(2, 4096, 4096, 64) == "tensor"     # two tokens: the split-K tensor kernel
    assert slr.select_path(4, 4096, 4096, 64) == "tensor"
    assert slr.select_path(16, 4096, 4096, 64) == "tensor"
    assert slr.select_path(1, 28672, 8192, 64) == "tensor"     # large layer: tensor-core streaming
    assert slr.select_path(2048, 14336, 4096, 64) == "tensor"
    assert slr.select_path(2048, 100, 4096, 64) == "decode"   # d_out % 8 != 0


def _fwd(X=0x1000, M=16, vals=0x2000, meta=0x3000, d_out=256, d_in=256, U=0x4000, V=0x5000, r=8,
         Y=0x6000, ws=0x7000, ws_bytes=1 << 20, path=0):
    return slr.lib().slr_forward_with_path(P(X), M, P(vals), P(meta), d_out, d_in, P(U), P(V), r, P(Y),
                                           P(ws), ws_bytes, path, None)


def test_forward_argument_errors():
    assert _fwd(M=0, X=0, vals=0, meta=0, Y=0) == OK          # empty problem: no-op
    assert _fwd(M=-1) == SHAPE
    assert _fwd(r=-8) == SHAPE
    assert _fwd(X=0) == NULL
    assert _fwd(meta=0) == NULL
    assert _fwd(Y=0) == NULL
    assert _fwd(U=0) == NULL
    assert _fwd(V=0, r=8) == NULL
    assert _fwd(ws=0) == NULL
    assert _fwd(d_in=200) == SHAPE             # not a multiple of 128
    assert _fwd(d_in=0) == SHAPE
    assert _fwd(r=12) == SHAPE                 # not a multiple of 8
    assert _fwd(d_out=0) == SHAPE
    assert _fwd(d_out=100, path=2) == SHAPE    # tensor path needs d_out % 8 == 0
    assert _fwd(X=0x1008) == ALIGN
    assert _fwd(vals=0x2004) == ALIGN
    assert _fwd(meta=0x3001) == ALIGN
    assert _fwd(U=0x4002) == ALIGN
    assert _fwd(ws=0x7010) == ALIGN            # workspace needs 256-byte alignment
    assert _fwd(ws_bytes=16) == WORKSPACE
    assert _fwd(path=7) == ARG


def test_forward_rank_zero_needs_no_factors_or_workspace():
    # With r == 0 the factors and the workspace may be NULL; validation then
    # reaches the device check (which fails here only when there is no GPU).
    if torch.cuda.is_available():
        pytest.skip("would launch with fake pointers on a GPU machine")
    assert _fwd(U=0, V=0, r=0, ws=0, ws_bytes=0) == DEVICE


def test_valid_arguments_without_gpu_report_device_error():
    if torch.cuda.is_available():
        pytest.skip("would launch with fake pointers on a GPU machine")
    assert _fwd() == DEVICE
    lib = slr.lib()
    assert lib.slr_pack_2to4(P(0x1000), 4, 8, 8, P(0x2000), P(0x3000), None) == DEVICE


def test_pack_argument_errors():
    lib = slr.lib()
    assert lib.slr_pack_2to4(P(0x1000), 4, 6, 6, P(0x2000), P(0x3000), None) == SHAPE   # d_in % 4
    assert lib.slr_pack_2to4(P(0x1000), 4, 8, 4, P(0x2000), P(0x3000), None) == SHAPE   # ldw < d_in
    assert lib.slr_pack_2to4(P(0x1000), -1, 8, 8, P(0x2000), P(0x3000), None) == SHAPE
    assert lib.slr_pack_2to4(P(0), 4, 8, 8, P(0x2000), P(0x3000), None) == NULL
    assert lib.slr_pack_2to4(P(0x1000), 4, 8, 8, P(0), P(0x3000), None) == NULL
    assert lib.slr_pack_2to4(P(0), 0, 8, 8, P(0), P(0), None) == OK                    # empty


def test_selftest_wait_timeout_arguments():
    lib = slr.lib()
    assert lib.slr_selftest_wait_timeout(0, None) == ARG
    assert lib.slr_selftest_wait_timeout(-1, None) == ARG
    assert lib.slr_selftest_wait_timeout(1 << 31, None) == ARG
    if not torch.cuda.is_available():
        assert lib.slr_selftest_wait_timeout(1000, None) == DEVICE


def test_pack_scaled_argument_errors():
    lib = slr.lib()
    f = lib.slr_pack_2to4_scaled
    assert f(P(0x1000), 4, 6, 6, P(0x4000), P(0x2000), P(0x3000), None) == SHAPE   # d_in % 4
    assert f(P(0x1000), 4, 8, 4, P(0x4000), P(0x2000), P(0x3000), None) == SHAPE   # ldw < d_in
    assert f(P(0x1000), 4, 8, 8, P(0), P(0x2000), P(0x3000), None) == NULL         # scale
    assert f(P(0), 0, 8, 8, P(0), P(0), P(0), None) == OK                           # empty
    if not torch.cuda.is_available():
        assert f(P(0x1000), 4, 8, 8, P(0x4000), P(0x2000), P(0x3000), None) == DEVICE


def test_column_norms_argument_errors_and_workspace():
    lib = slr.lib()
    f = lib.slr_column_norms
    assert f(P(0x1000), 4, 12, 12, P(0x2000), None, P(0x3000), 1 << 20, None) == SHAPE  # d_in % 8
    assert f(P(0x1000), 4, 16, 8, P(0x2000), None, P(0x3000), 1 << 20, None) == SHAPE   # ldx < d_in
    assert f(P(0x1000), 4, 16, 20, P(0x2000), None, P(0x3000), 1 << 20, None) == SHAPE  # ldx % 8
    assert f(P(0x1000), -1, 16, 16, P(0x2000), None, P(0x3000), 1 << 20, None) == SHAPE
    assert f(P(0x1000), 4, 16, 16, P(0), None, P(0x3000), 1 << 20, None) == NULL       # sumsq
    assert f(P(0), 4, 16, 16, P(0x2000), None, P(0x3000), 1 << 20, None) == NULL       # X
    assert f(P(0x1008), 4, 16, 16, P(0x2000), None, P(0x3000), 1 << 20, None) == ALIGN  # X 16 B
    assert f(P(0x1000), 4, 16, 16, P(0x2004), None, P(0x3000), 1 << 20, None) == ALIGN  # sumsq 8 B
    assert f(P(0x1000), 4, 16, 16, P(0x2000), None, P(0x3000), 0, None) == WORKSPACE
    assert f(P(0), 4, 0, 0, P(0), None, P(0), 0, None) == OK                           # d_in == 0
    if not torch.cuda.is_available():
        assert f(P(0), 0, 16, 16, P(0x2000), P(0x4000), P(0), 0, None) == DEVICE     # M == 0: norms only
    ws = slr.column_norms_workspace_size
    assert ws(0, 4096) == 0 and ws(16, 0) == 0
    # 2048 tokens x 4096 columns: 16 strips; one wave of 888 CTAs wants 37 rows
    # per split, rounded up to 64: 32 splits.
    assert ws(2048, 4096) == 32 * 4096 * 4
    # Very tall batches cap a split at 512 rows.
    assert ws(1 << 20, 4096) == (1 << 20) // 512 * 4096 * 4


def test_pack_2to8_argument_errors():
    f = slr.lib().slr_pack_2to8
    a, b, c, d = P(0x2000), P(0x3000), P(0x4000), P(0x5000)
    assert f(P(0x1000), 4, 12, 12, a, b, c, d, None) == SHAPE          # d_in % 8
    assert f(P(0x1000), 4, 16, 8, a, b, c, d, None) == SHAPE           # ldw < d_in
    assert f(P(0x1000), 4, 16, 16, a, P(0), c, d, None) == NULL        # half a pair
    assert f(P(0x1000), 4, 16, 16, P(0), P(0), P(0), P(0), None) == NULL  # no output
    assert f(P(0), 4, 16, 16, a, b, None, None, None) == NULL          # W
    assert f(P(0x1000), 4, 16, 16, P(0x2002), b, None, None, None) == ALIGN   # vals8 4 B
    assert f(P(0x1000), 4, 16, 16, None, None, P(0x4004), d, None) == ALIGN   # vals4 8 B
    assert f(P(0), 0, 16, 16, a, b, None, None, None) == OK            # empty
    if not torch.cuda.is_available():
        assert f(P(0x1000), 4, 16, 16, a, b, c, d, None) == DEVICE


def test_forward_2to8_argument_errors():
    f = slr.lib().slr_forward_2to8
    x, v, m, u, vv, y, ws = (P(0x10000 * k) for k in range(1, 8))
    assert f(x, 0, None, None, 8, 64, None, None, 0, None, None, 0, None) == OK        # M == 0
    assert f(x, 1, v, m, 8, 48, u, vv, 8, y, ws, 1 << 20, None) == SHAPE               # d_in % 32
    assert f(x, 1, v, m, 8, 64, u, vv, 4, y, ws, 1 << 20, None) == SHAPE               # r % 8
    assert f(x, 1 << 18, v, m, 8, 64, u, vv, 8, y, ws, 1 << 30, None) == SHAPE         # M too large
    assert f(x, 1, P(0), m, 8, 64, u, vv, 8, y, ws, 1 << 20, None) == NULL
    assert f(x, 1, v, m, 8, 64, P(0), vv, 8, y, ws, 1 << 20, None) == NULL             # U with r > 0
    assert f(P(0x10008), 1, v, m, 8, 64, u, vv, 8, y, ws, 1 << 20, None) == ALIGN
    assert f(x, 2, v, m, 8, 64, u, vv, 8, y, ws, 16, None) == WORKSPACE
    if not torch.cuda.is_available():
        assert f(x, 1, v, m, 8, 64, u, vv, 8, y, ws, 1 << 20, None) == DEVICE
        assert f(x, 1, v, m, 8, 64, None, None, 0, y, None, 0, None) == DEVICE        # r == 0: no factors


def test_decompose_argument_errors():
    f = slr.lib().slr_decompose_datafree
    w, q, v, m, u, vv, ws = (P(0x10000 * k) for k in range(1, 8))
    big = 1 << 30
    assert f(w, 64, 64, 12, 1, 1, 1, q, v, m, u, vv, None, ws, big, None) == SHAPE     # r % 8
    assert f(w, 64, 60, 8, 1, 1, 1, q, v, m, u, vv, None, ws, big, None) == SHAPE     # d_in % 8
    assert f(w, 64, 64, 136, 1, 1, 1, q, v, m, u, vv, None, ws, big, None) == SHAPE   # r > 128
    assert f(w, 8, 64, 16, 1, 1, 1, q, v, m, u, vv, None, ws, big, None) == SHAPE     # r > d_out
    assert f(w, 64, 64, 8, -1, 1, 1, q, v, m, u, vv, None, ws, big, None) == ARG
    assert f(w, 64, 64, 8, 1, 0, 1, q, v, m, u, vv, None, ws, big, None) == ARG
    assert f(w, 64, 64, 8, 1, 1, 1, P(0), v, m, u, vv, None, ws, big, None) == NULL   # Q0
    assert f(w, 64, 64, 8, 1, 1, 1, q, v, m, u, vv, P(0x80004), ws, big, None) == ALIGN
    assert f(w, 64, 64, 8, 1, 1, 1, q, v, m, u, vv, None, ws, 16, None) == WORKSPACE
    need = slr.lib().slr_decompose_workspace_size(14336, 4096, 64)
    assert need >= 14336 * 4096 * 4
    if not torch.cuda.is_available():
        assert f(w, 64, 64, 8, 1, 1, 1, q, v, m, u, vv, None, ws, big, None) == DEVICE


def test_forward_ex_flags():
    f = slr.lib().slr_forward_ex
    x, v, m, u, vv, y, ws = (P(0x10000 * k) for k in range(1, 8))
    assert f(x, 1, v, m, 8, 128, u, vv, 8, y, ws, 1 << 20, 0, 2, None) == ARG      # unknown option bit
    assert f(x, 1, v, m, 8, 128, u, vv, 8, y, ws, 1 << 20, 7, 1, None) == ARG      # unknown path
    assert f(x, 1, v, m, 8, 100, u, vv, 8, y, ws, 1 << 20, 0, 1, None) == SHAPE    # d_in % 128
    if not torch.cuda.is_available():
        assert f(x, 1, v, m, 8, 128, u, vv, 8, y, ws, 1 << 20, 0, 1, None) == DEVICE


def test_decompose_factors_f32_argument_errors():
    f = slr.lib().slr_decompose_factors_f32
    ws, u, v = P(0x10000), P(0x20000), P(0x30000)
    big = 1 << 30
    assert f(ws, big, 64, 64, 12, u, v, None) == SHAPE       # r % 8
    assert f(ws, big, 64, 64, 136, u, v, None) == SHAPE      # r > 128
    assert f(None, big, 64, 64, 8, u, v, None) == NULL
    assert f(ws, big, 64, 64, 8, None, None, None) == NULL   # no output
    assert f(ws, big, 64, 64, 8, P(0x20004), v, None) == ALIGN
    assert f(ws, 16, 64, 64, 8, u, v, None) == WORKSPACE
    if not torch.cuda.is_available():
        assert f(ws, big, 64, 64, 8, u, None, None) == DEVICE


def test_lora_backward_argument_errors():
    f = slr.lib().slr_lora_backward
    x, dy, u, v, du, dv, ws = (P(0x10000 * k) for k in range(1, 8))
    big = 1 << 30
    assert f(x, 8, dy, 12, 64, u, v, 8, None, du, dv, ws, big, None) == SHAPE     # d_out % 8
    assert f(x, 8, dy, 16, 96, u, v, 8, None, du, dv, ws, big, None) == SHAPE     # d_in % 64
    assert f(x, 8, dy, 16, 64, u, v, 264, None, du, dv, ws, big, None) == SHAPE   # r > 256
    assert f(x, 8, dy, 16, 64, u, v, 8, None, P(0), dv, ws, big, None) == NULL
    assert f(x, 8, P(0), 16, 64, u, v, 8, None, du, dv, ws, big, None) == NULL
    assert f(x, 8, dy, 16, 64, u, v, 8, P(0x80008), du, dv, ws, big, None) == ALIGN   # T
    assert f(x, 8, dy, 16, 64, u, v, 8, None, du, dv, ws, 16, None) == WORKSPACE
    assert slr.lib().slr_lora_backward_workspace_size(2048, 64) == 4 * 2048 * 64
    if not torch.cuda.is_available():
        assert f(x, 8, dy, 16, 64, u, v, 8, None, du, dv, ws, big, None) == DEVICE
        assert f(None, 0, None, 16, 64, None, None, 8, None, du, dv, None, 0, None) == DEVICE   # M == 0 zero-fills

"""Python binding of libslr: the 2:4-sparse + low-rank linear layer on B200.

Argument marshalling only.  Every step of the computation runs in the CUDA
kernels of ``libslr.so`` (built in-tree by ``python
sparse_rank_linear_02_b200/build.py``); there is no fallback of any kind, and the
import fails if the library is missing.

Functions mirror the C ABI in ``include/slr.h``:

* ``pack_2to4(W) -> (vals, meta)``  -- ``slr_pack_2to4``
* ``pack_2to4_scaled(W, scale) -> (vals, meta)``  -- ``slr_pack_2to4_scaled``
* ``column_norms(X, sumsq=None) -> (norms, sumsq)``  -- ``slr_column_norms``
* ``pack_2to8(W, dense=True, as_2to4=True)``  -- ``slr_pack_2to8``
* ``forward_2to8(X, vals8, meta8, U, V) -> Y``  -- ``slr_forward_2to8``
* ``lora_backward(X, dY, U, V, T=None) -> (dU, dV)``  -- ``slr_lora_backward``
* ``decompose_datafree(W, r, iters, ...) -> (vals, meta, U, V, objective)``  --
  ``slr_decompose_datafree``
* ``forward(X, vals, meta, U, V) -> Y``  -- ``slr_forward`` /
  ``slr_forward_with_path`` / ``slr_forward_ex``
* ``workspace_size``, ``select_path``, ``check_kernel_error``

Tensors are torch CUDA tensors (torch only provides memory and the current
stream): bf16 for W, X, U, V, vals and Y, uint8 for meta.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libslr.so")

SLR_OK = 0
STATUS_NAMES = {0: "SLR_OK", 1: "SLR_ERR_NULL", 2: "SLR_ERR_SHAPE", 3: "SLR_ERR_ALIGN",
                4: "SLR_ERR_WORKSPACE", 5: "SLR_ERR_DEVICE", 6: "SLR_ERR_CUDA",
                7: "SLR_ERR_TIMEOUT", 8: "SLR_ERR_ARG"}
PATHS = {"auto": 0, "decode": 1, "tensor": 2}
PATH_NAMES = {v: k for k, v in PATHS.items()}


class SlrError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)} "
                         f"({_lib.slr_status_string(status).decode()})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with "
                          f"`python sparse_rank_linear_02_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    i64, p, sz, st = ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    lib.slr_status_string.restype = ctypes.c_char_p
    lib.slr_status_string.argtypes = [st]
    lib.slr_version.restype = ctypes.c_int
    lib.slr_pack_2to4.restype = st
    lib.slr_pack_2to4.argtypes = [p, i64, i64, i64, p, p, p]
    lib.slr_meta_row_bytes.restype = i64
    lib.slr_meta_row_bytes.argtypes = [i64]
    lib.slr_pack_2to4_scaled.restype = st
    lib.slr_pack_2to4_scaled.argtypes = [p, i64, i64, i64, p, p, p, p]
    lib.slr_pack_2to8.restype = st
    lib.slr_pack_2to8.argtypes = [p, i64, i64, i64, p, p, p, p, p]
    lib.slr_forward_2to8.restype = st
    lib.slr_forward_2to8.argtypes = [p, i64, p, p, i64, i64, p, p, i64, p, p, sz, p]
    lib.slr_decompose_datafree.restype = st
    lib.slr_decompose_datafree.argtypes = [p, i64, i64, i64, ctypes.c_int, ctypes.c_int, ctypes.c_int, p, p, p, p,
                                           p, p, p, sz, p]
    lib.slr_decompose_factors_f32.restype = st
    lib.slr_decompose_factors_f32.argtypes = [p, sz, i64, i64, i64, p, p, p]
    lib.slr_decompose_workspace_size.restype = sz
    lib.slr_decompose_workspace_size.argtypes = [i64, i64, i64]
    lib.slr_lora_backward.restype = st
    lib.slr_lora_backward.argtypes = [p, i64, p, i64, i64, p, p, i64, p, p, p, p, sz, p]
    lib.slr_lora_backward_workspace_size.restype = sz
    lib.slr_lora_backward_workspace_size.argtypes = [i64, i64]
    lib.slr_column_norms.restype = st
    lib.slr_column_norms.argtypes = [p, i64, i64, i64, p, p, p, sz, p]
    lib.slr_column_norms_workspace_size.restype = sz
    lib.slr_column_norms_workspace_size.argtypes = [i64, i64]
    lib.slr_forward.restype = st
    lib.slr_forward.argtypes = [p, i64, p, p, i64, i64, p, p, i64, p, p, sz, p]
    lib.slr_forward_with_path.restype = st
    lib.slr_forward_with_path.argtypes = [p, i64, p, p, i64, i64, p, p, i64, p, p, sz, st, p]
    lib.slr_forward_ex.restype = st
    lib.slr_forward_ex.argtypes = [p, i64, p, p, i64, i64, p, p, i64, p, p, sz, st, ctypes.c_uint32, p]
    lib.slr_forward_workspace_size.restype = sz
    lib.slr_forward_workspace_size.argtypes = [i64, i64, i64, i64]
    lib.slr_forward_select_path.restype = st
    lib.slr_forward_select_path.argtypes = [i64, i64, i64, i64]
    lib.slr_check_kernel_error.restype = st
    lib.slr_check_kernel_error.argtypes = []
    lib.slr_forward_project.restype = st
    lib.slr_forward_project.argtypes = [p, i64, p, i64, i64, i64, p, sz, st, p]
    lib.slr_forward_combine.restype = st
    lib.slr_forward_combine.argtypes = [p, i64, p, p, i64, i64, p, i64, p, p, sz, st, p]
    lib.slr_forward_decode_noalloc.restype = st
    lib.slr_forward_decode_noalloc.argtypes = [p, i64, p, p, i64, i64, p, p, i64, p, p]
    lib.slr_selftest_wait_timeout.restype = st
    lib.slr_selftest_wait_timeout.argtypes = [i64, p]
    i32 = ctypes.c_int32
    lib.slr_plan_check.restype = i64
    lib.slr_plan_check.argtypes = [i64, i64, i64, i64, i32, i32, i32, i32]
    return lib


_lib = _load()


PLAN_KERNELS = {"2sm128": 0, "2sm240": 1, "2smtall": 2, "2sm256": 3}
PLAN_TAILS = {"whole": 0, "tokens": 1, "k": 2}


def plan_check(M: int, d_out: int, d_in: int, r: int, kernel: str, tail: str, max_pairs: int,
               chunk_units: int = 0) -> int:
    """``slr_plan_check``: the number of violations in the pair kernels' work
    plan for this shape (0 = sound; host only, no device needed)."""
    return int(_lib.slr_plan_check(M, d_out, d_in, r, PLAN_KERNELS[kernel], PLAN_TAILS[tail], max_pairs,
                                   chunk_units))


def lib() -> ctypes.CDLL:
    """The loaded ``libslr.so`` (for direct C-ABI calls)."""
    return _lib


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(status: int, what: str):
    if status != SLR_OK:
        raise SlrError(status, what)


def meta_row_bytes(d_in: int) -> int:
    return int(_lib.slr_meta_row_bytes(d_in))


def pack_2to4(W: torch.Tensor) -> tuple[torch.Tensor, torch.Tensor]:
    """2:4 projection by magnitude and packing of bf16 ``W`` [d_out, d_in]."""
    if W.dtype != torch.bfloat16 or W.dim() != 2 or not W.is_cuda or W.stride(1) != 1:
        raise ValueError("W must be a 2-D CUDA bf16 tensor with unit column stride")
    d_out, d_in = W.shape
    vals = torch.empty((d_out, d_in // 2), dtype=torch.bfloat16, device=W.device)
    meta = torch.empty((d_out, meta_row_bytes(d_in)), dtype=torch.uint8, device=W.device)
    _check(_lib.slr_pack_2to4(_ptr(W), d_out, d_in, W.stride(0), _ptr(vals), _ptr(meta), _stream()),
           "slr_pack_2to4")
    return vals, meta


def pack_2to4_scaled(W: torch.Tensor, scale: torch.Tensor) -> tuple[torch.Tensor, torch.Tensor]:
    """Activation-aware 2:4 projection of bf16 ``W`` [d_out, d_in]: weights of
    column j ranked by |w| * |scale[j]| (fp32 ``scale`` [d_in])."""
    if W.dtype != torch.bfloat16 or W.dim() != 2 or not W.is_cuda or W.stride(1) != 1:
        raise ValueError("W must be a 2-D CUDA bf16 tensor with unit column stride")
    d_out, d_in = W.shape
    if scale.dtype != torch.float32 or scale.shape != (d_in,) or not scale.is_contiguous() or \
            scale.device != W.device:
        raise ValueError("scale must be a contiguous fp32 tensor of d_in elements on W's device")
    vals = torch.empty((d_out, d_in // 2), dtype=torch.bfloat16, device=W.device)
    meta = torch.empty((d_out, meta_row_bytes(d_in)), dtype=torch.uint8, device=W.device)
    _check(_lib.slr_pack_2to4_scaled(_ptr(W), d_out, d_in, W.stride(0), _ptr(scale), _ptr(vals), _ptr(meta),
                                     _stream()), "slr_pack_2to4_scaled")
    return vals, meta


def column_norms_workspace_size(M: int, d_in: int) -> int:
    return int(_lib.slr_column_norms_workspace_size(M, d_in))


def column_norms(X: torch.Tensor, sumsq: torch.Tensor | None = None, *, want_norms: bool = True,
                 workspace: torch.Tensor | None = None) -> tuple[torch.Tensor | None, torch.Tensor]:
    """Add the column sums of squares of bf16 ``X`` [M, d_in] to the fp64
    running sum ``sumsq`` (a new zero sum when None) and return
    ``(norms, sumsq)``, norms = fp32 sqrt(sumsq) (None unless ``want_norms``)."""
    if X.dtype != torch.bfloat16 or X.dim() != 2 or not X.is_cuda or (X.numel() > 0 and X.stride(1) != 1):
        raise ValueError("X must be a 2-D CUDA bf16 tensor with unit column stride")
    M, d_in = X.shape
    ldx = X.stride(0) if X.numel() > 0 else d_in
    if sumsq is None:
        sumsq = torch.zeros(d_in, dtype=torch.float64, device=X.device)
    elif sumsq.dtype != torch.float64 or sumsq.shape != (d_in,) or not sumsq.is_contiguous():
        raise ValueError("sumsq must be a contiguous fp64 tensor of d_in elements")
    norms = torch.empty(d_in, dtype=torch.float32, device=X.device) if want_norms else None
    need = column_norms_workspace_size(M, d_in)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=X.device)
    _check(_lib.slr_column_norms(_ptr(X), M, d_in, ldx, _ptr(sumsq), _ptr(norms), _ptr(workspace),
                                 workspace.numel(), _stream()), "slr_column_norms")
    return norms, sumsq


def pack_2to8(W: torch.Tensor, *, dense: bool = True, as_2to4: bool = True):
    """2:8 projection of bf16 ``W`` [d_out, d_in]: returns ``(vals8, meta8,
    vals4, meta4)``, the dense 2:8 packing and the 2:4 packing of the same
    projected matrix (an unrequested pair is ``None``)."""
    if W.dtype != torch.bfloat16 or W.dim() != 2 or not W.is_cuda or W.stride(1) != 1:
        raise ValueError("W must be a 2-D CUDA bf16 tensor with unit column stride")
    d_out, d_in = W.shape
    dev = W.device
    vals8 = torch.empty((d_out, d_in // 4), dtype=torch.bfloat16, device=dev) if dense else None
    meta8 = torch.empty((d_out, d_in // 8), dtype=torch.uint8, device=dev) if dense else None
    vals4 = torch.empty((d_out, d_in // 2), dtype=torch.bfloat16, device=dev) if as_2to4 else None
    meta4 = torch.empty((d_out, meta_row_bytes(d_in)), dtype=torch.uint8, device=dev) if as_2to4 else None
    _check(_lib.slr_pack_2to8(_ptr(W), d_out, d_in, W.stride(0), _ptr(vals8), _ptr(meta8), _ptr(vals4),
                              _ptr(meta4), _stream()), "slr_pack_2to8")
    return vals8, meta8, vals4, meta4


def forward_2to8(X: torch.Tensor, vals8: torch.Tensor, meta8: torch.Tensor, U: torch.Tensor | None,
                 V: torch.Tensor | None, *, out: torch.Tensor | None = None,
                 workspace: torch.Tensor | None = None, vals4: torch.Tensor | None = None,
                 meta4: torch.Tensor | None = None) -> torch.Tensor:
    """``Y = X @ S.T + (X @ V.T) @ U.T`` with S in the dense 2:8 packing.

    The 2:8 streaming kernel is issue-bound and only pays at one token; given
    the 2:4 packing of the same matrix (``vals4``, ``meta4`` from
    :func:`pack_2to8`), calls with more than one token run ``slr_forward`` on
    it instead (the same product: a 2:8 pattern is a 2:4 pattern)."""
    M, d_in = X.shape
    d_out = vals8.shape[0]
    r = 0 if U is None else U.shape[1]
    if M > 1 and vals4 is not None and meta4 is not None:
        return forward(X, vals4, meta4, U, V, out=out, workspace=workspace)
    if out is None:
        out = torch.empty((M, d_out), dtype=torch.bfloat16, device=X.device)
    need = workspace_size(M, d_out, d_in, r)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=X.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.slr_forward_2to8(_ptr(X), M, _ptr(vals8), _ptr(meta8), d_out, d_in, _ptr(U), _ptr(V), r,
                                 _ptr(out), _ptr(workspace), ws_bytes, _stream()), "slr_forward_2to8")
    return out


def lora_backward(X: torch.Tensor, dY: torch.Tensor, U: torch.Tensor, V: torch.Tensor,
                  T: torch.Tensor | None = None) -> tuple[torch.Tensor, torch.Tensor]:
    """Gradients of the layer w.r.t. U and V for upstream ``dY`` [M, d_out]:
    ``dU = dY^T (X V^T)`` (fp32 [d_out, r]), ``dV = (dY U)^T X`` (fp32 [r, d_in]).
    ``T`` is the forward's ``X V^T`` (bf16 [M, r]) if kept."""
    M, d_in = X.shape
    d_out = dY.shape[1]
    r = U.shape[1]
    dU = torch.empty((d_out, r), dtype=torch.float32, device=X.device)
    dV = torch.empty((r, d_in), dtype=torch.float32, device=X.device)
    need = int(_lib.slr_lora_backward_workspace_size(M, r))
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device=X.device)
    _check(_lib.slr_lora_backward(_ptr(X), M, _ptr(dY), d_out, d_in, _ptr(U), _ptr(V), r, _ptr(T), _ptr(dU),
                                  _ptr(dV), _ptr(ws), ws.numel(), _stream()), "slr_lora_backward")
    return dU, dV


def decompose_datafree(W: torch.Tensor, r: int, iters: int, *, power_first: int = 8, power: int = 2,
                       Q0: torch.Tensor | None = None, seed: int = 0, factors_f32: bool = False):
    """Data-free alternating minimisation W ~ S + U V (S 2:4, rank r): returns
    ``(vals, meta, U, V, objective)`` with ``objective`` an fp64 CUDA tensor of
    ``iters + 1`` values.  ``Q0`` (fp32 [d_in, r]) is the random start of the
    subspace iteration; by default a standard normal one from ``seed``.  With
    ``factors_f32`` the fp32 factors before their rounding to bf16
    (``slr_decompose_factors_f32``) are appended: ``(..., U32, V32)``."""
    if W.dtype != torch.bfloat16 or W.dim() != 2 or not W.is_cuda or not W.is_contiguous():
        raise ValueError("W must be a contiguous 2-D CUDA bf16 tensor")
    d_out, d_in = W.shape
    dev = W.device
    if Q0 is None:
        g = torch.Generator(device=dev)
        g.manual_seed(seed)
        Q0 = torch.randn((d_in, r), generator=g, device=dev, dtype=torch.float32)
    vals = torch.empty((d_out, d_in // 2), dtype=torch.bfloat16, device=dev)
    meta = torch.empty((d_out, meta_row_bytes(d_in)), dtype=torch.uint8, device=dev)
    U = torch.empty((d_out, r), dtype=torch.bfloat16, device=dev)
    V = torch.empty((r, d_in), dtype=torch.bfloat16, device=dev)
    obj = torch.empty(iters + 1, dtype=torch.float64, device=dev)
    need = int(_lib.slr_decompose_workspace_size(d_out, d_in, r))
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    _check(_lib.slr_decompose_datafree(_ptr(W), d_out, d_in, r, iters, power_first, power, _ptr(Q0), _ptr(vals),
                                       _ptr(meta), _ptr(U), _ptr(V), _ptr(obj), _ptr(ws), ws.numel(), _stream()),
           "slr_decompose_datafree")
    if not factors_f32:
        return vals, meta, U, V, obj
    U32 = torch.empty((d_out, r), dtype=torch.float32, device=dev)
    V32 = torch.empty((r, d_in), dtype=torch.float32, device=dev)
    _check(_lib.slr_decompose_factors_f32(_ptr(ws), ws.numel(), d_out, d_in, r, _ptr(U32), _ptr(V32), _stream()),
           "slr_decompose_factors_f32")
    return vals, meta, U, V, obj, U32, V32


def workspace_size(M: int, d_out: int, d_in: int, r: int) -> int:
    return int(_lib.slr_forward_workspace_size(M, d_out, d_in, r))


def select_path(M: int, d_out: int, d_in: int, r: int) -> str:
    return PATH_NAMES[int(_lib.slr_forward_select_path(M, d_out, d_in, r))]


FWD_OVERLAP_PRECEDING = 1


def forward(X: torch.Tensor, vals: torch.Tensor, meta: torch.Tensor, U: torch.Tensor | None,
            V: torch.Tensor | None, *, path: str = "auto", out: torch.Tensor | None = None,
            workspace: torch.Tensor | None = None, overlap_preceding: bool = False) -> torch.Tensor:
    """``Y = X @ S.T + (X @ V.T) @ U.T`` with S given packed by ``pack_2to4``.

    ``overlap_preceding`` sets ``SLR_FWD_OVERLAP_PRECEDING`` (``slr_forward_ex``):
    the call may start reading its weights while the kernel queued just before
    it is still running, which that kernel must not write."""
    M, d_in = X.shape
    d_out = vals.shape[0]
    r = 0 if U is None else U.shape[1]
    if out is None:
        out = torch.empty((M, d_out), dtype=torch.bfloat16, device=X.device)
    need = workspace_size(M, d_out, d_in, r)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=X.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    flags = FWD_OVERLAP_PRECEDING if overlap_preceding else 0
    _check(_lib.slr_forward_ex(_ptr(X), M, _ptr(vals), _ptr(meta), d_out, d_in, _ptr(U), _ptr(V), r,
                               _ptr(out), _ptr(workspace), ws_bytes, PATHS[path], flags, _stream()),
           "slr_forward")
    return out


def forward_project(X: torch.Tensor, V: torch.Tensor | None, d_out: int, workspace: torch.Tensor, *,
                    path: str = "auto") -> None:
    """Stage 1 of ``forward``: T = X V^T into ``workspace`` (``slr_forward_project``)."""
    M, d_in = X.shape
    r = 0 if V is None else V.shape[0]
    _check(_lib.slr_forward_project(_ptr(X), M, _ptr(V), d_out, d_in, r, _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), PATHS[path], _stream()),
           "slr_forward_project")


def forward_combine(X: torch.Tensor, vals: torch.Tensor, meta: torch.Tensor, U: torch.Tensor | None,
                    out: torch.Tensor, workspace: torch.Tensor | None, *, path: str = "auto") -> torch.Tensor:
    """Stage 2 of ``forward``: Y = X S^T + T U^T with T from ``workspace``."""
    M, d_in = X.shape
    d_out = vals.shape[0]
    r = 0 if U is None else U.shape[1]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.slr_forward_combine(_ptr(X), M, _ptr(vals), _ptr(meta), d_out, d_in, _ptr(U), r, _ptr(out),
                                    _ptr(workspace), ws_bytes, PATHS[path], _stream()),
           "slr_forward_combine")
    return out


NOALLOC_MAX_T_ELEMS = 16384


def forward_decode_noalloc(X: torch.Tensor, vals: torch.Tensor, meta: torch.Tensor, U: torch.Tensor | None,
                           V: torch.Tensor | None, out: torch.Tensor) -> torch.Tensor:
    """Small-M forward for callers that cannot allocate device memory
    (``slr_forward_decode_noalloc``): no workspace; the rank projection lives in
    a fixed array inside the library (M * r <= NOALLOC_MAX_T_ELEMS).  ``out``
    must be provided."""
    M, d_in = X.shape
    d_out = vals.shape[0]
    r = 0 if U is None else U.shape[1]
    _check(_lib.slr_forward_decode_noalloc(_ptr(X), M, _ptr(vals), _ptr(meta), d_out, d_in, _ptr(U), _ptr(V), r,
                                           _ptr(out), _stream()),
           "slr_forward_decode_noalloc")
    return out


def check_kernel_error() -> None:
    """Synchronise and raise if a tensor-core kernel reported a bounded-wait timeout."""
    _check(_lib.slr_check_kernel_error(), "slr_check_kernel_error")


def selftest_wait_timeout(limit_cycles: int = 2_000_000) -> None:
    """Launch the failure-detection self-test (``slr_selftest_wait_timeout``): a
    bounded wait that expires after ``limit_cycles`` SM cycles and records a
    timeout that the next :func:`check_kernel_error` raises."""
    _check(_lib.slr_selftest_wait_timeout(int(limit_cycles), _stream()), "slr_selftest_wait_timeout")

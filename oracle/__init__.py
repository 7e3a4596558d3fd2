"""CPU oracle for the 2:4-sparse + low-rank linear layer (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library in
``sparse_rank_linear_02_b200``) never does, and shares no code with it.

The arithmetic lives in ``slr_oracle.c`` (plain C, fp64, scalar loops); this
module compiles it with gcc and wraps it with ctypes.  Every function cites the
passage of the pages that defines it in the C file's header:

* ``pack_2to4`` -- HASSLE-free, section 4.1.1 (data-free sparse update is
  hard-thresholding) with the 2:4 pattern of the 3BASiL summary page;
* ``forward``   -- LoSparse, sections 3 and 3.2 (sparse and low-rank terms in
  parallel), evaluated as ``X @ (S + U @ V).T`` in fp64.

Arrays are numpy ``uint16`` bf16 bit patterns; results are ``float64``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "slr_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libslr_oracle.so")

_lock = threading.Lock()
_default = None


def compile_source(src_path: str, out_path: str) -> str:
    """Compile an oracle C source with gcc (no fast-math, no FP contraction)."""
    os.makedirs(os.path.dirname(out_path), exist_ok=True)
    tmp = out_path + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", src_path, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out_path)
    return out_path


def build(force: bool = False) -> str:
    """Compile ``slr_oracle.c`` into ``oracle/_build`` if it is missing or stale."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        compile_source(_SRC, _LIB_PATH)
    return _LIB_PATH


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"expected uint16 bf16 bit patterns, got {a.dtype}")
    return a


class Oracle:
    """ctypes view of one compiled oracle library."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        i64, p = ctypes.c_int64, ctypes.c_void_p
        lib.oracle_meta_row_bytes.restype = i64
        lib.oracle_meta_row_bytes.argtypes = [i64]
        lib.oracle_pack_2to4.restype = ctypes.c_int
        lib.oracle_pack_2to4.argtypes = [p, i64, i64, i64, p, p]
        lib.oracle_unpack_2to4.restype = ctypes.c_int
        lib.oracle_unpack_2to4.argtypes = [p, p, i64, i64, p]
        lib.oracle_forward.restype = ctypes.c_int
        lib.oracle_forward.argtypes = [p, i64, p, p, i64, i64, p, p, i64, p, i64, p, i64, p, p, ctypes.c_int]
        lib.oracle_lowrank_project.restype = ctypes.c_int
        lib.oracle_lowrank_project.argtypes = [p, i64, p, i64, i64, p]
        lib.oracle_max_threads.restype = ctypes.c_int
        lib.oracle_pack_2to4_scaled.restype = ctypes.c_int
        lib.oracle_pack_2to4_scaled.argtypes = [p, i64, i64, i64, p, p, p]
        lib.oracle_pack_2to8.restype = ctypes.c_int
        lib.oracle_pack_2to8.argtypes = [p, i64, i64, i64, p, p]
        lib.oracle_unpack_2to8.restype = ctypes.c_int
        lib.oracle_unpack_2to8.argtypes = [p, p, i64, i64, p]
        lib.oracle_column_norms.restype = ctypes.c_int
        lib.oracle_column_norms.argtypes = [p, i64, i64, p]
        self._lib = lib
        self.path = lib_path

    def meta_row_bytes(self, d_in: int) -> int:
        return int(self._lib.oracle_meta_row_bytes(d_in))

    def max_threads(self) -> int:
        return int(self._lib.oracle_max_threads())

    def pack_2to4(self, W: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
        """Project dense bf16 ``W`` [d_out, d_in] onto 2:4 and pack it.

        Returns ``(vals, meta)``: ``vals`` uint16 [d_out, d_in/2] (kept values
        in ascending index order), ``meta`` uint8 [d_out, ceil(d_in/8)].
        """
        W = _u16(W)
        d_out, d_in = W.shape
        vals = np.zeros((d_out, d_in // 2), dtype=np.uint16)
        meta = np.zeros((d_out, self.meta_row_bytes(d_in)), dtype=np.uint8)
        rc = self._lib.oracle_pack_2to4(_ptr(W), d_out, d_in, d_in, _ptr(vals), _ptr(meta))
        if rc != 0:
            raise ValueError(f"oracle_pack_2to4 rejected shape {W.shape} (rc={rc})")
        return vals, meta

    def pack_2to4_scaled(self, W: np.ndarray, scale: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
        """Activation-aware 2:4 projection: weights of column j ranked by the
        float32 product |w| * |scale[j]| (HASSLE-free, section 4.1.2, diagonal
        Hessian); same packed format as :meth:`pack_2to4`."""
        W = _u16(W)
        d_out, d_in = W.shape
        scale = np.ascontiguousarray(scale, dtype=np.float32).reshape(-1)
        if scale.shape[0] != d_in:
            raise ValueError("scale must hold one float per input column")
        vals = np.zeros((d_out, d_in // 2), dtype=np.uint16)
        meta = np.zeros((d_out, self.meta_row_bytes(d_in)), dtype=np.uint8)
        rc = self._lib.oracle_pack_2to4_scaled(_ptr(W), d_out, d_in, d_in, _ptr(scale), _ptr(vals), _ptr(meta))
        if rc != 0:
            raise ValueError(f"oracle_pack_2to4_scaled rejected shape {W.shape} (rc={rc})")
        return vals, meta

    def pack_2to8(self, W: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
        """2:8 projection by magnitude: (vals [d_out, d_in/4], meta [d_out, d_in/8]),
        meta byte = idx0 | idx1 << 3."""
        W = _u16(W)
        d_out, d_in = W.shape
        vals = np.zeros((d_out, d_in // 4), dtype=np.uint16)
        meta = np.zeros((d_out, d_in // 8), dtype=np.uint8)
        rc = self._lib.oracle_pack_2to8(_ptr(W), d_out, d_in, d_in, _ptr(vals), _ptr(meta))
        if rc != 0:
            raise ValueError(f"oracle_pack_2to8 rejected shape {W.shape} (rc={rc})")
        return vals, meta

    def unpack_2to8(self, vals: np.ndarray, meta: np.ndarray, d_in: int) -> np.ndarray:
        """Dense bf16 bits [d_out, d_in] of a 2:8 packing (+0 elsewhere)."""
        vals = _u16(vals)
        meta = np.ascontiguousarray(meta, dtype=np.uint8)
        d_out = vals.shape[0]
        S = np.zeros((d_out, d_in), dtype=np.uint16)
        if self._lib.oracle_unpack_2to8(_ptr(vals), _ptr(meta), d_out, d_in, _ptr(S)) != 0:
            raise ValueError("oracle_unpack_2to8 rejected its arguments")
        return S

    def as_2to4(self, vals8: np.ndarray, meta8: np.ndarray, d_in: int) -> tuple[np.ndarray, np.ndarray]:
        """The 2:4 packing of a 2:8 matrix (lossless: every half-group of four
        holds at most two of the kept positions)."""
        return self.pack_2to4(self.unpack_2to8(vals8, meta8, d_in))

    def forward_2to8(self, X, vals8, meta8, U, V, rows=None, outs=None):
        """Forward of a 2:8 layer: the forward of its 2:4 packing."""
        d_in = _u16(X).shape[1]
        vals, meta = self.as_2to4(vals8, meta8, d_in)
        return self.forward(X, vals, meta, U, V, rows=rows, outs=outs)

    def column_norms(self, X: np.ndarray) -> np.ndarray:
        """fp64 norms of the columns of bf16 ``X`` [M, d_in]."""
        X = _u16(X)
        M, d_in = X.shape
        out = np.zeros(d_in, dtype=np.float64)
        if self._lib.oracle_column_norms(_ptr(X), M, d_in, _ptr(out)) != 0:
            raise ValueError("oracle_column_norms rejected its arguments")
        return out

    def unpack_2to4(self, vals: np.ndarray, meta: np.ndarray, d_in: int) -> np.ndarray:
        """Dense bf16 bits [d_out, d_in] of a packed 2:4 matrix (zeros elsewhere)."""
        vals = _u16(vals)
        meta = np.ascontiguousarray(meta, dtype=np.uint8)
        d_out = vals.shape[0]
        S = np.zeros((d_out, d_in), dtype=np.uint16)
        rc = self._lib.oracle_unpack_2to4(_ptr(vals), _ptr(meta), d_out, d_in, _ptr(S))
        if rc != 0:
            raise ValueError("oracle_unpack_2to4 rejected its arguments")
        return S

    def forward(self, X, vals, meta, U, V, rows=None, outs=None, with_bound: bool = True,
                nthreads: int = 0):
        """fp64 ``Y = X @ (S + U @ V).T`` and the bound ``|X| @ |S + U @ V|.T``.

        ``rows`` selects token rows of X and ``outs`` output features (default:
        all of each).  ``U``/``V`` may be None (no low-rank term).  Returns
        ``(Y, B)`` as float64 [n_rows, n_outs]; ``B`` is None when
        ``with_bound`` is False.
        """
        X = _u16(X)
        vals = _u16(vals)
        meta = np.ascontiguousarray(meta, dtype=np.uint8)
        M, d_in = X.shape
        d_out = vals.shape[0]
        if U is None or V is None:
            U = np.zeros((d_out, 0), dtype=np.uint16)
            V = np.zeros((0, d_in), dtype=np.uint16)
        U = _u16(U)
        V = _u16(V)
        r = U.shape[1]
        if U.shape != (d_out, r) or V.shape != (r, d_in):
            raise ValueError(f"bad low-rank shapes U{U.shape} V{V.shape}")
        if rows is None:
            n, rows_arr = M, None
        else:
            rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
            n = rows_arr.shape[0]
        if outs is None:
            no, outs_arr = d_out, None
        else:
            outs_arr = np.ascontiguousarray(outs, dtype=np.int64)
            no = outs_arr.shape[0]
        Y = np.zeros((n, no), dtype=np.float64)
        B = np.zeros((n, no), dtype=np.float64) if with_bound else None
        rc = self._lib.oracle_forward(
            _ptr(X), M, _ptr(vals), _ptr(meta), d_out, d_in,
            _ptr(U) if r else None, _ptr(V) if r else None, r,
            _ptr(rows_arr) if rows_arr is not None else None, n,
            _ptr(outs_arr) if outs_arr is not None else None, no,
            _ptr(Y), _ptr(B) if B is not None else None, int(nthreads))
        if rc != 0:
            raise ValueError(f"oracle_forward failed (rc={rc})")
        return Y, B

    def lowrank_project(self, X, V) -> np.ndarray:
        """fp64 ``T = X @ V.T`` ([M, r])."""
        X = _u16(X)
        V = _u16(V)
        M, d_in = X.shape
        r = V.shape[0]
        T = np.zeros((M, r), dtype=np.float64)
        rc = self._lib.oracle_lowrank_project(_ptr(X), M, _ptr(V), d_in, r, _ptr(T))
        if rc != 0:
            raise ValueError("oracle_lowrank_project failed")
        return T


def default() -> Oracle:
    """The oracle built from ``slr_oracle.c`` (compiled on first use)."""
    global _default
    with _lock:
        if _default is None:
            _default = Oracle(build())
    return _default


def meta_row_bytes(d_in: int) -> int:
    return default().meta_row_bytes(d_in)


def max_threads() -> int:
    return default().max_threads()


def pack_2to4_scaled(W, scale):
    return default().pack_2to4_scaled(W, scale)


def column_norms(X):
    return default().column_norms(X)


def pack_2to8(W):
    return default().pack_2to8(W)


def unpack_2to8(vals, meta, d_in):
    return default().unpack_2to8(vals, meta, d_in)


def as_2to4(vals8, meta8, d_in):
    return default().as_2to4(vals8, meta8, d_in)


def forward_2to8(X, vals8, meta8, U, V, rows=None, outs=None):
    return default().forward_2to8(X, vals8, meta8, U, V, rows=rows, outs=outs)


def pack_2to4(W):
    return default().pack_2to4(W)


def unpack_2to4(vals, meta, d_in: int):
    return default().unpack_2to4(vals, meta, d_in)


def forward(X, vals, meta, U, V, rows=None, outs=None, with_bound: bool = True, nthreads: int = 0):
    return default().forward(X, vals, meta, U, V, rows=rows, outs=outs, with_bound=with_bound,
                             nthreads=nthreads)


def lowrank_project(X, V):
    return default().lowrank_project(X, V)

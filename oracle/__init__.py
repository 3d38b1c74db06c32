"""fp64 CPU oracle for the B-spline KAN layer (ctypes binding of kan_oracle.c).

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package.  It shares no code with
the CUDA path: the C source here is compiled on its own with gcc, and nothing
under ``kolmogorov_arnold_network_b200`` imports it.

What each function computes is stated in ``kan_oracle.c``: the textbook
Cox-de Boor recursion (named by the FlashKAN abstract on the mlsift "GPU
kernel" listing), the KAN layer sum of per-edge B-splines (InKAN landing page,
"What is a KAN?"), an optional SiLU base branch, and the gradients of that
layer, all in fp64 with ascending-order sums.

Every function has at least one pin in ``tests/test_oracle_pins.py``; none is
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kan_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_i64 = ctypes.c_int64


def build(force: bool = False, extra_flags: tuple = (), out_path: str | None = None) -> str:
    """Compile kan_oracle.c with gcc (IEEE fp64, no fast-math). Returns the .so path."""
    path = out_path or _LIB_PATH
    if not force and os.path.exists(path) and os.path.getmtime(path) >= os.path.getmtime(_SRC):
        return path
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-fno-fast-math",
           "-ffp-contract=off", *extra_flags, _SRC, "-o", path + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(path + ".tmp", path)
    return path


def _declare(lib):
    lib.kan_oracle_knots.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_double, _dp]
    lib.kan_oracle_knots.restype = None
    lib.kan_oracle_basis_many.argtypes = [_dp, _i64, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                          ctypes.c_double, _dp, _dp]
    lib.kan_oracle_basis_many.restype = None
    lib.kan_oracle_silu_many.argtypes = [_dp, _i64, _dp, _dp]
    lib.kan_oracle_silu_many.restype = None
    lib.kan_oracle_forward.argtypes = [_i64, _i64, _i64, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                       ctypes.c_double, _dp, _dp, _dp, _dp, ctypes.c_int]
    lib.kan_oracle_forward.restype = ctypes.c_int
    lib.kan_oracle_backward.argtypes = [_i64, _i64, _i64, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                        ctypes.c_double, _dp, _dp, _dp, _dp, _dp, _dp, _dp, ctypes.c_int]
    lib.kan_oracle_backward.restype = ctypes.c_int
    lib.kan_oracle_dense_basis.argtypes = [_i64, _i64, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                           ctypes.c_double, _dp, _dp]
    lib.kan_oracle_dense_basis.restype = None
    return lib


def load(path: str | None = None):
    """Load (building first if needed) the oracle library."""
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            _lib = _declare(ctypes.CDLL(build()))
    return _lib


def _f64(a) -> np.ndarray:
    """fp64 C-contiguous copy/view of an array-like (torch tensors included)."""
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_dp)


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


class Oracle:
    """Thin object wrapper so that a test can load a differently-built oracle."""

    def __init__(self, lib=None):
        self.lib = lib if lib is not None else load()

    def knots(self, G, lo, hi, k=3):
        t = np.empty(G + 2 * k + 1)
        self.lib.kan_oracle_knots(G, k, lo, hi, _ptr(t))
        return t

    def basis(self, x, G, lo, hi, k=3):
        """B[n, G+k], dB[n, G+k] for the flattened points x."""
        x = _f64(x).reshape(-1)
        B = np.empty((x.size, G + k))
        dB = np.empty((x.size, G + k))
        self.lib.kan_oracle_basis_many(_ptr(x), x.size, G, k, lo, hi, _ptr(B), _ptr(dB))
        return B, dB

    def silu(self, x):
        x = _f64(x).reshape(-1)
        y = np.empty_like(x)
        dy = np.empty_like(x)
        self.lib.kan_oracle_silu_many(_ptr(x), x.size, _ptr(y), _ptr(dy))
        return y, dy

    def dense_basis(self, x, G, lo, hi, k=3):
        x = _f64(x)
        batch, n_in = x.shape
        A = np.empty((batch, n_in * (G + k)))
        self.lib.kan_oracle_dense_basis(batch, n_in, G, k, lo, hi, _ptr(x), _ptr(A))
        return A

    def forward(self, x, coef, G, lo, hi, w_base=None, k=3, nthreads=None):
        x = _f64(x)
        coef = _f64(coef)
        batch, n_in = x.shape
        n_out = coef.shape[0]
        assert coef.shape == (n_out, n_in, G + k), coef.shape
        wb = None if w_base is None else _f64(w_base)
        if wb is not None:
            assert wb.shape == (n_out, n_in)
        y = np.zeros((batch, n_out))
        rc = self.lib.kan_oracle_forward(batch, n_in, n_out, G, k, lo, hi, _ptr(x), _ptr(coef), _ptr(wb),
                                         _ptr(y), nthreads or default_threads())
        if rc != 0:
            raise ValueError("kan_oracle_forward rejected its arguments")
        return y

    def backward(self, x, coef, dY, G, lo, hi, w_base=None, k=3, nthreads=None,
                 want_dx=True, want_dcoef=True, want_dw_base=True):
        x = _f64(x)
        coef = _f64(coef)
        dY = _f64(dY)
        batch, n_in = x.shape
        n_out = coef.shape[0]
        assert coef.shape == (n_out, n_in, G + k), coef.shape
        assert dY.shape == (batch, n_out)
        wb = None if w_base is None else _f64(w_base)
        dx = np.zeros((batch, n_in)) if want_dx else None
        dcoef = np.zeros((n_out, n_in, G + k)) if want_dcoef else None
        dwb = np.zeros((n_out, n_in)) if (want_dw_base and wb is not None) else None
        rc = self.lib.kan_oracle_backward(batch, n_in, n_out, G, k, lo, hi, _ptr(x), _ptr(coef), _ptr(wb),
                                          _ptr(dY), _ptr(dx), _ptr(dcoef), _ptr(dwb),
                                          nthreads or default_threads())
        if rc != 0:
            raise ValueError("kan_oracle_backward rejected its arguments")
        return dx, dcoef, dwb


_default = None


def get() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default

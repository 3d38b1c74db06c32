"""ctypes binding of libkan_b200.so (declared in include/kan_b200.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  The library must exist (``python -m kolmogorov_arnold_network_b200.build``);
there is no fallback of any kind when it does not.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkan_b200.so")

KAN_F32, KAN_BF16 = 0, 1
KAN_PATH_AUTO, KAN_PATH_TENSOR, KAN_PATH_SIMT = 0, 1, 2
STATUS = {0: "KAN_OK", 1: "KAN_ERR_INVALID_ARG", 2: "KAN_ERR_UNSUPPORTED", 3: "KAN_ERR_WORKSPACE",
          4: "KAN_ERR_CUDA", 5: "KAN_ERR_TIMEOUT", 6: "KAN_ERR_DEVICE_CHECK"}

#: every symbol the header declares
EXPORTS = ("kan_abi_version", "kan_workspace_size", "kan_forward", "kan_backward", "kan_basis", "kan_sync_status",
           "kan_launch_count", "kan_forward_fixed_scratch", "kan_set_timing_marks", "kan_ffma_probe",
           "kan_grkan_workspace_size", "kan_grkan_forward", "kan_grkan_backward",
           "kan_ukan_layer_shape", "kan_ukan_generate", "kan_ukan_workspace_size", "kan_ukan_generate_backward",
           "kan_input_range",
           "kan_selftest_wait_timeout", "kan_status_string", "kan_last_error")


class kan_shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("in_", ctypes.c_int64), ("out", ctypes.c_int64),
                ("G", ctypes.c_int32), ("lo", ctypes.c_float), ("hi", ctypes.c_float),
                ("dtype", ctypes.c_int32), ("has_base", ctypes.c_int32), ("path", ctypes.c_int32),
                ("degree", ctypes.c_int32), ("dims", ctypes.c_int32)]


class kan_grkan_shape(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int64), ("channels", ctypes.c_int64), ("groups", ctypes.c_int32),
                ("num_degree", ctypes.c_int32), ("den_degree", ctypes.c_int32), ("dtype", ctypes.c_int32)]


class kan_ukan_shape(ctypes.Structure):
    _fields_ = [("in_", ctypes.c_int64), ("out", ctypes.c_int64), ("group", ctypes.c_int32),
                ("pe_dim", ctypes.c_int32), ("hidden", ctypes.c_int32), ("q0", ctypes.c_int32), ("nq", ctypes.c_int32),
                ("dtype", ctypes.c_int32)]


class KanError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}: {detail}")


_lib = None
_vp = ctypes.c_void_p


def load(path: str | None = None):
    """Load libkan_b200.so; raises if it is missing (no fallback)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise ImportError(f"{p} is missing: build it with `python -m kolmogorov_arnold_network_b200.build`")
    lib = ctypes.CDLL(p)
    sp = ctypes.POINTER(kan_shape)
    lib.kan_abi_version.restype = ctypes.c_int
    lib.kan_abi_version.argtypes = []
    lib.kan_workspace_size.restype = ctypes.c_int
    lib.kan_workspace_size.argtypes = [sp, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t)]
    lib.kan_forward.restype = ctypes.c_int
    lib.kan_forward.argtypes = [sp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
    lib.kan_backward.restype = ctypes.c_int
    lib.kan_backward.argtypes = [sp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
    lib.kan_basis.restype = ctypes.c_int
    lib.kan_basis.argtypes = [sp, _vp, _vp, _vp, _vp, _vp]
    lib.kan_sync_status.restype = ctypes.c_int
    lib.kan_sync_status.argtypes = [_vp]
    lib.kan_selftest_wait_timeout.restype = ctypes.c_int
    lib.kan_selftest_wait_timeout.argtypes = [ctypes.c_int64, _vp]
    lib.kan_status_string.restype = ctypes.c_char_p
    lib.kan_status_string.argtypes = [ctypes.c_int]
    lib.kan_last_error.restype = ctypes.c_char_p
    lib.kan_last_error.argtypes = []
    lib.kan_launch_count.restype = ctypes.c_uint64
    lib.kan_launch_count.argtypes = []
    lib.kan_forward_fixed_scratch.restype = ctypes.c_int
    lib.kan_forward_fixed_scratch.argtypes = [sp, _vp, _vp, _vp, _vp, _vp]
    gp = ctypes.POINTER(kan_grkan_shape)
    lib.kan_grkan_workspace_size.restype = ctypes.c_int
    lib.kan_grkan_workspace_size.argtypes = [gp, ctypes.POINTER(ctypes.c_size_t)]
    lib.kan_grkan_forward.restype = ctypes.c_int
    lib.kan_grkan_forward.argtypes = [gp, _vp, _vp, _vp, _vp, _vp]
    lib.kan_grkan_backward.restype = ctypes.c_int
    lib.kan_grkan_backward.argtypes = [gp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
    up = ctypes.POINTER(kan_ukan_shape)
    lib.kan_ukan_layer_shape.restype = ctypes.c_int
    lib.kan_ukan_layer_shape.argtypes = [up, ctypes.c_int64, ctypes.c_float, sp]
    lib.kan_ukan_generate.restype = ctypes.c_int
    lib.kan_ukan_generate.argtypes = [up, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
    lib.kan_ukan_workspace_size.restype = ctypes.c_int
    lib.kan_ukan_workspace_size.argtypes = [up, ctypes.POINTER(ctypes.c_size_t)]
    lib.kan_ukan_generate_backward.restype = ctypes.c_int
    lib.kan_ukan_generate_backward.argtypes = [up, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
    lib.kan_input_range.restype = ctypes.c_int
    lib.kan_input_range.argtypes = [ctypes.c_int64, _vp, ctypes.c_int32, _vp, _vp, ctypes.c_size_t, _vp]
    lib.kan_set_timing_marks.restype = ctypes.c_int
    lib.kan_set_timing_marks.argtypes = [_vp, _vp]
    lib.kan_ffma_probe.restype = ctypes.c_int
    lib.kan_ffma_probe.argtypes = [ctypes.c_int32, ctypes.c_int64, _vp, ctypes.POINTER(ctypes.c_double), _vp]
    if path is None:
        _lib = lib
    return lib


def check(status: int, where: str):
    if status != 0:
        raise KanError(status, where, load().kan_last_error().decode())


def make_shape(batch, n_in, n_out, G, lo, hi, dtype, has_base, path=KAN_PATH_AUTO, degree=3, dims=1) -> kan_shape:
    return kan_shape(int(batch), int(n_in), int(n_out), int(G), float(lo), float(hi), int(dtype), int(bool(has_base)),
                     int(path), int(degree), int(dims))


# ---- the C-ABI calls, same names, raw pointers (ints) and sizes ----
def kan_abi_version() -> int:
    return load().kan_abi_version()


def kan_workspace_size(shape: kan_shape, for_backward: bool) -> int:
    n = ctypes.c_size_t(0)
    check(load().kan_workspace_size(ctypes.byref(shape), int(bool(for_backward)), ctypes.byref(n)),
          "kan_workspace_size")
    return n.value


def kan_forward(shape, x, coef, w_base, y, workspace, ws_bytes, stream):
    check(load().kan_forward(ctypes.byref(shape), x, coef, w_base, y, workspace, ws_bytes, stream), "kan_forward")


def kan_forward_fixed_scratch(shape, x, coef, w_base, y, stream):
    check(load().kan_forward_fixed_scratch(ctypes.byref(shape), x, coef, w_base, y, stream),
          "kan_forward_fixed_scratch")


def kan_backward(shape, x, coef, w_base, dY, dx, dcoef, dw_base, workspace, ws_bytes, stream):
    check(load().kan_backward(ctypes.byref(shape), x, coef, w_base, dY, dx, dcoef, dw_base, workspace, ws_bytes,
                              stream), "kan_backward")


def kan_basis(shape, x, span, w, dw, stream):
    check(load().kan_basis(ctypes.byref(shape), x, span, w, dw, stream), "kan_basis")


def make_grkan_shape(rows, channels, groups, num_degree, den_degree, dtype) -> kan_grkan_shape:
    return kan_grkan_shape(int(rows), int(channels), int(groups), int(num_degree), int(den_degree), int(dtype))


def kan_grkan_workspace_size(shape: kan_grkan_shape) -> int:
    n = ctypes.c_size_t(0)
    check(load().kan_grkan_workspace_size(ctypes.byref(shape), ctypes.byref(n)), "kan_grkan_workspace_size")
    return n.value


def kan_grkan_forward(shape, x, a, b, y, stream):
    check(load().kan_grkan_forward(ctypes.byref(shape), x, a, b, y, stream), "kan_grkan_forward")


def kan_grkan_backward(shape, x, a, b, dY, dx, da, db, workspace, ws_bytes, stream):
    check(load().kan_grkan_backward(ctypes.byref(shape), x, a, b, dY, dx, da, db, workspace, ws_bytes, stream),
          "kan_grkan_backward")


def make_ukan_shape(n_in, n_out, group, pe_dim, hidden, q0, nq, dtype) -> kan_ukan_shape:
    return kan_ukan_shape(int(n_in), int(n_out), int(group), int(pe_dim), int(hidden), int(q0), int(nq), int(dtype))


def kan_ukan_layer_shape(shape: kan_ukan_shape, batch, h) -> kan_shape:
    out = kan_shape()
    check(load().kan_ukan_layer_shape(ctypes.byref(shape), int(batch), float(h), ctypes.byref(out)),
          "kan_ukan_layer_shape")
    return out


def kan_ukan_generate(shape, W1, b1, W2, b2, coef, pre, stream):
    check(load().kan_ukan_generate(ctypes.byref(shape), W1, b1, W2, b2, coef, pre, stream), "kan_ukan_generate")


def kan_ukan_workspace_size(shape: kan_ukan_shape) -> int:
    n = ctypes.c_size_t(0)
    check(load().kan_ukan_workspace_size(ctypes.byref(shape), ctypes.byref(n)), "kan_ukan_workspace_size")
    return n.value


def kan_ukan_generate_backward(shape, W1, W2, pre, dcoef, dW1, db1, dW2, db2, workspace, ws_bytes, stream):
    check(load().kan_ukan_generate_backward(ctypes.byref(shape), W1, W2, pre, dcoef, dW1, db1, dW2, db2, workspace,
                                            ws_bytes, stream), "kan_ukan_generate_backward")


def kan_input_range(n, x, dtype, minmax, workspace, ws_bytes, stream):
    check(load().kan_input_range(int(n), x, int(dtype), minmax, workspace, ws_bytes, stream), "kan_input_range")


def kan_set_timing_marks(after_prep, after_dcoef):
    """Events (cudaEvent_t handles as ints, or None) recorded inside later calls on this thread."""
    check(load().kan_set_timing_marks(after_prep, after_dcoef), "kan_set_timing_marks")


def kan_ffma_probe(blocks, iters, sink, stream) -> float:
    """Launch the fp32 FMA calibration kernel; returns the FLOPs it executes."""
    f = ctypes.c_double(0.0)
    check(load().kan_ffma_probe(int(blocks), int(iters), sink, ctypes.byref(f), stream), "kan_ffma_probe")
    return f.value


def kan_sync_status(stream) -> int:
    """Returns the status code (does not raise) so callers can test for timeouts."""
    return load().kan_sync_status(stream)


def kan_selftest_wait_timeout(limit_ns: int, stream):
    check(load().kan_selftest_wait_timeout(int(limit_ns), stream), "kan_selftest_wait_timeout")


def kan_status_string(st: int) -> str:
    return load().kan_status_string(int(st)).decode()


def kan_last_error() -> str:
    return load().kan_last_error().decode()


def kan_launch_count() -> int:
    return int(load().kan_launch_count())

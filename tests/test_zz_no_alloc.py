"""kan_forward_fixed_scratch: the forward for callers that cannot allocate
device memory while they run the layer (a framework's own allocator is the
only source of memory, or a serving loop must not stall on cudaMalloc).  It
takes its workspace from a fixed array inside the library instead of from
the caller.

Checked here, through the C ABI: two calls in a row give the same result as
kan_forward with a caller-allocated workspace (within the parity tolerance of
the other tests), on shapes that do use workspace (split-K partial sums, and
the fp16 hi/lo copies for fp32), and a shape whose workspace exceeds the
fixed size is refused with KAN_ERR_WORKSPACE.  This file is named to be
collected last, and passes alone in a fresh process as well.
"""
import numpy as np
import pytest
import torch

from kolmogorov_arnold_network_b200 import _native as N
from kolmogorov_arnold_network_b200 import layer as L
from kolmogorov_arnold_network_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 2e-2}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _rel(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_fixed_scratch_matches_caller_workspace(dt):
    # 512 x 256 -> 64: few output tiles, so the forward splits K and needs workspace
    w = W.custom(512, 256, 64, 8, -1.0, 1.0, dtype=dt, base=True)
    d = W.draw_all(w)
    x, coef, wb = (d[k].cuda() for k in ("x", "coef0", "w_base0"))
    s = L.shape_of(x, coef, 8, -1.0, 1.0, wb, N.KAN_PATH_TENSOR)
    need = N.kan_workspace_size(s, False)
    assert 0 < need <= 32 * 1024 * 1024
    y_ref = L.forward(x, coef, 8, -1.0, 1.0, wb, path=N.KAN_PATH_TENSOR)
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        y = torch.full_like(y_ref, float("nan"))
        N.kan_forward_fixed_scratch(s, x.data_ptr(), coef.data_ptr(), wb.data_ptr(), y.data_ptr(), stream)
        torch.cuda.synchronize()
        assert N.kan_sync_status(None) == 0
        assert torch.isfinite(y).all()
        assert _rel(y, y_ref) <= TOL[dt]


def test_fixed_scratch_refuses_oversized_workspace():
    # fp32, 512 x 2048 -> 512, G = 50: the fp16 hi/lo copies of coef alone exceed 32 MiB
    s = N.make_shape(4096, 2048, 512, 50, -1.0, 1.0, N.KAN_F32, False, N.KAN_PATH_TENSOR)
    assert N.kan_workspace_size(s, False) > 32 * 1024 * 1024
    lib = N.load()
    import ctypes
    dummy = torch.empty(16, device="cuda")
    p = dummy.data_ptr()
    rc = lib.kan_forward_fixed_scratch(ctypes.byref(s), p, p, None, p, None)
    assert rc == 3  # KAN_ERR_WORKSPACE, refused before any launch
    assert "fixed" in N.kan_last_error()

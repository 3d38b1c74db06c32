"""kan_forward_fixed_scratch: the forward for callers that cannot allocate
device memory while they run the layer (a framework's own allocator is the
only source of memory, or a serving loop must not stall on cudaMalloc).  It
takes its workspace from a fixed array inside the library instead of from
the caller.

Checked here, through the C ABI: two calls in a row give the same result as
kan_forward with a caller-allocated workspace (within the parity tolerance of
the other tests) and match the fp64 oracle, on shapes that do use workspace
(split-K partial sums, and the fp16 hi/lo copies for fp32); a call with a
different workspace layout (another split count, other offsets of the fp16
copies) between the two leaves nothing behind that changes the second
result; and a shape whose workspace exceeds the fixed size is refused with
KAN_ERR_WORKSPACE.  This file is named to be collected last, and passes alone
in a fresh process as well.
"""
import ctypes

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
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def _case(batch, n_in, n_out, G, dt):
    w = W.custom(batch, n_in, n_out, G, -1.0, 1.0, dtype=dt, base=True)
    d = W.draw_all(w)
    x, coef, wb = (d[k].cuda() for k in ("x", "coef0", "w_base0"))
    s = L.shape_of(x, coef, G, -1.0, 1.0, wb, N.KAN_PATH_TENSOR)
    return d, x, coef, wb, s


def _fixed(s, x, coef, wb, like):
    y = torch.full_like(like, float("nan"))
    N.kan_forward_fixed_scratch(s, x.data_ptr(), coef.data_ptr(), wb.data_ptr(), y.data_ptr(),
                                torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert N.kan_sync_status(None) == 0
    return y


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_fixed_scratch_matches_caller_workspace(oracle, dt):
    # 512 x 256 -> 64: few output tiles, so the forward splits K and needs workspace
    d, x, coef, wb, s = _case(512, 256, 64, 8, dt)
    need = N.kan_workspace_size(s, False)
    assert 0 < need <= 32 * 1024 * 1024
    y_ref = L.forward(x, coef, 8, -1.0, 1.0, wb, path=N.KAN_PATH_TENSOR)
    # a second shape with another workspace layout (G = 20: other split count, other fp16-copy sizes)
    d2, x2, coef2, wb2, s2 = _case(640, 64, 32, 20, dt)
    assert N.kan_workspace_size(s2, False) != need
    y2_ref = L.forward(x2, coef2, 20, -1.0, 1.0, wb2, path=N.KAN_PATH_TENSOR)
    rows = np.arange(0, 512, 7)
    o_ref = oracle.forward(d["x"][rows], d["coef0"], 8, -1.0, 1.0, w_base=d["w_base0"])
    for call in range(2):
        y = _fixed(s, x, coef, wb, y_ref)
        assert torch.isfinite(y).all()
        assert _rel(y.double().cpu().numpy(), y_ref.double().cpu().numpy()) <= TOL[dt]
        assert _rel(y.double().cpu().numpy()[rows], o_ref) <= TOL[dt]
        if call == 0:
            y2 = _fixed(s2, x2, coef2, wb2, y2_ref)
            assert _rel(y2.double().cpu().numpy(), y2_ref.double().cpu().numpy()) <= TOL[dt]


def test_fixed_scratch_refuses_oversized_workspace():
    # fp32, 512 x 2048 -> 512, G = 50: the fp16 hi/lo copies of coef alone exceed 32 MiB
    s = N.make_shape(4096, 2048, 512, 50, -1.0, 1.0, N.KAN_F32, False, N.KAN_PATH_TENSOR)
    assert N.kan_workspace_size(s, False) > 32 * 1024 * 1024
    lib = N.load()
    dummy = torch.empty(16, device="cuda")
    p = dummy.data_ptr()
    rc = lib.kan_forward_fixed_scratch(ctypes.byref(s), p, p, None, p, None)
    assert rc == 3  # KAN_ERR_WORKSPACE, refused before any launch
    assert "fixed" in N.kan_last_error()

"""2-D tensor-product B-spline surfaces (kan_shape.dims = 2) through the C ABI, against the fp64 oracle.

The InKAN landing page ("Why InKAN?", item "1D and 2D Splines") names
"tensor-product B-spline surfaces for joint function approximation"; the
layer here takes the inputs in consecutive pairs and gives every edge a cubic
surface (oracle/kan2d.py states the reading).  Bars as for the 1-D layer:
normwise max-relative error 1e-5 (fp32) and 2e-2 (bf16), bitwise repeatability.
"""
import numpy as np
import pytest
import torch

from kolmogorov_arnold_network_b200 import _native as N
from kolmogorov_arnold_network_b200 import layer as L
from kolmogorov_arnold_network_b200 import workloads as W
from oracle import kan2d

import pins
from gpu_util import TOL, cuda, f64, rel_err, sample_rows, tile_rows, workload_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def run2d(x, coef, dY, G, lo, hi, path=N.KAN_PATH_AUTO):
    y = L.forward(x, coef, G, lo, hi, path=path, dims=2)
    dx, dc, _ = L.backward(x, coef, dY, G, lo, hi, path=path, dims=2)
    torch.cuda.synchronize()
    assert N.kan_sync_status(None) == 0
    return y, dx, dc


SMALL = [
    # batch, in, out, G, lo, hi
    (300, 32, 296, 8, -1.0, 1.0),
    (257, 16, 64, 4, -1.0, 1.0),
    (130, 8, 48, 1, -1.0, 1.0),
    (200, 48, 520, 5, -3.0, 3.0),
    (300, 16, 1000, 8, -1.0, 1.0),      # wide bf16 tiles as CTA pairs, a padding M tile
    (800, 24, 296, 5, -1.0, 1.0),       # dx as CTA pairs over 256-row tiles
    (129, 64, 16, 2, -1.0, 1.0),
]


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("case", SMALL, ids=lambda c: "b{}_i{}_o{}_g{}".format(*c[:4]))
def test_surface_small_parity(oracle, dt, case):
    batch, n_in, n_out, G, lo, hi = case
    w = W.custom(batch, n_in, n_out, G, lo, hi, dtype=dt, dims=2)
    x, coef, _, dY = workload_inputs(w)
    s = L.shape_of(cuda(x), cuda(coef), G, lo, hi, None, N.KAN_PATH_AUTO, 3, 2)
    try:
        N.kan_workspace_size(s, True)
    except N.KanError as e:
        assert e.status == 2   # the tensor-core path cannot address this shape: refused, not run elsewhere
        pytest.skip(f"not addressable by TMA: {e}")
    y, dx, dc = run2d(cuda(x), cuda(coef), cuda(dY), G, lo, hi)
    y_ref = kan2d.forward(x, coef, G, lo, hi, o=oracle)
    dx_ref, dc_ref = kan2d.backward(x, coef, dY, G, lo, hi, o=oracle)
    errs = {"y": rel_err(f64(y.cpu()), y_ref), "dx": rel_err(f64(dx.cpu()), dx_ref),
            "dcoef": rel_err(f64(dc.cpu()), dc_ref)}
    assert all(v <= TOL[dt] for v in errs.values()), errs


def test_surface_marsden_closed_form():
    # coef[j,p,m1,m2] = psi_m1(s) psi_m2(r): y = sum_p (s - u)^3 (r - v)^3 and both dx in closed form, any batch
    G, lo, hi = 8, -1.0, 1.0
    batch, n_in, n_out = 16384, 32, 96
    g = torch.Generator().manual_seed(61)
    x = torch.rand(batch, n_in, generator=g) * 2 - 1
    s = (torch.rand(n_out, n_in // 2, generator=g) - 0.5).double().numpy()
    r = (torch.rand(n_out, n_in // 2, generator=g) - 0.5).double().numpy()
    ps, pr = pins.marsden_coef(s, G, lo, hi), pins.marsden_coef(r, G, lo, hi)
    coef = torch.from_numpy(ps[:, :, :, None] * pr[:, :, None, :]).float()
    dY = torch.randn(batch, n_out, generator=g)
    y, dx, _ = run2d(cuda(x), cuda(coef), cuda(dY), G, lo, hi, path=N.KAN_PATH_TENSOR)
    xd = f64(x)
    fu = s[None] - xd[:, None, 0::2]
    fv = r[None] - xd[:, None, 1::2]
    ref = (fu ** 3 * fv ** 3).sum(2)
    du = np.einsum("bj,bjp->bp", f64(dY), -3 * fu ** 2 * fv ** 3)
    dv = np.einsum("bj,bjp->bp", f64(dY), -3 * fu ** 3 * fv ** 2)
    assert rel_err(f64(y.cpu()), ref) <= TOL["f32"]
    dxd = f64(dx.cpu())
    assert rel_err(dxd[:, 0::2], du) <= TOL["f32"] and rel_err(dxd[:, 1::2], dv) <= TOL["f32"]


@pytest.mark.parametrize("name", ["surface512_g8_bf16_fwdbwd", "surface512_g8_f32_fwdbwd"])
def test_surface_workload_parity(oracle, name):
    w = W.WORKLOADS[name]
    Ly = w.layers[0]
    x, coef, _, dY = workload_inputs(w)
    y, dx, dc = run2d(cuda(x), cuda(coef), cuda(dY), Ly.G, Ly.lo, Ly.hi)
    rows = np.union1d(tile_rows(w.batch), sample_rows(w.batch))
    y_ref = kan2d.forward(x[rows], coef, Ly.G, Ly.lo, Ly.hi, o=oracle)
    dx_ref, _ = kan2d.backward(x[rows], coef, dY[rows], Ly.G, Ly.lo, Ly.hi, o=oracle, want_dcoef=False)
    # dcoef: every output and every column of the pairs in the first two 128-column M tiles and the last
    nbu = Ly.cols
    units = Ly.units
    cols = np.concatenate([np.arange(2 * 128), np.arange(((units * nbu - 1) // 128) * 128, units * nbu)])
    pairs = np.unique(cols // nbu)
    xp = torch.stack([x[:, 2 * p + c] for p in pairs for c in (0, 1)], dim=1)
    _, dc_ref = kan2d.backward(xp, coef[:, pairs], dY, Ly.G, Ly.lo, Ly.hi, o=oracle, want_dx=False)
    errs = {"y": rel_err(f64(y.cpu()[rows]), y_ref), "dx": rel_err(f64(dx.cpu()[rows]), dx_ref),
            "dcoef": rel_err(f64(dc.cpu()[:, pairs]), dc_ref)}
    assert all(v <= TOL[w.dtype] for v in errs.values()), errs


def test_surface_deterministic():
    w = W.WORKLOADS["surface512_g8_bf16_fwdbwd"]
    Ly = w.layers[0]
    x, coef, _, dY = (cuda(t) for t in workload_inputs(w))
    first = run2d(x, coef, dY, Ly.G, Ly.lo, Ly.hi)
    for _ in range(10):
        again = run2d(x, coef, dY, Ly.G, Ly.lo, Ly.hi)
        for a, b in zip(first, again):
            assert torch.equal(a, b)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_surface_no_store_outside_the_outputs(dt):
    from test_gpu_guard import Guarded
    batch, n_in, n_out, G = 300, 16, 1000, 8
    w = W.custom(batch, n_in, n_out, G, -1.0, 1.0, dtype=dt, dims=2)
    x, coef, _, dY = (cuda(t) for t in workload_inputs(w))
    s = L.shape_of(x, coef, G, -1.0, 1.0, None, N.KAN_PATH_TENSOR, 3, 2)
    y = Guarded((batch, n_out), x.dtype)
    dx = Guarded((batch, n_in), x.dtype)
    dc = Guarded(tuple(coef.shape), torch.float32)
    wsf = Guarded((max(1, N.kan_workspace_size(s, False)),), torch.uint8)
    wsb = Guarded((max(1, N.kan_workspace_size(s, True)),), torch.uint8)
    L.forward(x, coef, G, -1.0, 1.0, path=N.KAN_PATH_TENSOR, y=y.t, ws=wsf.t, dims=2)
    L.backward(x, coef, dY, G, -1.0, 1.0, path=N.KAN_PATH_TENSOR, out=(dx.t, dc.t, None), ws=wsb.t, dims=2)
    torch.cuda.synchronize()
    assert N.kan_sync_status(None) == 0
    y.check("y")
    dx.check("dx")
    dc.check("dcoef")
    wsf.check("forward workspace", all_written=False)
    wsb.check("backward workspace", all_written=False)


def test_surface_module_autograd(oracle):
    torch.manual_seed(2)
    layer = L.KANLayer2D(8, 6, G=5).cuda()
    x = (torch.rand(40, 8, device="cuda") * 2.4 - 1.2).requires_grad_(True)
    y = layer(x)
    g = torch.randn_like(y)
    y.backward(g)
    xc, cc, gc = x.detach().cpu(), layer.coef.detach().cpu(), g.cpu()
    assert rel_err(f64(y.detach().cpu()), kan2d.forward(xc, cc, 5, -1.0, 1.0, o=oracle)) <= 1e-5
    dx_ref, dc_ref = kan2d.backward(xc, cc, gc, 5, -1.0, 1.0, o=oracle)
    assert rel_err(f64(x.grad.cpu()), dx_ref) <= 1e-5
    assert rel_err(f64(layer.coef.grad.cpu()), dc_ref) <= 1e-5

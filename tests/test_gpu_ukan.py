"""UKAN layers (unbounded grid, generated coefficients) through the C ABI, against the fp64 oracle.

"Want to train KANS at scale? Now UKAN!" (Abstract): a coefficient generator
fed with the positional encodings of grid groups produces only the
coefficients the batch needs, on an unbounded grid; oracle/ukan.py states the
reading.  Bars: normwise max-relative error 1e-5 (fp32 window) and 2e-2 (bf16
window) per output; bitwise repeatability.
"""
import numpy as np
import pytest
import torch

from kolmogorov_arnold_network_b200 import _native as N
from kolmogorov_arnold_network_b200 import layer as L
from kolmogorov_arnold_network_b200 import workloads as W
from oracle import ukan as ref

from gpu_util import TOL, f64, rel_err, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _layer_run(w, d):
    """Forward and backward through the functional path; returns y, dx, dW1, db1, dW2, db2, dcoef, (q0, nq)."""
    x = d["x"].cuda()
    W1, b1, W2, b2 = (d[k].cuda() for k in ("W1", "b1", "W2", "b2"))
    dY = d["dY"].cuda()
    q0, nq = L.ukan_window(x, w.h, w.group)
    coef, pre = L.ukan_generate(W1, b1, W2, b2, w.inp, w.out, w.group, q0, nq, x.dtype)
    ks = N.kan_ukan_layer_shape(L.ukan_shape(w.inp, w.out, w.group, W1, q0, nq, x.dtype), w.batch, w.h)
    y = L.forward(x, coef, ks.G, ks.lo, ks.hi)
    dx, dcoef, _ = L.backward(x, coef, dY, ks.G, ks.lo, ks.hi)
    dW1, db1, dW2, db2 = L.ukan_generate_backward(W1, W2, pre, dcoef, w.inp, w.out, w.group, q0, nq, x.dtype)
    torch.cuda.synchronize()
    assert N.kan_sync_status(None) == 0
    return y, dx, dW1, db1, dW2, db2, dcoef, (q0, nq)


CASES = [
    # batch, in, out, h, group, pe_dim, hidden, x_std, shift
    (300, 16, 24, 0.25, 4, 16, 32, 1.0, 0.0),
    (257, 8, 40, 0.5, 3, 8, 16, 3.0, 0.0),
    (200, 16, 32, 0.25, 4, 16, 32, 1.0, 40.0),       # inputs far from 0: no normalisation needed
    (129, 24, 16, 0.1, 8, 32, 64, 0.5, -3.0),
]


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "b{}_i{}_o{}_h{}_g{}_s{}".format(c[0], c[1], c[2], c[3], c[4],
                                                                                          c[8]))
def test_ukan_parity(dt, case):
    batch, n_in, n_out, h, g, d_pe, H, xs, shift = case
    w = W.custom_ukan(batch, n_in, n_out, h, g, d_pe, H, dtype=dt, x_std=xs)
    d = W.draw_ukan(w)
    d["x"] = (d["x"].float() + shift).to(w.torch_dtype)
    y, dx, dW1, db1, dW2, db2, _, (q0, nq) = _layer_run(w, d)
    assert (q0, nq) == ref.groups_of(d["x"], h, g)
    args = (d["W1"], d["b1"], d["W2"], d["b2"])
    y_ref = ref.forward(d["x"], *args, n_out, h, g)
    dx_ref, dW1_ref, db1_ref, dW2_ref, db2_ref, _ = ref.backward(d["x"], *args, d["dY"], n_out, h, g)
    errs = {"y": rel_err(f64(y.cpu()), y_ref), "dx": rel_err(f64(dx.cpu()), dx_ref),
            "dW1": rel_err(f64(dW1.cpu()), dW1_ref), "db1": rel_err(f64(db1.cpu()), db1_ref),
            "dW2": rel_err(f64(dW2.cpu()), dW2_ref), "db2": rel_err(f64(db2.cpu()), db2_ref)}
    assert all(v <= TOL[dt] for v in errs.values()), errs


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_ukan_generator_window(dt):
    w = W.custom_ukan(64, 32, 48, 0.25, 4, 16, 32, dtype=dt)
    d = W.draw_ukan(w)
    W1, b1, W2, b2 = (d[k].cuda() for k in ("W1", "b1", "W2", "b2"))
    coef, pre = L.ukan_generate(W1, b1, W2, b2, 32, 48, 4, -7, 9, w.torch_dtype)
    torch.cuda.synchronize()
    c_ref, pre_ref = ref.cg_coef(d["W1"], d["b1"], d["W2"], d["b2"], 48, 32, 4, -7, 9)
    assert rel_err(f64(pre.cpu()), pre_ref) <= 1e-5
    assert rel_err(f64(coef.cpu()), c_ref) <= TOL[dt] if dt == "bf16" else rel_err(f64(coef.cpu()), c_ref) <= 1e-5


@pytest.mark.parametrize("name", sorted(W.UK_WORKLOADS))
def test_ukan_workload_parity(name):
    w = W.UK_WORKLOADS[name]
    d = W.draw_ukan(w)
    y, dx, dW1, db1, dW2, db2, dcoef, (q0, nq) = _layer_run(w, d)
    args = (d["W1"], d["b1"], d["W2"], d["b2"])
    rows = np.union1d(sample_rows(w.batch, 32), np.arange(w.batch - 8, w.batch))
    y_ref = ref.forward(d["x"][rows], *args, w.out, w.h, w.group, q0, nq)
    dx_ref = ref.backward(d["x"][rows], *args, d["dY"][rows], w.out, w.h, w.group, q0, nq)[0]
    # the generator's gradients from the GPU's window dcoef (the layer's dcoef is checked by the KAN tests)
    g_ref = ref.generator_backward(d["W1"], d["b1"], d["W2"], dcoef.cpu(), q0, nq)
    errs = {"y": rel_err(f64(y.cpu()[rows]), y_ref), "dx": rel_err(f64(dx.cpu()[rows]), dx_ref)}
    for nm, got, want in zip(("dW1", "db1", "dW2", "db2"), (dW1, db1, dW2, db2), g_ref):
        errs[nm] = rel_err(f64(got.cpu()), want)
    tol = TOL[w.dtype]
    assert errs["y"] <= tol and errs["dx"] <= tol, errs
    assert all(errs[k] <= 1e-5 for k in ("dW1", "db1", "dW2", "db2")), errs


def test_ukan_deterministic():
    w = W.custom_ukan(4096, 64, 64, 0.25, 4, 16, 32, dtype="bf16")
    d = W.draw_ukan(w)
    first = _layer_run(w, d)
    for _ in range(10):
        again = _layer_run(w, d)
        for a, b in zip(first[:7], again[:7]):
            assert torch.equal(a, b)


def test_ukan_module_autograd():
    torch.manual_seed(3)
    layer = L.UKANLayer(12, 20, h=0.5, group=4, pe_dim=8, hidden=16).cuda()
    with torch.no_grad():
        layer.b2.normal_(0, 0.2)
    x = (torch.randn(50, 12, device="cuda") * 2).requires_grad_(True)
    y = layer(x)
    g = torch.randn_like(y)
    y.backward(g)
    args = [p.detach().cpu() for p in (layer.W1, layer.b1, layer.W2, layer.b2)]
    xc = x.detach().cpu()
    assert rel_err(f64(y.detach().cpu()), ref.forward(xc, *args, 20, 0.5, 4)) <= 1e-5
    dx_ref, dW1_ref, db1_ref, dW2_ref, db2_ref, _ = ref.backward(xc, *args, g.cpu(), 20, 0.5, 4)
    for got, want in ((x.grad, dx_ref), (layer.W1.grad, dW1_ref), (layer.b1.grad, db1_ref), (layer.W2.grad, dW2_ref),
                      (layer.b2.grad, db2_ref)):
        assert rel_err(f64(got.cpu()), want) <= 1e-5


def test_input_range():
    x = torch.randn(1000, 37, device="cuda") * 5
    x[3, 4] = -123.5
    x[999, 36] = 77.25
    ws = torch.empty(2368, dtype=torch.uint8, device="cuda")
    mm = torch.empty(2, device="cuda")
    N.kan_input_range(x.numel(), x.data_ptr(), N.KAN_F32, mm.data_ptr(), ws.data_ptr(), 2368,
                      torch.cuda.current_stream().cuda_stream)
    assert mm.tolist() == [-123.5, 77.25]

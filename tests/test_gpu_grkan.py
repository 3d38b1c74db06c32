"""GR-KAN (group-rational activation) through the C ABI on the GPU, against the fp64 oracle.

Bars: normwise max-relative error 1e-5 for fp32 operands and 2e-2 for bf16
operands, per output tensor (y, dx, da, db); bitwise equality for the
determinism check (the FlashKAT abstract's point: gradient accumulation
without atomic adds).
"""
import numpy as np
import pytest
import torch

from kolmogorov_arnold_network_b200 import _native as N
from kolmogorov_arnold_network_b200 import layer as L
from kolmogorov_arnold_network_b200 import workloads as W
from oracle import grkan as ref

from gpu_util import TOL, f64, rel_err, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _run(d, groups):
    x, a, b, dY = (d[k].cuda() for k in ("x", "a", "b", "dY"))
    y = L.grkan_forward(x, a, b, groups)
    dx, da, db = L.grkan_backward(x, a, b, dY, groups)
    torch.cuda.synchronize()
    assert N.kan_sync_status(None) == 0
    return y, dx, da, db


SMALL = [
    # rows, channels, groups, m, n
    (1000, 768, 8, 5, 4),
    (333, 96, 1, 3, 2),
    (77, 64, 4, 7, 8),
    (2, 16, 2, 1, 1),
    (1500, 4096, 2, 5, 4),     # 2048-channel groups: two 256-thread strips per group (fp32)
    (129, 3072, 8, 2, 5),
]


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("case", SMALL, ids=lambda c: "r{}_c{}_g{}_m{}n{}".format(*c))
def test_grkan_small_parity(dt, case):
    rows, C, G, m, n = case
    if dt == "f32" and (C // G) % 4 or dt == "bf16" and (C // G) % 8:
        pytest.skip("channels per group not a whole number of 16-byte vectors")
    w = W.custom_grkan(rows, C, G, m, n, dtype=dt)
    d = W.draw_grkan(w)
    y, dx, da, db = _run(d, G)
    y_ref = ref.forward(d["x"], d["a"], d["b"], G)
    dx_ref, da_ref, db_ref = ref.backward(d["x"], d["a"], d["b"], d["dY"], G)
    errs = {"y": rel_err(f64(y.cpu()), y_ref), "dx": rel_err(f64(dx.cpu()), dx_ref),
            "da": rel_err(f64(da.cpu()), da_ref), "db": rel_err(f64(db.cpu()), db_ref)}
    assert all(v <= TOL[dt] for v in errs.values()), errs


@pytest.mark.parametrize("name", sorted(W.GR_WORKLOADS))
def test_grkan_workload_parity(name):
    w = W.GR_WORKLOADS[name]
    d = W.draw_grkan(w)
    y, dx, da, db = _run(d, w.groups)
    rows = np.union1d(sample_rows(w.rows, 64), np.arange(w.rows - 8, w.rows))
    xr, gr = d["x"][rows], d["dY"][rows]
    y_ref = ref.forward(xr, d["a"], d["b"], w.groups)
    dx_ref, _, _ = ref.backward(xr, d["a"], d["b"], gr, w.groups)
    _, da_ref, db_ref = ref.backward(d["x"], d["a"], d["b"], d["dY"], w.groups)
    errs = {"y": rel_err(f64(y.cpu()[rows]), y_ref), "dx": rel_err(f64(dx.cpu()[rows]), dx_ref),
            "da": rel_err(f64(da.cpu()), da_ref), "db": rel_err(f64(db.cpu()), db_ref)}
    assert all(v <= TOL[w.dtype] for v in errs.values()), errs


def test_grkan_deterministic():
    w = W.GR_WORKLOADS["grkan_vitb_bf16"]
    d = W.draw_grkan(w)
    first = _run(d, w.groups)
    for _ in range(10):
        again = _run(d, w.groups)
        for u, v in zip(first, again):
            assert torch.equal(u, v)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_grkan_identity_initialisation(dt):
    # a = (0, 1, 0, ...), b = 0: phi(x) = x / 1, exactly, and dx = dY
    w = W.custom_grkan(300, 768, 8, 5, 4, dtype=dt)
    d = W.draw_grkan(w)
    d["a"] = torch.zeros_like(d["a"])
    d["a"][:, 1] = 1.0
    d["b"] = torch.zeros_like(d["b"])
    y, dx, _, _ = _run(d, 8)
    assert torch.equal(y.cpu(), d["x"])
    assert torch.equal(dx.cpu(), d["dY"])


def test_grkan_skips_and_empty():
    w = W.custom_grkan(64, 96, 3, 5, 4, dtype="f32")
    d = W.draw_grkan(w)
    x, a, b, dY = (d[k].cuda() for k in ("x", "a", "b", "dY"))
    dx, da, db = L.grkan_backward(x, a, b, dY, 3, need_da=False, need_db=False)
    assert da is None and db is None
    dx2, da2, db2 = L.grkan_backward(x, a, b, dY, 3, need_dx=False)
    torch.cuda.synchronize()
    dx_ref, da_ref, db_ref = ref.backward(d["x"], d["a"], d["b"], d["dY"], 3)
    assert rel_err(f64(dx.cpu()), dx_ref) <= TOL["f32"]
    assert rel_err(f64(da2.cpu()), da_ref) <= TOL["f32"] and rel_err(f64(db2.cpu()), db_ref) <= TOL["f32"]
    xe = torch.empty(0, 96, device="cuda")
    assert L.grkan_forward(xe, a, b, 3).shape == (0, 96)
    _, dae, dbe = L.grkan_backward(xe, a, b, xe, 3)
    torch.cuda.synchronize()
    assert torch.all(dae == 0) and torch.all(dbe == 0)


def test_grkan_module_autograd():
    torch.manual_seed(1)
    act = L.GRKAN(192, groups=4).cuda()
    with torch.no_grad():
        act.a.normal_(0, 0.5)
        act.b.normal_(0, 0.5)
    x = torch.randn(2, 50, 192, device="cuda", requires_grad=True)
    y = act(x)
    g = torch.randn_like(y)
    y.backward(g)
    xr = x.detach().reshape(-1, 192).cpu()
    dx_ref, da_ref, db_ref = ref.backward(xr, act.a.detach().cpu(), act.b.detach().cpu(), g.reshape(-1, 192).cpu(), 4)
    assert rel_err(f64(x.grad.reshape(-1, 192).cpu()), dx_ref) <= 1e-5
    assert rel_err(f64(act.a.grad.cpu()), da_ref) <= 1e-5
    assert rel_err(f64(act.b.grad.cpu()), db_ref) <= 1e-5


class _Guard:
    def __init__(self, n, dtype, pat):
        esz = torch.empty((), dtype=dtype).element_size()
        self.g = 512 // esz
        self.n = n
        self.buf = torch.full((n + 2 * self.g,), float("nan"), dtype=dtype, device="cuda")
        self.t = self.buf[self.g:self.g + n]

    def ok(self):
        b = self.buf.cpu()
        return bool(torch.isnan(b[:self.g]).all() and torch.isnan(b[self.g + self.n:]).all()
                    and not torch.isnan(b[self.g:self.g + self.n]).any())


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_grkan_no_store_outside_the_outputs(dt):
    w = W.custom_grkan(257, 3072, 8, 5, 4, dtype=dt)
    d = W.draw_grkan(w)
    x, a, b, dY = (d[k].cuda() for k in ("x", "a", "b", "dY"))
    y = _Guard(x.numel(), x.dtype, None)
    dx = _Guard(x.numel(), x.dtype, None)
    da = _Guard(a.numel(), torch.float32, None)
    db = _Guard(b.numel(), torch.float32, None)
    L.grkan_forward(x, a, b, 8, y=y.t.view(x.shape))
    L.grkan_backward(x, a, b, dY, 8, out=(dx.t.view(x.shape), da.t.view(a.shape), db.t.view(b.shape)))
    torch.cuda.synchronize()
    assert N.kan_sync_status(None) == 0
    assert y.ok() and dx.ok() and da.ok() and db.ok()

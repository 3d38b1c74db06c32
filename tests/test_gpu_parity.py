"""Parity of the CUDA path (through the C ABI) with the fp64 oracle, on the GPU.

Bars: normwise max-relative error 1e-5 for fp32 operands and 2e-2 for bf16
operands (fp32 accumulation), per output tensor; bitwise equality for the
determinism check.
"""
import math

import numpy as np
import pytest
import torch

from kolmogorov_arnold_network_b200 import _native as N
from kolmogorov_arnold_network_b200 import layer as L
from kolmogorov_arnold_network_b200 import workloads as W

import pins
from gpu_util import (TOL, check_layer_against_oracle, cuda, f64, gpu_layer, rel_err, sample_cols, sample_rows,
                      tile_inputs, tile_rows, workload_inputs)

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "bf16": torch.bfloat16}
PATHS = {"tensor": N.KAN_PATH_TENSOR, "simt": N.KAN_PATH_SIMT}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


# ---------------------------------------------------------------------------
# basis step (S1, S2)
def dense_from_basis(span, w, nb, k=3):
    span = span.cpu().numpy().reshape(-1)
    w = w.cpu().double().numpy().reshape(-1, k + 1)
    out = np.zeros((span.size, nb))
    for e in range(span.size):
        if span[e] == np.iinfo(np.int32).min:
            continue
        for r in range(k + 1):
            m = span[e] + r
            if 0 <= m < nb:
                out[e, m] = w[e, r]
    return out


def test_basis_exact_local_weights():
    # inputs exactly on t_s + u*h with h = 1/4 (all exact in fp32): the weights
    # then carry only the evaluation error, "Float32 accuracy ~1.2e-7"
    # (InKAN landing page, "Numerically Stable").
    G, lo, hi = 8, -1.0, 1.0
    h = (hi - lo) / G
    rows = pins.read_golden()
    xs, exp_w, exp_dw = [], [], []
    for s in range(-3, G + 3):
        for row in rows:
            xs.append(lo + (s + float(row[0])) * h)
            exp_w.append([float(v) for v in row[1:5]])
            exp_dw.append([float(v) / h for v in row[5:9]])
    x = torch.tensor(xs, dtype=torch.float32, device="cuda").reshape(-1, 1)
    span, w, dw = L.basis(x, G, lo, hi)
    assert np.max(np.abs(w.cpu().double().numpy().reshape(-1, 4) - np.array(exp_w))) <= 4 * 2.0 ** -23
    assert np.max(np.abs(dw.cpu().double().numpy().reshape(-1, 4) - np.array(exp_dw))) * h <= 4 * 2.0 ** -23
    assert np.all(w.cpu().numpy() >= 0.0)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("G,lo,hi", [(8, -1.0, 1.0), (20, -1.0, 1.0), (5, -3.0, 3.0), (50, -1.0, 1.0)])
def test_basis_vs_oracle(oracle, dt, G, lo, hi):
    h = (hi - lo) / G
    g = torch.Generator().manual_seed(G)
    x = (torch.rand(4096, generator=g) * (hi - lo + 8 * h) + lo - 4 * h)
    x = torch.cat([x, torch.tensor([lo, hi, lo - 3 * h, hi + 3 * h, hi + 3.2 * h, float("inf"), -float("inf"),
                                    float("nan"), 1e30, -1e30])]).to(DT[dt])
    xd = x.reshape(-1, 1).to("cuda")
    span, w, dw = L.basis(xd, G, lo, hi)
    B_ref, dB_ref = oracle.basis(f64(x), G, lo, hi)
    B = dense_from_basis(span, w, G + 3)
    dB = dense_from_basis(span, dw, G + 3)
    u = np.abs((f64(x) - lo) / h)
    u = np.where(np.isfinite(u), u, 0.0)
    # fp32 rounding of u = (x-lo)/h moves the local coordinate by ~ulp(u)
    tol = 2.0 ** -22 * (1.0 + u)[:, None]
    assert np.all(np.abs(B - B_ref) <= tol)
    assert np.all(np.abs(dB - dB_ref) * h <= 4 * tol)
    assert np.all(B >= 0.0)
    assert np.max((B != 0).sum(1)) <= 4


# ---------------------------------------------------------------------------
# small problems, both kernel families, against the full oracle
SMALL = [
    # batch, in, out, G, lo, hi, base
    (300, 40, 296, 8, -1.0, 1.0, False),
    (257, 24, 64, 20, -1.0, 1.0, True),
    (130, 16, 48, 50, -1.0, 1.0, False),
    (200, 32, 520, 5, -3.0, 3.0, True),
    (129, 8, 16, 8, -1.0, 1.0, True),
    # wide bf16 tiles run as CTA pairs: odd M-tile counts (a padding tile), ragged N
    (300, 32, 1000, 8, -1.0, 1.0, False),
    (300, 16, 256, 8, -1.0, 1.0, True),
    (300, 8, 696, 20, -1.0, 1.0, True),
    # dx as CTA pairs over 256-row tiles: an odd batch-tile count, dY resident or streamed
    (800, 32, 64, 8, -1.0, 1.0, True),
    (800, 24, 296, 20, -1.0, 1.0, False),
    # G = 5: a ragged last k-block, x rows not 16-byte aligned
    (300, 20, 256, 5, -3.0, 3.0, False),
]


@pytest.mark.parametrize("path", ["tensor", "simt"])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("case", SMALL, ids=lambda c: "b{}_i{}_o{}_g{}{}".format(c[0], c[1], c[2], c[3],
                                                                                    "_silu" if c[6] else ""))
def test_small_parity(oracle, path, dt, case):
    batch, n_in, n_out, G, lo, hi, base = case
    w = W.custom(batch, n_in, n_out, G, lo, hi, dtype=dt, base=base)
    x, coef, wb, dY = workload_inputs(w)
    y, dx, dc, dwb = gpu_layer(cuda(x), cuda(coef), cuda(wb), cuda(dY), G, lo, hi, path=PATHS[path])
    torch.cuda.synchronize()
    assert N.kan_sync_status(None) == 0
    errs = check_layer_against_oracle(oracle, x, coef, wb, dY, G, lo, hi, y.cpu(), dx.cpu(), dc.cpu(),
                                      None if dwb is None else dwb.cpu(), dt)
    bad = {k: v for k, v in errs.items() if not v <= TOL[dt]}
    assert not bad, f"{errs}"


# ---------------------------------------------------------------------------
# spline degree k = 1..5 (FlashKAN abstract: degree-k splines, coordinate bounded to [0, k+1])
DEGREES = [1, 2, 4, 5]
DEG_SMALL = [
    (300, 40, 296, 8, -1.0, 1.0, False),
    (257, 24, 64, 20, -1.0, 1.0, True),
    # CTA pairs (forward, dcoef), dx pairs over 256-row tiles
    (300, 16, 256, 8, -1.0, 1.0, True),
    (800, 24, 296, 20, -1.0, 1.0, False),
    # x rows not 16-byte aligned (bf16), G + k = 8
    (300, 20, 256, None, -3.0, 3.0, False),
]


@pytest.mark.parametrize("k", DEGREES)
@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("G,lo,hi", [(8, -1.0, 1.0), (50, -1.0, 1.0), (5, -3.0, 3.0)])
def test_basis_degree_vs_oracle(oracle, k, dt, G, lo, hi):
    h = (hi - lo) / G
    g = torch.Generator().manual_seed(100 + k)
    x = (torch.rand(4096, generator=g) * (hi - lo + 2 * (k + 1) * h) + lo - (k + 1) * h)
    x = torch.cat([x, torch.tensor([lo, hi, lo - k * h, hi + k * h, float("inf"), -float("inf"),
                                    float("nan")])]).to(DT[dt])
    span, w, dw = L.basis(x.reshape(-1, 1).to("cuda"), G, lo, hi, degree=k)
    B_ref, dB_ref = oracle.basis(f64(x), G, lo, hi, k=k)
    B = dense_from_basis(span, w, G + k, k)
    dB = dense_from_basis(span, dw, G + k, k)
    u = np.abs((f64(x) - lo) / h)
    u = np.where(np.isfinite(u), u, 0.0)
    tol = 2.0 ** -21 * (1.0 + u)[:, None]
    assert np.all(np.abs(B - B_ref) <= tol)
    # degree 1 is not differentiable at the knots: within the fp32 rounding of u = (x - lo)/h of a knot,
    # the derivative of either side is correct, so those inputs are left out of the derivative check
    near_knot = np.abs(u - np.round(u)) < 2.0 ** -20 * (1.0 + u) if k == 1 else np.zeros_like(u, dtype=bool)
    assert np.all((np.abs(dB - dB_ref) * h <= 4 * tol) | near_knot[:, None])
    assert np.all(B >= 0.0)
    assert np.max((B != 0).sum(1)) <= k + 1


@pytest.mark.parametrize("k", DEGREES)
@pytest.mark.parametrize("path", ["tensor", "simt"])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("case", DEG_SMALL, ids=lambda c: "b{}_i{}_o{}_g{}{}".format(c[0], c[1], c[2], c[3],
                                                                                        "_silu" if c[6] else ""))
def test_degree_parity(oracle, k, path, dt, case):
    batch, n_in, n_out, G, lo, hi, base = case
    G = G if G is not None else 8 - k
    w = W.custom(batch, n_in, n_out, G, lo, hi, dtype=dt, base=base, degree=k)
    x, coef, wb, dY = workload_inputs(w)
    y, dx, dc, dwb = gpu_layer(cuda(x), cuda(coef), cuda(wb), cuda(dY), G, lo, hi, path=PATHS[path], degree=k)
    torch.cuda.synchronize()
    assert N.kan_sync_status(None) == 0
    errs = check_layer_against_oracle(oracle, x, coef, wb, dY, G, lo, hi, y.cpu(), dx.cpu(), dc.cpu(),
                                      None if dwb is None else dwb.cpu(), dt, k=k)
    bad = {kk: v for kk, v in errs.items() if not v <= TOL[dt]}
    assert not bad, f"{errs}"


@pytest.mark.parametrize("k", DEGREES)
def test_marsden_degree_closed_form(k):
    # coef[j,i,m] = prod_{l=1..k} (y_ji - t_{m+l}) reproduces y[b,j] = sum_i (y_ji - x_bi)^k and
    # dx = -k sum_j dY (y_ji - x_bi)^(k-1) for x in [lo, hi] (Marsden's identity), at any batch size
    G, lo, hi = 8, -1.0, 1.0
    batch, n_in, n_out = 16384, 32, 96
    g = torch.Generator().manual_seed(50 + k)
    x = torch.rand(batch, n_in, generator=g) * 2 - 1
    yt = (torch.rand(n_out, n_in, generator=g) * 0.5 - 0.25).double().numpy()
    coef = torch.from_numpy(pins.marsden_coef(yt, G, lo, hi, k)).float()
    dY = torch.randn(batch, n_out, generator=g)
    y, dx, _, _ = gpu_layer(cuda(x), cuda(coef), None, cuda(dY), G, lo, hi, path=N.KAN_PATH_TENSOR, degree=k)
    xd = f64(x)
    ref = ((yt[None, :, :] - xd[:, None, :]) ** k).sum(2)
    dref = np.einsum("bj,bji->bi", f64(dY), -k * (yt[None, :, :] - xd[:, None, :]) ** (k - 1))
    assert rel_err(f64(y.cpu()), ref) <= TOL["f32"]
    assert rel_err(f64(dx.cpu()), dref) <= TOL["f32"]


@pytest.mark.parametrize("name", [f"degree512_k{k}_g20_bf16_fwdbwd" for k in DEGREES])
def test_degree_workload_parity(oracle, name):
    w = W.WORKLOADS[name]
    Ly = w.layers[0]
    x, coef, wb, dY = workload_inputs(w)
    y, dx, dc, dwb = gpu_layer(cuda(x), cuda(coef), cuda(wb), cuda(dY), Ly.G, Ly.lo, Ly.hi, degree=Ly.degree)
    torch.cuda.synchronize()
    assert N.kan_sync_status(None) == 0
    rows = np.union1d(tile_rows(w.batch), sample_rows(w.batch))
    errs = check_layer_against_oracle(oracle, x, coef, wb, dY, Ly.G, Ly.lo, Ly.hi, y.cpu(), dx.cpu(), dc.cpu(), None,
                                      w.dtype, rows=rows, cols_in=tile_inputs(Ly.inp, Ly.nb),
                                      cols_out=np.arange(Ly.out), k=Ly.degree)
    assert all(v <= TOL[w.dtype] for v in errs.values()), errs


# ---------------------------------------------------------------------------
# the named workloads at full size, in the launch configuration of the benchmark
LAYER_WORKLOADS = ["layer8x4", "layer784x64_silu", "layer1024_g20_bf16"] + \
    [f"sweep512_g{G}_{dt}_fwdbwd" for G in (8, 20, 50) for dt in ("f32", "bf16")]


@pytest.mark.parametrize("name", LAYER_WORKLOADS)
def test_workload_parity(oracle, name):
    w = W.WORKLOADS[name]
    Ly = w.layers[0]
    x, coef, wb, dY = workload_inputs(w)
    y, dx, dc, dwb = gpu_layer(cuda(x), cuda(coef), cuda(wb), cuda(dY), Ly.G, Ly.lo, Ly.hi)
    torch.cuda.synchronize()
    assert N.kan_sync_status(None) == 0
    small = w.batch * Ly.inp * Ly.out <= 4096 * 784 * 64
    # large workloads: every row of whole batch tiles (the first CTA pair and the last, ragged tile) plus a
    # random sample; dcoef for every output of the inputs of whole M tiles (the first pair, the last tile)
    rows = None if small else np.union1d(tile_rows(w.batch), sample_rows(w.batch))
    ci = None if small else tile_inputs(Ly.inp, Ly.G + 3)
    co = None if small else np.arange(Ly.out)
    errs = check_layer_against_oracle(oracle, x, coef, wb, dY, Ly.G, Ly.lo, Ly.hi, y.cpu(), dx.cpu(), dc.cpu(),
                                      None if dwb is None else dwb.cpu(), w.dtype, rows=rows, cols_in=ci,
                                      cols_out=co)
    bad = {k: v for k, v in errs.items() if not v <= TOL[w.dtype]}
    assert not bad, f"{errs}"


def test_tiny_layer_on_the_tensor_path(oracle):
    # KANLayer(8, 4) (out = 4, fp32): the fp16 copies of dY are padded to 8 columns for TMA
    w = W.WORKLOADS["layer8x4"]
    Ly = w.layers[0]
    x, coef, wb, dY = workload_inputs(w)
    y, dx, dc, dwb = gpu_layer(cuda(x), cuda(coef), cuda(wb), cuda(dY), Ly.G, Ly.lo, Ly.hi,
                               path=N.KAN_PATH_TENSOR)
    torch.cuda.synchronize()
    assert N.kan_sync_status(None) == 0
    errs = check_layer_against_oracle(oracle, x, coef, wb, dY, Ly.G, Ly.lo, Ly.hi, y.cpu(), dx.cpu(), dc.cpu(),
                                      None, w.dtype)
    assert all(v <= TOL[w.dtype] for v in errs.values()), errs


def test_ffn_block_parity(oracle):
    w = W.WORKLOADS["ffn768_3072_bf16"]
    L1, L2 = w.layers
    d = W.draw_all(w)
    x, c1, c2, dY = d["x"], d["coef0"], d["coef1"], d["dY"]
    xg, c1g, c2g, dYg = cuda(x), cuda(c1), cuda(c2), cuda(dY)
    h = L.forward(xg, c1g, L1.G, L1.lo, L1.hi)
    y = L.forward(h, c2g, L2.G, L2.lo, L2.hi)
    dh, dc2, _ = L.backward(h, c2g, dYg, L2.G, L2.lo, L2.hi)
    dx, dc1, _ = L.backward(xg, c1g, dh, L1.G, L1.lo, L1.hi)
    torch.cuda.synchronize()
    assert N.kan_sync_status(None) == 0
    rows = np.union1d(tile_rows(w.batch), sample_rows(w.batch, 16))
    tol = TOL["bf16"]
    # per layer, each fed the GPU's own bf16 inputs; whole batch tiles, and dcoef for every output of the
    # inputs of whole M tiles
    e1 = check_layer_against_oracle(oracle, x, c1, None, dh.cpu(), L1.G, L1.lo, L1.hi, h.cpu(), dx.cpu(), dc1.cpu(),
                                    None, "bf16", rows=rows, cols_in=tile_inputs(L1.inp, L1.G + 3),
                                    cols_out=np.arange(L1.out))
    e2 = check_layer_against_oracle(oracle, h.cpu(), c2, None, dY, L2.G, L2.lo, L2.hi, y.cpu(), dh.cpu(), dc2.cpu(),
                                    None, "bf16", rows=rows, cols_in=tile_inputs(L2.inp, L2.G + 3),
                                    cols_out=np.arange(L2.out))
    # end to end, the oracle's h in fp64 (not re-rounded)
    h_ref = oracle.forward(x[rows], c1, L1.G, L1.lo, L1.hi)
    y_ref = oracle.forward(h_ref, c2, L2.G, L2.lo, L2.hi)
    e_end = rel_err(f64(y.cpu()[rows]), y_ref)
    assert all(v <= tol for v in e1.values()), e1
    assert all(v <= tol for v in e2.values()), e2
    assert e_end <= tol, e_end


# dcoef with the outputs on M and the spline columns on N (the plan takes it for bf16 layers whose `out`
# 512-column tiles would pad, when its waves of 512-column pair tiles are fewer): a ragged batch (last
# k-block), a ragged last M tile (out = 648), a ragged last N tile (in * (G+3) not a multiple of 512),
# rows of x not 16-byte aligned (the general producer) and G = 8 (11 columns per input)
DCB_CASES = [
    # batch, in, out, G, lo, hi
    (300, 1536, 648, 5, -3.0, 3.0),
    (257, 1532, 768, 5, -3.0, 3.0),
    (300, 1024, 768, 8, -1.0, 1.0),
]


@pytest.mark.parametrize("case", DCB_CASES, ids=lambda c: "b{}_i{}_o{}_g{}".format(*c[:4]))
def test_dcoef_outputs_on_m(oracle, case):
    batch, n_in, n_out, G, lo, hi = case
    w = W.custom(batch, n_in, n_out, G, lo, hi, dtype="bf16")
    x, coef, _, dY = workload_inputs(w)
    y, dx, dc, _ = gpu_layer(cuda(x), cuda(coef), None, cuda(dY), G, lo, hi)
    torch.cuda.synchronize()
    assert N.kan_sync_status(None) == 0
    nb = G + 3
    kt = n_in * nb
    # the inputs of the first 512-column tile (both CTAs' halves), of one in the middle and of the last
    # (ragged) one; every output, the padded M rows included
    mid = (kt // 2) // 512 * 512
    cols = np.concatenate([np.arange(512), np.arange(mid, mid + 512), np.arange((kt - 1) // 512 * 512, kt)])
    ci = np.unique(cols // nb)
    rows = np.union1d(tile_rows(batch), sample_rows(batch))
    errs = check_layer_against_oracle(oracle, x, coef, None, dY, G, lo, hi, y.cpu(), dx.cpu(), dc.cpu(), None,
                                      "bf16", rows=rows, cols_in=ci, cols_out=np.arange(n_out))
    assert all(v <= TOL["bf16"] for v in errs.values()), errs
    # bitwise repeatable
    _, _, dc2, _ = gpu_layer(cuda(x), cuda(coef), None, cuda(dY), G, lo, hi)
    torch.cuda.synchronize()
    assert torch.equal(dc, dc2)


# ---------------------------------------------------------------------------
# properties that hold at any size
@pytest.mark.parametrize("path", ["tensor", "simt"])
def test_marsden_cubic_closed_form(path):
    # fp32: coef[j,i,m] = psi_m(y_ji) = (y-t_{m+1})(y-t_{m+2})(y-t_{m+3})
    # reproduces y[b,j] = sum_i (y_ji - x_bi)^3 and dx = -3 sum_j dY (y_ji - x_bi)^2
    # for x in [lo,hi] (Marsden's identity), at any batch size.
    G, lo, hi = 8, -1.0, 1.0
    batch, n_in, n_out = (1000 if path == "simt" else 16384), 32, 96
    g = torch.Generator().manual_seed(5)
    x = torch.rand(batch, n_in, generator=g) * 2 - 1
    yt = (torch.rand(n_out, n_in, generator=g) * 0.5 - 0.25).double().numpy()
    coef = torch.from_numpy(pins.marsden_coef(yt, G, lo, hi)).float()
    dY = torch.randn(batch, n_out, generator=g)
    y, dx, _, _ = gpu_layer(cuda(x), cuda(coef), None, cuda(dY), G, lo, hi, path=PATHS[path])
    xd = f64(x)
    ref = ((yt[None, :, :] - xd[:, None, :]) ** 3).sum(2)
    dref = np.einsum("bj,bji->bi", f64(dY), -3.0 * (yt[None, :, :] - xd[:, None, :]) ** 2)
    assert rel_err(f64(y.cpu()), ref) <= TOL["f32"]
    assert rel_err(f64(dx.cpu()), dref) <= TOL["f32"]


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("path", ["tensor", "simt"])
def test_linear_reproduction_closed_form(path, dt):
    # coef[j,i,m] = a_ji * t_{m+2} + c_ji (Greville abscissae of the uniform
    # cubic B-splines are the middle knots): sum_m coef B_m(x) = a x + c on
    # [lo,hi], so y = x a^T + sum_i c and dx = dY a.  Every coefficient is a
    # multiple of 1/64 below 4 in magnitude, exact in bf16.
    G, lo, hi = 8, -1.0, 1.0
    batch, n_in, n_out = (512 if path == "simt" else 16384), 256, 320
    g = torch.Generator().manual_seed(6)
    x = (torch.rand(batch, n_in, generator=g) * 2 - 1).to(DT[dt])
    a = (torch.randint(-4, 5, (n_out, n_in), generator=g) / 4.0).double()
    c = (torch.randint(-4, 5, (n_out, n_in), generator=g) / 16.0).double()
    t = torch.tensor(pins.knots_np(G, lo, hi), dtype=torch.float64)
    coef = (a[:, :, None] * t[2:G + 5][None, None, :] + c[:, :, None]).to(DT[dt])
    assert torch.equal(coef.double(), a[:, :, None] * t[2:G + 5][None, None, :] + c[:, :, None])
    dY = torch.randn(batch, n_out, generator=g).to(DT[dt])
    y, dx, _, _ = gpu_layer(cuda(x), cuda(coef), None, cuda(dY), G, lo, hi, path=PATHS[path])
    xd, dYd = x.double(), dY.double()
    ref = (xd @ a.T + c.sum(1)[None, :]).numpy()
    dref = (dYd @ a).numpy()
    assert rel_err(f64(y.cpu()), ref) <= TOL[dt]
    assert rel_err(f64(dx.cpu()), dref) <= TOL[dt]


@pytest.mark.parametrize("name", ["layer784x64_silu", "layer1024_g20_bf16", "sweep512_g50_f32_fwdbwd"])
def test_adjoint_identity_full_size(name):
    w = W.WORKLOADS[name]
    Ly = w.layers[0]
    x, coef, wb, dY = workload_inputs(w)
    y, dx, dc, dwb = gpu_layer(cuda(x), cuda(coef), cuda(wb), cuda(dY), Ly.G, Ly.lo, Ly.hi)
    lhs = (cuda(dY).double() * y.double()).sum().item()
    rhs = (dc.double() * cuda(coef).double()).sum().item()
    if dwb is not None:
        rhs += (dwb.double() * cuda(wb).double()).sum().item()
    scale = (cuda(dY).double() * y.double()).abs().sum().item()
    assert abs(lhs - rhs) <= TOL[w.dtype] * scale


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_one_hot_coef_returns_basis(oracle, dt):
    G, lo, hi = 20, -1.0, 1.0
    batch, n_in, n_out = 512, 16, 64
    g = torch.Generator().manual_seed(9)
    x = (torch.rand(batch, n_in, generator=g) * 2.4 - 1.2).to(DT[dt])
    coef = torch.zeros(n_out, n_in, G + 3)
    picks = [(j, (j * 7) % n_in, (j * 5) % (G + 3)) for j in range(n_out)]
    for j, i, m in picks:
        coef[j, i, m] = 1.0
    y = L.forward(cuda(x), cuda(coef.to(DT[dt])), G, lo, hi, path=N.KAN_PATH_TENSOR)
    B, _ = oracle.basis(f64(x).reshape(-1), G, lo, hi)
    B = B.reshape(batch, n_in, G + 3)
    ref = np.stack([B[:, i, m] for j, i, m in picks], axis=1)
    # bf16: basis rounded for the tensor core and y rounded at the store;
    # fp32: the fp32 rounding of the local coordinate (u up to G+3)
    tol = 2.0 ** -8 if dt == "bf16" else 1e-5
    assert np.max(np.abs(f64(y.cpu()) - ref)) <= tol


@pytest.mark.parametrize("name", ["layer784x64_silu", "layer1024_g20_bf16"])
def test_deterministic(name):
    w = W.WORKLOADS[name]
    Ly = w.layers[0]
    x, coef, wb, dY = [cuda(t) for t in workload_inputs(w)]
    first = gpu_layer(x, coef, wb, dY, Ly.G, Ly.lo, Ly.hi)
    for _ in range(10):
        again = gpu_layer(x, coef, wb, dY, Ly.G, Ly.lo, Ly.hi)
        for a, b in zip(first, again):
            if a is not None:
                assert torch.equal(a, b)


# ---------------------------------------------------------------------------
# edge cases
@pytest.mark.parametrize("path", ["tensor", "simt", "auto"])
def test_empty_batch(path):
    p = {"tensor": 1, "simt": 2, "auto": 0}[path]
    x = torch.empty(0, 16, device="cuda")
    coef = torch.randn(32, 16, 11, device="cuda")
    y = L.forward(x, coef, 8, -1.0, 1.0, path=p)
    assert y.shape == (0, 32)
    dY = torch.empty(0, 32, device="cuda")
    dx, dc, _ = L.backward(x, coef, dY, 8, -1.0, 1.0, path=p)
    assert dx.shape == (0, 16) and torch.all(dc == 0)


@pytest.mark.parametrize("path", ["tensor", "simt"])
def test_nonfinite_and_boundary_inputs(oracle, path):
    G, lo, hi = 20, -1.0, 1.0
    h = (hi - lo) / G
    g = torch.Generator().manual_seed(21)
    x = torch.rand(256, 16, generator=g) * 2 - 1
    special = [lo, hi, lo - 3 * h, hi + 3 * h, -1.3, 1.3, -1.31, 1.31, 5.0, -5.0, float("inf"), -float("inf"),
               float("nan"), 1e30]
    for k, v in enumerate(special):
        x[k % 256, k % 16] = v
    coef = torch.randn(64, 16, G + 3, generator=g) * 0.1
    dY = torch.randn(256, 64, generator=g)
    y, dx, dc, _ = gpu_layer(cuda(x), cuda(coef), None, cuda(dY), G, lo, hi, path=PATHS[path])
    torch.cuda.synchronize()
    # the oracle's basis is 0 for NaN and inf as well
    errs = check_layer_against_oracle(oracle, x, coef, None, dY, G, lo, hi, y.cpu(), dx.cpu(), dc.cpu(), None,
                                      "f32")
    assert np.all(np.isfinite(f64(y.cpu())))
    assert all(v <= TOL["f32"] for v in errs.values()), errs


def test_single_row_and_column(oracle):
    for (batch, n_in, n_out) in [(1, 4, 4), (3, 1, 4), (5, 4, 1)]:
        w = W.custom(batch, n_in, n_out, 8, -1.0, 1.0, dtype="f32", base=True)
        x, coef, wb, dY = workload_inputs(w)
        y, dx, dc, dwb = gpu_layer(cuda(x), cuda(coef), cuda(wb), cuda(dY), 8, -1.0, 1.0)
        errs = check_layer_against_oracle(oracle, x, coef, wb, dY, 8, -1.0, 1.0, y.cpu(), dx.cpu(), dc.cpu(),
                                          dwb.cpu(), "f32")
        assert all(v <= TOL["f32"] for v in errs.values()), (batch, n_in, n_out, errs)


# ---------------------------------------------------------------------------
# failure path: a bounded device wait that runs out
def test_device_wait_timeout_is_reported():
    assert N.kan_sync_status(None) == 0
    N.kan_selftest_wait_timeout(20_000_000, None)   # 20 ms
    assert N.kan_sync_status(None) == 5             # KAN_ERR_TIMEOUT
    assert N.kan_sync_status(None) == 0             # cleared
    # the context is still usable
    x = torch.rand(64, 8, device="cuda") * 2 - 1
    coef = torch.randn(16, 8, 11, device="cuda")
    y = L.forward(x, coef, 8, -1.0, 1.0)
    torch.cuda.synchronize()
    assert torch.isfinite(y).all()


# ---------------------------------------------------------------------------
# drop-in module with autograd
def test_kan_layer_autograd(oracle):
    torch.manual_seed(0)
    layer = L.KANLayer(8, 4, base=True).cuda()
    x = (torch.rand(32, 8, device="cuda") * 2 - 1).requires_grad_(True)
    y = layer(x)
    assert y.shape == (32, 4)
    g = torch.randn_like(y)
    y.backward(g)
    xc, cc, wbc, gc = x.detach().cpu(), layer.coef.detach().cpu(), layer.w_base.detach().cpu(), g.cpu()
    y_ref = oracle.forward(xc, cc, 8, -1.0, 1.0, w_base=wbc)
    dx_ref, dc_ref, dwb_ref = oracle.backward(xc, cc, gc, 8, -1.0, 1.0, w_base=wbc)
    assert rel_err(f64(y.detach().cpu()), y_ref) <= 1e-5
    assert rel_err(f64(x.grad.cpu()), dx_ref) <= 1e-5
    assert rel_err(f64(layer.coef.grad.cpu()), dc_ref) <= 1e-5
    assert rel_err(f64(layer.w_base.grad.cpu()), dwb_ref) <= 1e-5

"""Helpers of the GPU parity tests: running the library on workload inputs and
comparing with the fp64 oracle."""
from __future__ import annotations

import numpy as np
import torch

from kolmogorov_arnold_network_b200 import layer as L
from kolmogorov_arnold_network_b200 import workloads as W

#: normwise max-relative error bound per operand dtype (max|g-r| / max|r|)
TOL = {"f32": 1e-5, "bf16": 2e-2}


def rel_err(g, r) -> float:
    g = np.asarray(g, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    scale = float(np.max(np.abs(r))) if r.size else 0.0
    diff = float(np.max(np.abs(g - r))) if r.size else 0.0
    return diff / scale if scale > 0 else diff


def f64(t) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def cuda(t):
    return None if t is None else t.to("cuda").contiguous()


def sample_rows(batch, n=24, seed=0):
    rng = np.random.default_rng(seed)
    k = min(n, batch)
    rows = set(rng.choice(batch, size=k, replace=False).tolist())
    rows.update({0, batch - 1})
    return np.array(sorted(rows))


def sample_cols(n, k=12, seed=1):
    rng = np.random.default_rng(seed)
    c = set(rng.choice(n, size=min(k, n), replace=False).tolist())
    c.update({0, n - 1})
    return np.array(sorted(c))


def tile_rows(batch, tile=128):
    """Every row of the first two batch tiles (a whole CTA pair of the paired kernels) and of the last
    batch tile (ragged or not)."""
    first = np.arange(min(batch, 2 * tile))
    last = np.arange(((batch - 1) // tile) * tile, batch)
    return np.unique(np.concatenate([first, last]))


def tile_inputs(n_in, nb, tile=128):
    """The inputs whose basis columns (nb per input) fall in the first four 128-column tiles of the
    dcoef GEMM (a whole CTA pair of 128-column M tiles, and a whole 512-column N tile when the spline
    columns run along N) or in its last 128-column tile."""
    kt = n_in * nb
    cols = np.concatenate([np.arange(min(kt, 4 * tile)), np.arange(((kt - 1) // tile) * tile, kt)])
    return np.unique(cols // nb)


def gpu_layer(x, coef, w_base, dY, G, lo, hi, path=0, want_bwd=True, degree=3):
    """Run forward (+ backward) through the C ABI on CUDA tensors; returns CUDA tensors."""
    y = L.forward(x, coef, G, lo, hi, w_base, path=path, degree=degree)
    if not want_bwd:
        return y, None, None, None
    dx, dcoef, dwb = L.backward(x, coef, dY, G, lo, hi, w_base, path=path, degree=degree)
    return y, dx, dcoef, dwb


def check_layer_against_oracle(o, x, coef, w_base, dY, G, lo, hi, y, dx, dcoef, dwb, dtype, rows=None,
                               cols_in=None, cols_out=None, k=3):
    """Compare GPU outputs (CPU tensors) with the oracle, on sampled rows / (j, i) slices if given.

    Returns a dict of errors."""
    errs = {}
    xr = x if rows is None else x[rows]
    dYr = dY if rows is None else dY[rows]
    y_ref = o.forward(xr, coef, G, lo, hi, w_base=w_base, k=k)
    errs["y"] = rel_err(f64(y if rows is None else y[rows]), y_ref)
    if dx is not None:
        dx_ref, _, _ = o.backward(xr, coef, dYr, G, lo, hi, w_base=w_base, want_dcoef=False, want_dw_base=False,
                                  k=k)
        errs["dx"] = rel_err(f64(dx if rows is None else dx[rows]), dx_ref)
    if dcoef is not None:
        if cols_in is None:
            _, dc_ref, dwb_ref = o.backward(x, coef, dY, G, lo, hi, w_base=w_base, want_dx=False, k=k)
            errs["dcoef"] = rel_err(f64(dcoef), dc_ref)
            if dwb is not None:
                errs["dw_base"] = rel_err(f64(dwb), dwb_ref)
        else:
            xs = x[:, cols_in]
            dYs = dY[:, cols_out]
            cs = coef[cols_out][:, cols_in]
            wbs = None if w_base is None else w_base[cols_out][:, cols_in]
            _, dc_ref, dwb_ref = o.backward(xs, cs, dYs, G, lo, hi, w_base=wbs, want_dx=False, k=k)
            errs["dcoef"] = rel_err(f64(dcoef[cols_out][:, cols_in]), dc_ref)
            if dwb is not None:
                errs["dw_base"] = rel_err(f64(dwb[cols_out][:, cols_in]), dwb_ref)
    return errs


def workload_inputs(w: W.Workload, layer=0):
    d = W.draw_all(w)
    return d["x"], d[f"coef{layer}"], d[f"w_base{layer}"], d["dY"]

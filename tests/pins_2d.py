"""Pins of the 2-D (tensor-product surface) oracle, oracle/kan2d.py: facts that do not come from it.

  T1  Marsden's identity in each coordinate: coef[j,p,m1,m2] = psi_m1(s) psi_m2(r)
      with psi_m(y) = prod_{l=1..k} (y - t_{m+l}) reproduces
      y = sum_p (s_jp - u)^k (r_jp - v)^k, and both dx entries in closed form
      (u, v in [lo, hi]).
  T2  partition of unity: coef = 1 gives y = in/2 and dx = 0 on [lo, hi]^2.
  T3  a surface constant along its second coordinate is the 1-D spline of the
      first: coef[j,p,m1,m2] = c[j,p,m1] gives the 1-D layer on x[:, 0::2]
      (the 1-D oracle, pinned on its own); dx[:, 1::2] = 0.
  T4  central finite differences of <dY, y(x)> against dx.
  T5  y is linear in coef: <dY, y(coef + E)> - <dY, y(coef)> = <dcoef, E>.
"""
from __future__ import annotations

import numpy as np

import pins


def _problem(rng, G=6, lo=-1.0, hi=1.0, batch=11, n_in=6, n_out=3, k=3):
    h = (hi - lo) / G
    x = rng.uniform(lo - 2 * h, hi + 2 * h, size=(batch, n_in))
    coef = rng.normal(0, 0.3, size=(n_out, n_in // 2, G + k, G + k))
    dY = rng.normal(size=(batch, n_out))
    return x, coef, dY


def pin_marsden(m, rng=None, k=3):
    rng = rng or np.random.default_rng(41)
    for G, lo, hi in ((8, -1.0, 1.0), (5, -3.0, 3.0)):
        batch, n_in, n_out = 23, 6, 2
        x = rng.uniform(lo, hi, size=(batch, n_in))
        s = rng.uniform(-2, 2, size=(n_out, n_in // 2))
        r = rng.uniform(-2, 2, size=(n_out, n_in // 2))
        ps = pins.marsden_coef(s, G, lo, hi, k)          # [out, pairs, nb]
        pr = pins.marsden_coef(r, G, lo, hi, k)
        coef = ps[:, :, :, None] * pr[:, :, None, :]
        u, v = x[:, 0::2], x[:, 1::2]
        fu = s[None] - u[:, None, :]                      # [batch, out, pairs]
        fv = r[None] - v[:, None, :]
        ref = (fu ** k * fv ** k).sum(2)
        y = m.forward(x, coef, G, lo, hi, k=k)
        if np.max(np.abs(y - ref)) > 1e-11 * max(1.0, np.max(np.abs(ref))):
            return f"T1 k={k} G={G}: forward != sum_p (s-u)^k (r-v)^k"
        dY = rng.normal(size=(batch, n_out))
        dx, _ = m.backward(x, coef, dY, G, lo, hi, k=k, want_dcoef=False)
        du = np.einsum("bj,bjp->bp", dY, -k * fu ** (k - 1) * fv ** k)
        dv = np.einsum("bj,bjp->bp", dY, -k * fu ** k * fv ** (k - 1))
        scale = max(1.0, np.max(np.abs(du)), np.max(np.abs(dv)))
        if np.max(np.abs(dx[:, 0::2] - du)) > 1e-10 * scale or np.max(np.abs(dx[:, 1::2] - dv)) > 1e-10 * scale:
            return f"T1 k={k} G={G}: dx differs from the closed form"
    return None


def pin_partition(m, rng=None):
    rng = rng or np.random.default_rng(42)
    G, lo, hi = 7, -1.0, 1.0
    x = rng.uniform(lo, hi, size=(9, 8))
    coef = np.ones((2, 4, G + 3, G + 3))
    y = m.forward(x, coef, G, lo, hi)
    dx, _ = m.backward(x, coef, rng.normal(size=(9, 2)), G, lo, hi, want_dcoef=False)
    if np.max(np.abs(y - 4.0)) > 1e-13 or np.max(np.abs(dx)) > 1e-12:
        return "T2: all-ones surfaces do not give y = pairs, dx = 0 inside the grid"
    return None


def pin_reduces_to_1d(m, o1, rng=None):
    rng = rng or np.random.default_rng(43)
    G, lo, hi = 8, -1.0, 1.0
    batch, n_in, n_out = 13, 6, 3
    x = rng.uniform(lo - 0.2, hi + 0.2, size=(batch, n_in))
    x[:, 1::2] = rng.uniform(lo, hi, size=(batch, n_in // 2))   # v inside: sum_m2 B_m2(v) = 1
    c = rng.normal(size=(n_out, n_in // 2, G + 3))
    coef = np.repeat(c[:, :, :, None], G + 3, axis=3)
    y = m.forward(x, coef, G, lo, hi)
    ref = o1.forward(x[:, 0::2], c, G, lo, hi)
    if np.max(np.abs(y - ref)) > 1e-12 * max(1.0, np.max(np.abs(ref))):
        return "T3: surface constant in v differs from the 1-D layer on u"
    dY = rng.normal(size=(batch, n_out))
    dx, _ = m.backward(x, coef, dY, G, lo, hi, want_dcoef=False)
    dref, _, _ = o1.backward(x[:, 0::2], c, dY, G, lo, hi, want_dcoef=False, want_dw_base=False)
    if np.max(np.abs(dx[:, 0::2] - dref)) > 1e-11 * max(1.0, np.max(np.abs(dref))):
        return "T3: dx of u differs from the 1-D layer's"
    if np.max(np.abs(dx[:, 1::2])) > 1e-11:
        return "T3: dx of v is not 0 for a surface constant in v"
    return None


def pin_finite_difference(m, rng=None):
    rng = rng or np.random.default_rng(44)
    G, lo, hi = 6, -1.0, 1.0
    x, coef, dY = _problem(rng, G, lo, hi)
    dx, _ = m.backward(x, coef, dY, G, lo, hi, want_dcoef=False)
    eps = 1e-6
    fd = np.zeros_like(x)
    for b in range(x.shape[0]):
        for i in range(x.shape[1]):
            xp = x[b:b + 1].copy(); xp[0, i] += eps
            xm = x[b:b + 1].copy(); xm[0, i] -= eps
            fd[b, i] = float(((m.forward(xp, coef, G, lo, hi) - m.forward(xm, coef, G, lo, hi)) * dY[b]).sum()) / (2 * eps)
    err = np.max(np.abs(fd - dx)) / np.max(np.abs(dx))
    return None if err <= 1e-7 else f"T4: dx vs central differences rel err {err:.2e}"


def pin_linear(m, rng=None):
    rng = rng or np.random.default_rng(45)
    G, lo, hi = 6, -1.0, 1.0
    x, coef, dY = _problem(rng, G, lo, hi)
    _, dcoef = m.backward(x, coef, dY, G, lo, hi, want_dx=False)
    E = rng.normal(size=coef.shape)
    lhs = float((dY * (m.forward(x, coef + E, G, lo, hi) - m.forward(x, coef, G, lo, hi))).sum())
    rhs = float((dcoef * E).sum())
    return None if abs(lhs - rhs) <= 1e-10 * max(1.0, abs(lhs)) else f"T5: {lhs} != <dcoef, E> = {rhs}"


def run_all(m, o1):
    fails = []
    for p in (pin_marsden, pin_partition, pin_finite_difference, pin_linear):
        try:
            r = p(m)
        except Exception as e:
            r = f"{p.__name__} raised {type(e).__name__}: {e}"
        if r:
            fails.append(r)
    try:
        r = pin_reduces_to_1d(m, o1)
    except Exception as e:
        r = f"pin_reduces_to_1d raised {type(e).__name__}: {e}"
    if r:
        fails.append(r)
    return fails

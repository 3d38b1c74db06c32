"""Pins of the GR-KAN oracle (oracle/grkan.py): checks against facts that do not come from it.

Each pin takes the oracle module (so that the mutation test can run the same
pins on deliberately broken copies) and returns None or a failure string.

  R1  b = 0 reduces phi to the polynomial P: numpy's polyval and polyder
      (library routines) give y and dx.
  R2  m = n = 1, a = (0, 1), b = (1): phi(x) = x / (1 + |x|), torch's softsign
      (library), and its derivative by torch autograd.
  R3  central finite differences of <dY, y> against dx, da and db (tiny
      inputs, fp64, away from S(x) = 0 where |S| has a kink).
  R4  phi is linear in a: <dY, y(a + E)> - <dY, y(a)> = <da, E> exactly.
  R5  groups: with every group given the same coefficients, the group
      gradients sum to those of one group over all channels; changing one
      group's coefficients changes only that group's channels.
"""
from __future__ import annotations

import numpy as np


def _problem(rng, rows=9, C=12, groups=3, m=5, n=4, scale=1.0):
    x = rng.normal(0, scale, size=(rows, C))
    a = rng.normal(0, 0.5, size=(groups, m + 1))
    b = rng.normal(0, 0.5, size=(groups, n))
    dY = rng.normal(size=(rows, C))
    return x, a, b, dY


def pin_polynomial(g, rng=None):
    rng = rng or np.random.default_rng(31)
    x, a, _, dY = _problem(rng)
    b = np.zeros((3, 4))
    y = g.forward(x, a, b, 3)
    dx, _, _ = g.backward(x, a, b, dY, 3)
    cg = x.shape[1] // 3
    for grp in range(3):
        sl = slice(grp * cg, (grp + 1) * cg)
        ref = np.polynomial.polynomial.polyval(x[:, sl], a[grp])
        dref = dY[:, sl] * np.polynomial.polynomial.polyval(x[:, sl], np.polynomial.polynomial.polyder(a[grp]))
        if np.max(np.abs(y[:, sl] - ref)) > 1e-12 * max(1.0, np.max(np.abs(ref))):
            return f"R1 group {grp}: phi with b = 0 differs from polyval"
        if np.max(np.abs(dx[:, sl] - dref)) > 1e-12 * max(1.0, np.max(np.abs(dref))):
            return f"R1 group {grp}: dx with b = 0 differs from polyder"
    return None


def pin_softsign(g):
    import torch
    xs = torch.linspace(-6, 6, 2001, dtype=torch.float64, requires_grad=True)
    ys = torch.nn.functional.softsign(xs)
    (gr,) = torch.autograd.grad(ys.sum(), xs)
    x = xs.detach().numpy().reshape(1, -1)
    a = np.array([[0.0, 1.0]])
    b = np.array([[1.0]])
    y = g.forward(x, a, b, 1)
    dx, _, _ = g.backward(x, a, b, np.ones_like(x), 1)
    if np.max(np.abs(y - ys.detach().numpy())) > 1e-15:
        return "R2: x / (1 + |x|) differs from torch softsign"
    if np.max(np.abs(dx - gr.numpy())) > 1e-15:
        return "R2: derivative differs from torch autograd of softsign"
    return None


def pin_finite_difference(g, rng=None):
    rng = rng or np.random.default_rng(32)
    x, a, b, dY = _problem(rng, rows=5, C=8, groups=2)
    dx, da, db = g.backward(x, a, b, dY, 2)
    eps = 1e-6

    def f(xx, aa, bb):
        return float(np.sum(g.forward(xx, aa, bb, 2) * dY))

    # keep away from the kink of |S| (S changes sign within eps)
    cg = 4
    for r in range(x.shape[0]):
        for c in range(x.shape[1]):
            grp = c // cg
            s = lambda v: sum(b[grp, q] * v ** (q + 1) for q in range(b.shape[1]))
            if np.sign(s(x[r, c] - 2 * eps)) != np.sign(s(x[r, c] + 2 * eps)):
                continue
            xp = x.copy(); xp[r, c] += eps
            xm = x.copy(); xm[r, c] -= eps
            fd = (f(xp, a, b) - f(xm, a, b)) / (2 * eps)
            if abs(fd - dx[r, c]) > 1e-6 * max(1.0, abs(dx[r, c])):
                return f"R3: dx[{r},{c}] = {dx[r, c]} vs finite difference {fd}"
    for arr, grad, nm in ((a, da, "da"), (b, db, "db")):
        for idx in np.ndindex(arr.shape):
            ap = arr.copy(); ap[idx] += eps
            am = arr.copy(); am[idx] -= eps
            if nm == "da":
                fd = (f(x, ap, b) - f(x, am, b)) / (2 * eps)
            else:
                fd = (f(x, a, ap) - f(x, a, am)) / (2 * eps)
            if abs(fd - grad[idx]) > 1e-6 * max(1.0, abs(grad[idx])):
                return f"R3: {nm}{idx} = {grad[idx]} vs finite difference {fd}"
    return None


def pin_linear_in_a(g, rng=None):
    rng = rng or np.random.default_rng(33)
    x, a, b, dY = _problem(rng, rows=40, C=24, groups=4)
    _, da, _ = g.backward(x, a, b, dY, 4)
    E = rng.normal(size=a.shape)
    lhs = float(np.sum(dY * g.forward(x, a + E, b, 4)) - np.sum(dY * g.forward(x, a, b, 4)))
    rhs = float(np.sum(da * E))
    if abs(lhs - rhs) > 1e-10 * max(1.0, abs(lhs)):
        return f"R4: <dY, y(a+E) - y(a)> = {lhs} != <da, E> = {rhs}"
    return None


def pin_groups(g, rng=None):
    rng = rng or np.random.default_rng(34)
    x, a, b, dY = _problem(rng, rows=30, C=24, groups=4)
    a_same = np.repeat(a[:1], 4, axis=0)
    b_same = np.repeat(b[:1], 4, axis=0)
    _, da4, db4 = g.backward(x, a_same, b_same, dY, 4)
    _, da1, db1 = g.backward(x, a[:1], b[:1], dY, 1)
    if np.max(np.abs(da4.sum(0) - da1[0])) > 1e-10 * max(1.0, np.max(np.abs(da1))):
        return "R5: group da do not sum to the one-group da"
    if np.max(np.abs(db4.sum(0) - db1[0])) > 1e-10 * max(1.0, np.max(np.abs(db1))):
        return "R5: group db do not sum to the one-group db"
    y0 = g.forward(x, a, b, 4)
    a2 = a.copy(); a2[2] += 1.0
    b2 = b.copy(); b2[2] += 0.5
    y1 = g.forward(x, a2, b2, 4)
    changed = np.any(y1 != y0, axis=0)
    want = np.zeros(24, dtype=bool); want[12:18] = True
    if not np.array_equal(changed, want):
        return "R5: changing group 2's coefficients changed channels outside 12..17 (or not all of them)"
    return None


ALL_PINS = [pin_polynomial, pin_softsign, pin_finite_difference, pin_linear_in_a, pin_groups]


def run_all(g):
    fails = []
    for p in ALL_PINS:
        try:
            r = p(g)
        except Exception as e:  # a crashing mutant counts as detected
            r = f"{p.__name__} raised {type(e).__name__}: {e}"
        if r:
            fails.append(r)
    return fails

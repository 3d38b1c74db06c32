"""Pins of the fp64 oracle: checks against facts that do not come from the oracle.

Each pin returns ``None`` on success or a short failure string.  They take an
``oracle.Oracle`` instance so that the mutation test can run the same pins on
deliberately broken builds of the oracle.

Sources of the facts:
  P1  truncated power closed form of the uniform B-spline on the bounded
      coordinate v in [0, k+1] (FlashKAN abstract, mlsift "GPU kernel"
      listing), written independently here in numpy.
  P2  partition of unity inside [lo, hi] (textbook), < 1 in the extended
      intervals, 0 beyond them.
  P3  non-negativity (InKAN landing page, "Numerically Stable"), local
      support over 4 knot intervals (InKAN landing page, "What is a KAN?").
  P4  exact local weights of the uniform cubic B-spline
      (tests/golden/cubic_bspline_local_weights.txt); for degrees 1-5, the
      weights at a knot (Eulerian numbers over k!, textbook).
  P5  Marsden's identity, degree-k polynomial reproduction (textbook),
      through the layer forward and dx.
  P6  finite differences of <dY, y(x)> against dx.
  P7  dcoef and dw_base entries equal <dY, y(one-hot parameter)>.
  P8  bilinear adjoint identity <dY, y> = <dcoef, coef> + <dw_base, w_base>.
  P9  the dense basis expansion times a library matmul equals the forward;
      dcoef equals A^T dY by library matmul; silu against torch.
  P10 one-hot coefficients return the basis value itself.
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "cubic_bspline_local_weights.txt")


def knots_np(G, lo, hi, k=3):
    h = (hi - lo) / G
    return lo + (np.arange(G + 2 * k + 1) - k) * h


def truncated_power_basis(x, G, lo, hi, k=3):
    """B_m(x) = (1/k!) sum_q (-1)^q C(k+1,q) (v-q)_+^k, v = clamp((x-t_m)/h, 0, k+1).

    The closed form on the bounded coordinate (FlashKAN abstract).  Beyond
    the last knot of B_m's support v is clamped to k+1 where the sum is 0
    in exact arithmetic; it is set to 0 explicitly there to keep the check
    free of cancellation noise.
    """
    x = np.asarray(x, dtype=np.float64).reshape(-1)
    h = (hi - lo) / G
    t = knots_np(G, lo, hi, k)
    out = np.zeros((x.size, G + k))
    for m in range(G + k):
        v = np.clip((x - t[m]) / h, 0.0, k + 1.0)
        acc = np.zeros_like(v)
        for q in range(k + 2):
            acc += (-1) ** q * math.comb(k + 1, q) * np.maximum(v - q, 0.0) ** k
        acc /= math.factorial(k)
        acc[(v <= 0.0) | (v >= k + 1.0)] = 0.0
        out[:, m] = acc
    return out


def _sweep(G, lo, hi, k=3, n=4001):
    t = knots_np(G, lo, hi, k)
    h = (hi - lo) / G
    dense = np.linspace(t[0] - 2 * h, t[-1] + 2 * h, n)
    mids = (t[:-1] + t[1:]) / 2
    return np.concatenate([dense, t, mids, [-np.inf, np.inf]])


# ----------------------------------------------------------------------------
def pin_truncated_power(o, grids=((8, -1.0, 1.0), (20, -1.0, 1.0), (5, -3.0, 3.0), (50, -1.0, 1.0)),
                        degrees=(3,)):
    for k in degrees:
        for G, lo, hi in grids:
            x = _sweep(G, lo, hi, k)
            B, _ = o.basis(x, G, lo, hi, k=k)
            ref = truncated_power_basis(x, G, lo, hi, k)
            tol = 1e-13 * (k + 1) ** k / math.factorial(k) * 2
            err = np.max(np.abs(B - ref))
            if not err <= tol:
                return f"P1 k={k} G={G}: max |CoxdeBoor - truncated power| = {err:.3e} > {tol:.1e}"
    return None


def pin_partition_of_unity(o, grids=((8, -1.0, 1.0), (20, -1.0, 1.0), (5, -3.0, 3.0)), k=3):
    for G, lo, hi in grids:
        h = (hi - lo) / G
        inside = np.linspace(lo, hi, 2001)
        B, dB = o.basis(inside, G, lo, hi, k=k)
        if np.max(np.abs(B.sum(1) - 1.0)) > 1e-14:
            return f"P2 G={G}: sum B != 1 inside [lo,hi]"
        # (degree 1 is not differentiable at the knots; with half-open intervals its derivative at
        # x = hi is the right-hand one, taken in the extended interval, so hi itself is left out)
        dsum = dB.sum(1) if k > 1 else dB[:-1].sum(1)
        if np.max(np.abs(dsum)) * h > 1e-13:
            return f"P2 G={G}: sum B' != 0 inside [lo,hi]"
        ext = np.concatenate([np.linspace(lo - k * h, lo, 200, endpoint=False)[1:],
                              np.linspace(hi, hi + k * h, 200, endpoint=False)[1:]])
        Be, _ = o.basis(ext, G, lo, hi, k=k)
        s = Be.sum(1)
        if not (np.all(s < 1.0 - 1e-15) and np.all(s > 0.0)):
            return f"P2 G={G}: sum B not in (0,1) in the extended intervals"
        beyond = np.array([lo - k * h - 1e-9, lo - k * h - 0.5, hi + k * h + 1e-9, hi + k * h + 0.3, -np.inf, np.inf])
        Bb, dBb = o.basis(beyond, G, lo, hi, k=k)
        if np.any(Bb != 0.0) or np.any(dBb != 0.0):
            return f"P2 G={G}: basis not zero beyond the extended knots"
    return None


def pin_nonneg_local(o, grids=((8, -1.0, 1.0), (20, -1.0, 1.0), (5, -3.0, 3.0)), k=3):
    # the cubic B-spline peaks at 2/3 (its value at the middle knot); any degree stays within [0, 1]
    top = 2.0 / 3.0 if k == 3 else 1.0
    for G, lo, hi in grids:
        x = _sweep(G, lo, hi, k)
        B, _ = o.basis(x, G, lo, hi, k=k)
        if np.any(B < 0.0) or np.any(B > top + 1e-15):
            return f"P3 k={k} G={G}: basis outside [0, {top}]"
        if np.max((B != 0.0).sum(1)) > k + 1:
            return f"P3 G={G}: more than k+1 non-zero basis values"
        t = knots_np(G, lo, hi, k)
        for m in range(G + k):
            # knots here and in the oracle may differ by an ulp: leave out
            # points within 1e-12 of the support's ends
            outside = (x < t[m] - 1e-12) | (x >= t[m + k + 1] + 1e-12)
            if np.any(B[outside, m] != 0.0):
                return f"P3 G={G}: B_{m} non-zero outside [t_m, t_(m+4))"
    return None


def read_golden():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            rows.append([Fraction(tok) for tok in line.split()])
    return rows


def pin_exact_values(o):
    rows = read_golden()
    for G, lo, hi in ((8, -1.0, 1.0), (4, 0.0, 1.0)):
        h = (hi - lo) / G
        for s in (-3, 0, 2, G - 1, G + 2):
            for row in rows:
                u = float(row[0])
                x = lo + (s + u) * h
                B, dB = o.basis([x], G, lo, hi)
                for r in range(4):
                    m = s + r
                    if 0 <= m <= G + 2:
                        if abs(B[0, m] - float(row[1 + r])) > 1e-15:
                            return f"P4 G={G} s={s} u={u}: B_{m} = {B[0, m]!r} != {row[1 + r]}"
                        if abs(dB[0, m] * h - float(row[5 + r])) > 1e-14:
                            return f"P4 G={G} s={s} u={u}: h*B'_{m} = {dB[0, m] * h!r} != {row[5 + r]}"
    return None


def marsden_coef(targets, G, lo, hi, k=3):
    """coef[j,i,m] = psi_m(y_ji) = prod_{l=1..k} (y - t_{m+l}) for y = targets[j,i] (Marsden's identity:
    sum_m psi_m(y) B_m(x) = (y - x)^k for x in [lo, hi], degree-k B-splines)."""
    t = knots_np(G, lo, hi, k)
    y = np.asarray(targets, dtype=np.float64)[..., None]
    m = np.arange(G + k)
    out = np.ones(y.shape[:-1] + (G + k,))
    for l in range(1, k + 1):
        out = out * (y - t[m + l])
    return out


def pin_marsden(o, rng=None, k=3):
    rng = rng or np.random.default_rng(11)
    for G, lo, hi in ((8, -1.0, 1.0), (5, -3.0, 3.0), (20, -1.0, 1.0)):
        batch, n_in, n_out = 37, 6, 3
        x = rng.uniform(lo, hi, size=(batch, n_in))
        x[0, 0], x[1, 1] = lo, hi - 1e-12
        yt = rng.uniform(-2, 2, size=(n_out, n_in))
        coef = marsden_coef(yt, G, lo, hi, k)
        y = o.forward(x, coef, G, lo, hi, k=k)
        ref = ((yt[None, :, :] - x[:, None, :]) ** k).sum(2)
        if np.max(np.abs(y - ref)) > 1e-12 * max(1.0, np.max(np.abs(ref))):
            return f"P5 k={k} G={G}: forward != sum_i (y_ji - x_bi)^k"
        dY = rng.normal(size=(batch, n_out))
        dx, _, _ = o.backward(x, coef, dY, G, lo, hi, k=k)
        dref = np.einsum("bj,bji->bi", dY, -k * (yt[None, :, :] - x[:, None, :]) ** (k - 1))
        if np.max(np.abs(dx - dref)) > 1e-11 * max(1.0, np.max(np.abs(dref))):
            return f"P5 k={k} G={G}: dx != -k sum_j dY_bj (y_ji - x_bi)^(k-1)"
    return None


def pin_knot_values_eulerian(o, degrees=(1, 2, 3, 4, 5)):
    """At a knot, the k+1 local weights of the uniform degree-k B-spline are the Eulerian numbers
    A(k, 0..k-1) over k! followed by 0 (textbook: the cardinal B-spline at the integers)."""
    euler = {1: (1,), 2: (1, 1), 3: (1, 4, 1), 4: (1, 11, 11, 1), 5: (1, 26, 66, 26, 1)}
    G, lo, hi = 8, -1.0, 1.0
    h = (hi - lo) / G
    for k in degrees:
        want = [a / math.factorial(k) for a in euler[k]] + [0.0]
        for s in (-k, 0, 3, G - 1):
            x = lo + s * h
            B, _ = o.basis([x], G, lo, hi, k=k)
            for r in range(k + 1):
                m = s + r
                if 0 <= m < G + k and abs(B[0, m] - want[r]) > 1e-14:
                    return f"P4 k={k} s={s}: B_{m} at the knot = {B[0, m]!r} != {want[r]}"
    return None


def _small_problem(rng, G, lo, hi, base, batch=32, n_in=8, n_out=4, k=3):
    h = (hi - lo) / G
    x = rng.uniform(lo - 2 * h, hi + 2 * h, size=(batch, n_in))
    coef = rng.normal(0, 0.1, size=(n_out, n_in, G + k))
    wb = rng.normal(0, 0.3, size=(n_out, n_in)) if base else None
    dY = rng.normal(size=(batch, n_out))
    return x, coef, wb, dY


def pin_finite_difference(o, rng=None, k=3):
    rng = rng or np.random.default_rng(12)
    G, lo, hi = 8, -1.0, 1.0
    for base in (False, True):
        x, coef, wb, dY = _small_problem(rng, G, lo, hi, base, k=k)
        dx, _, _ = o.backward(x, coef, dY, G, lo, hi, w_base=wb, k=k)
        eps = 1e-6
        fd = np.zeros_like(x)
        for b in range(x.shape[0]):
            for i in range(x.shape[1]):
                xp = x.copy(); xp[b, i] += eps
                xm = x.copy(); xm[b, i] -= eps
                yp = o.forward(xp[b:b + 1], coef, G, lo, hi, w_base=wb, k=k)
                ym = o.forward(xm[b:b + 1], coef, G, lo, hi, w_base=wb, k=k)
                fd[b, i] = float(((yp - ym) * dY[b:b + 1]).sum()) / (2 * eps)
        # degree 1 has kinks at the knots: leave out inputs within eps of one
        if k == 1:
            u = (x - lo) / ((hi - lo) / G)
            far = np.abs(u - np.round(u)) > 1e-4
        else:
            far = np.ones_like(x, dtype=bool)
        err = np.max(np.abs(fd - dx)[far]) / np.max(np.abs(dx))
        if not err <= 1e-7:
            return f"P6 k={k} base={base}: dx vs central differences rel err {err:.2e}"
    return None


def pin_param_gradients(o, rng=None):
    rng = rng or np.random.default_rng(13)
    G, lo, hi = 8, -1.0, 1.0
    x, coef, wb, dY = _small_problem(rng, G, lo, hi, True)
    _, dcoef, dwb = o.backward(x, coef, dY, G, lo, hi, w_base=wb)
    n_out, n_in, nb = coef.shape
    zero_c = np.zeros_like(coef)
    zero_w = np.zeros_like(wb)
    picks = [(j, i, m) for j in range(n_out) for i in range(n_in) for m in (0, 3, 5, nb - 1)]
    for (j, i, m) in picks[:: max(1, len(picks) // 40)]:
        E = zero_c.copy(); E[j, i, m] = 1.0
        val = float((o.forward(x, E, G, lo, hi, w_base=zero_w) * dY).sum())
        if abs(val - dcoef[j, i, m]) > 1e-12 * max(1.0, abs(val)):
            return f"P7 dcoef[{j},{i},{m}] = {dcoef[j, i, m]} != <dY, y(E)> = {val}"
    for (j, i) in [(0, 0), (n_out - 1, n_in - 1), (1, 3), (2, 5)]:
        E = zero_w.copy(); E[j, i] = 1.0
        val = float((o.forward(x, zero_c, G, lo, hi, w_base=E) * dY).sum())
        if abs(val - dwb[j, i]) > 1e-12 * max(1.0, abs(val)):
            return f"P7 dw_base[{j},{i}] = {dwb[j, i]} != <dY, y(E)> = {val}"
    return None


def pin_adjoint(o, rng=None):
    rng = rng or np.random.default_rng(14)
    for G, lo, hi in ((8, -1.0, 1.0), (20, -1.0, 1.0)):
        x, coef, wb, dY = _small_problem(rng, G, lo, hi, True, batch=64, n_in=12, n_out=7)
        y = o.forward(x, coef, G, lo, hi, w_base=wb)
        _, dcoef, dwb = o.backward(x, coef, dY, G, lo, hi, w_base=wb)
        lhs = float((dY * y).sum())
        rhs = float((dcoef * coef).sum() + (dwb * wb).sum())
        scale = float(np.abs(dY * y).sum())
        if abs(lhs - rhs) > 1e-12 * scale:
            return f"P8 G={G}: <dY,y> = {lhs} != <dcoef,coef>+<dwb,wb> = {rhs}"
    return None


def pin_library_matmul(o, rng=None):
    import torch
    rng = rng or np.random.default_rng(15)
    for G, lo, hi in ((8, -1.0, 1.0), (5, -3.0, 3.0)):
        x, coef, wb, dY = _small_problem(rng, G, lo, hi, True, batch=48, n_in=10, n_out=6)
        A = o.dense_basis(x, G, lo, hi)
        xs = torch.from_numpy(x)
        silu_t = torch.nn.functional.silu(xs).numpy()
        ref_y = A @ coef.reshape(coef.shape[0], -1).T + silu_t @ wb.T
        y = o.forward(x, coef, G, lo, hi, w_base=wb)
        if np.max(np.abs(y - ref_y)) > 1e-13 * max(1.0, np.max(np.abs(ref_y))):
            return f"P9 G={G}: forward != dense basis @ coef^T + silu @ w_base^T"
        _, dcoef, dwb = o.backward(x, coef, dY, G, lo, hi, w_base=wb)
        ref_dc = (A.T @ dY).T.reshape(coef.shape)
        if np.max(np.abs(dcoef - ref_dc)) > 1e-13 * max(1.0, np.max(np.abs(ref_dc))):
            return f"P9 G={G}: dcoef != (A^T dY)^T"
        ref_dwb = (silu_t.T @ dY).T
        if np.max(np.abs(dwb - ref_dwb)) > 1e-13 * max(1.0, np.max(np.abs(ref_dwb))):
            return f"P9 G={G}: dw_base != (silu(x)^T dY)^T"
    xs = torch.linspace(-12, 12, 4001, dtype=torch.float64, requires_grad=True)
    ys = torch.nn.functional.silu(xs)
    (g,) = torch.autograd.grad(ys.sum(), xs)
    s, ds = o.silu(xs.detach().numpy())
    if np.max(np.abs(s - ys.detach().numpy())) > 1e-14 or np.max(np.abs(ds - g.numpy())) > 1e-14:
        return "P9: silu / silu' differ from torch"
    return None


def pin_one_hot(o, rng=None):
    rng = rng or np.random.default_rng(16)
    G, lo, hi = 8, -1.0, 1.0
    x = rng.uniform(-1.5, 1.5, size=(20, 5))
    B, _ = o.basis(x.reshape(-1), G, lo, hi)
    B = B.reshape(20, 5, G + 3)
    for (j, i, m) in [(0, 0, 0), (2, 4, 10), (1, 2, 5), (3, 1, 3)]:
        coef = np.zeros((4, 5, G + 3)); coef[j, i, m] = 1.0
        y = o.forward(x, coef, G, lo, hi)
        if np.any(y[:, j] != B[:, i, m]) or np.any(np.delete(y, j, axis=1) != 0.0):
            return f"P10: one-hot coef[{j},{i},{m}] does not return B_{m}(x[:,{i}])"
    return None


ALL_PINS = [pin_truncated_power, pin_partition_of_unity, pin_nonneg_local, pin_exact_values, pin_marsden,
            pin_finite_difference, pin_param_gradients, pin_adjoint, pin_library_matmul, pin_one_hot,
            pin_knot_values_eulerian]


def run_all(o):
    """List of failure strings (empty = every pin holds)."""
    fails = []
    for p in ALL_PINS:
        try:
            r = p(o)
        except Exception as e:  # a crashing mutant counts as detected
            r = f"{p.__name__} raised {type(e).__name__}: {e}"
        if r:
            fails.append(r)
    return fails

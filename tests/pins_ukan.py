"""Pins of the UKAN oracle (oracle/ukan.py): facts that do not come from it.

  V1  the unbounded basis is the bounded one shifted: B_m on knots j h equals
      the truncated-power closed form of the bounded grid (pins.truncated_power_basis,
      written independently) three indices on.
  V2  partition of unity everywhere on the unbounded grid, including far from
      0 (|x| up to 10^3 h), with sum B' = 0; at most four non-zero values.
  V3  the positional encoding at q = 0 is (0, 1, 0, 1, ...) and its first two
      components are sin q and cos q.
  V4  the generated coefficients equal torch's linear / silu / linear on the
      encodings, laid out as coef[j, i, q g + r] = c(q)[(j in + i) g + r].
  V5  a generator that outputs 1 for every coefficient (W2 = 0, b2 = 1) gives
      y = in and dx = 0 for any x.
  V6  central finite differences of <dY, y> against dx, dW1, db1, dW2, db2.
  V7  y is linear in b2: <dY, y(b2 + E)> - <dY, y(b2)> = <db2, E>.
"""
from __future__ import annotations

import numpy as np

import pins


def _problem(rng, batch=7, n_in=3, n_out=2, H=5, d=6, g=3, h=0.5, scale=1.5):
    x = rng.normal(0, scale, size=(batch, n_in))
    W1 = rng.normal(0, 0.5, size=(H, d))
    b1 = rng.normal(0, 0.5, size=H)
    W2 = rng.normal(0, 0.5, size=(n_out * n_in * g, H))
    b2 = rng.normal(0, 0.5, size=n_out * n_in * g)
    dY = rng.normal(size=(batch, n_out))
    return x, W1, b1, W2, b2, dY


def pin_shifted_basis(u):
    h, G = 0.25, 24
    x = np.linspace(-0.3, G * h + 0.3, 3001)
    ref = pins.truncated_power_basis(x, G, 0.0, G * h, 3)         # bounded: knots (j - 3) h
    for mb in range(G + 3):
        B, _ = u.basis(x, mb - 3, h)
        if np.max(np.abs(B - ref[:, mb])) > 1e-13:
            return f"V1: unbounded B_{mb - 3} differs from the bounded closed form"
    return None


def pin_partition(u):
    h = 0.3
    x = np.concatenate([np.linspace(-300 * h, 300 * h, 4001), [1000 * h + 0.1, -1000 * h - 0.1]])
    s = np.floor(x / h)
    tot = np.zeros_like(x)
    dtot = np.zeros_like(x)
    nz = np.zeros_like(x)
    for off in range(-5, 3):
        B, dB = u.basis(x, s + off, h)
        tot += B
        dtot += dB
        nz += B != 0
    if np.max(np.abs(tot - 1.0)) > 1e-12 or np.max(np.abs(dtot)) * h > 1e-11 or np.max(nz) > 4:
        return "V2: the unbounded basis is not a partition of unity with four non-zeros"
    return None


def pin_posenc(u):
    pe0 = u.posenc([0], 8)[0]
    if not np.array_equal(pe0, np.array([0.0, 1.0] * 4)):
        return "V3: PE(0) is not (0, 1, 0, 1, ...)"
    q = np.array([-7, 3, 11])
    pe = u.posenc(q, 6)
    if np.max(np.abs(pe[:, 0] - np.sin(q))) > 1e-15 or np.max(np.abs(pe[:, 1] - np.cos(q))) > 1e-15:
        return "V3: PE(q)[0:2] is not (sin q, cos q)"
    return None


def pin_generator_torch(u, rng=None):
    import torch
    rng = rng or np.random.default_rng(51)
    _, W1, b1, W2, b2, _ = _problem(rng)
    n_out, n_in, g, q0, nq = 2, 3, 3, -2, 4
    coef, _ = u.cg_coef(W1, b1, W2, b2, n_out, n_in, g, q0, nq)
    pe = torch.from_numpy(u.posenc(np.arange(q0, q0 + nq), W1.shape[1]))
    c = torch.nn.functional.linear(torch.nn.functional.silu(torch.nn.functional.linear(
        pe, torch.from_numpy(W1), torch.from_numpy(b1))), torch.from_numpy(W2), torch.from_numpy(b2)).numpy()
    for j in range(n_out):
        for i in range(n_in):
            for ql in range(nq):
                for r in range(g):
                    if abs(coef[j, i, ql * g + r] - c[ql, (j * n_in + i) * g + r]) > 1e-13:
                        return f"V4: coef[{j},{i},{ql * g + r}] differs from the torch generator"
    return None


def pin_constant_generator(u, rng=None):
    rng = rng or np.random.default_rng(52)
    x, W1, b1, W2, b2, dY = _problem(rng, scale=20.0)
    W2 = np.zeros_like(W2)
    b2 = np.ones_like(b2)
    y = u.forward(x, W1, b1, W2, b2, 2, 0.5, 3)
    dx = u.backward(x, W1, b1, W2, b2, dY, 2, 0.5, 3)[0]
    if np.max(np.abs(y - 3.0)) > 1e-12 or np.max(np.abs(dx)) > 1e-11:
        return "V5: an all-ones generator does not give y = in, dx = 0"
    return None


def pin_finite_difference(u, rng=None):
    rng = rng or np.random.default_rng(53)
    x, W1, b1, W2, b2, dY = _problem(rng)
    q0, nq = u.groups_of(x, 0.5, 3)
    q0, nq = q0 - 1, nq + 2            # fixed window with a margin, so that small moves of x stay inside it
    dx, dW1, db1, dW2, db2, _ = u.backward(x, W1, b1, W2, b2, dY, 2, 0.5, 3, q0, nq)
    eps = 1e-6

    def f(xx=x, a=W1, b=b1, c=W2, e=b2):
        return float((u.forward(xx, a, b, c, e, 2, 0.5, 3, q0, nq) * dY).sum())

    for name, arr, grad in (("x", x, dx), ("W1", W1, dW1), ("b1", b1, db1), ("W2", W2, dW2), ("b2", b2, db2)):
        for idx in list(np.ndindex(arr.shape))[:: max(1, arr.size // 25)]:
            p, m = arr.copy(), arr.copy()
            p[idx] += eps
            m[idx] -= eps
            kw = {"x": "xx", "W1": "a", "b1": "b", "W2": "c", "b2": "e"}[name]
            fd = (f(**{kw: p}) - f(**{kw: m})) / (2 * eps)
            if abs(fd - grad[idx]) > 1e-6 * max(1.0, abs(grad[idx])):
                return f"V6: d{name}{idx} = {grad[idx]} vs finite difference {fd}"
    return None


def pin_linear_b2(u, rng=None):
    rng = rng or np.random.default_rng(54)
    x, W1, b1, W2, b2, dY = _problem(rng, batch=30)
    db2 = u.backward(x, W1, b1, W2, b2, dY, 2, 0.5, 3)[4]
    E = rng.normal(size=b2.shape)
    lhs = float((dY * (u.forward(x, W1, b1, W2, b2 + E, 2, 0.5, 3) - u.forward(x, W1, b1, W2, b2, 2, 0.5, 3))).sum())
    rhs = float((db2 * E).sum())
    return None if abs(lhs - rhs) <= 1e-10 * max(1.0, abs(lhs)) else f"V7: {lhs} != <db2, E> = {rhs}"


ALL_PINS = [pin_shifted_basis, pin_partition, pin_posenc, pin_generator_torch, pin_constant_generator,
            pin_finite_difference, pin_linear_b2]


def run_all(u):
    fails = []
    for p in ALL_PINS:
        try:
            r = p(u)
        except Exception as e:
            r = f"{p.__name__} raised {type(e).__name__}: {e}"
        if r:
            fails.append(r)
    return fails

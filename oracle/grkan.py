"""fp64 CPU oracle for the group-rational KAN (GR-KAN) activation, forward and backward.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this module.  It shares no code with
the CUDA path and nothing under ``kolmogorov_arnold_network_b200`` imports it.

What it computes (sources):
  - GR-KAN, the Group-Rational KAN of the Kolmogorov-Arnold Transformer, whose
    backward pass (gradient accumulation, atomic adds) is the bottleneck the
    FlashKAT abstract ("FlashKAT: Understanding and Addressing Performance
    Bottlenecks in the Kolmogorov-Arnold Transformer", Abstract) identifies.
  - The rational function is the Pade activation unit named in the same
    page's reference list ("Pad'e Activation Units: End-to-end Learning of
    Flexible Activation Functions in Deep Networks"), read in its "safe" form,
    whose denominator cannot vanish:
        phi(x) = P(x) / Q(x),  P(x) = sum_{p=0..m} a_p x^p,
                               Q(x) = 1 + |S(x)|,  S(x) = sum_{q=1..n} b_q x^q.
  - "Group": the channels are split into G equal, contiguous groups; every
    channel of group g uses the coefficients a[g, :], b[g, :]
    (channel c belongs to group c // (C / G)).
  - Backward, for upstream gradient dY (calculus, with sign(0) = 0):
        dx       = dY * (P'(x) - phi(x) sign(S(x)) S'(x)) / Q(x)
        da[g, p] = sum over rows and the channels of group g of dY x^p / Q(x)
        db[g, q] = sum over the same of -dY phi(x) sign(S(x)) x^q / Q(x)
Sums run in fp64 (numpy's own summation over the flattened group), rows in
chunks so that the memory stays bounded at large sizes.
"""
from __future__ import annotations

import numpy as np


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _parts(x, a, b, groups):
    """P, P', S, S' per element, each channel with its group's coefficients."""
    rows, C = x.shape
    cg = C // groups
    gi = np.arange(C) // cg                    # group of every channel
    A = a[gi]                                  # [C, m+1]
    Bq = np.concatenate([np.zeros((groups, 1)), b], axis=1)[gi]   # [C, n+1], S has no constant term
    m = a.shape[1] - 1
    n = b.shape[1]
    dA = A[:, 1:] * np.arange(1, m + 1)        # coefficients of P'
    dB = Bq[:, 1:] * np.arange(1, n + 1)       # coefficients of S'
    P = _horner_cols(A, x)
    dP = _horner_cols(dA, x) if m >= 1 else np.zeros_like(x)
    S = _horner_cols(Bq, x)
    dS = _horner_cols(dB, x)
    return P, dP, S, dS


def _horner_cols(coef_c, x):
    """sum_p coef_c[c, p] x[:, c]^p for every row (coefficients per channel)."""
    acc = np.broadcast_to(coef_c[:, -1], x.shape).copy()
    for p in range(coef_c.shape[1] - 2, -1, -1):
        acc = acc * x + coef_c[:, p]
    return acc


def check_shapes(x, a, b, groups):
    rows, C = x.shape
    assert groups >= 1 and C % groups == 0, (C, groups)
    assert a.shape[0] == groups and b.shape[0] == groups, (a.shape, b.shape)


def forward(x, a, b, groups):
    """phi(x) elementwise, [rows, C] in fp64."""
    x, a, b = _f64(x), _f64(a), _f64(b)
    check_shapes(x, a, b, groups)
    P, _, S, _ = _parts(x, a, b, groups)
    return P / (1.0 + np.abs(S))


def backward(x, a, b, dY, groups, chunk=4096):
    """(dx [rows, C], da [G, m+1], db [G, n]) in fp64."""
    x, a, b, dY = _f64(x), _f64(a), _f64(b), _f64(dY)
    check_shapes(x, a, b, groups)
    rows, C = x.shape
    cg = C // groups
    m1, n = a.shape[1], b.shape[1]
    dx = np.empty_like(x)
    da = np.zeros((groups, m1))
    db = np.zeros((groups, n))
    for r0 in range(0, rows, chunk):
        xs, gs = x[r0:r0 + chunk], dY[r0:r0 + chunk]
        P, dP, S, dS = _parts(xs, a, b, groups)
        Q = 1.0 + np.abs(S)
        phi = P / Q
        sg = np.sign(S)                         # sign(0) = 0
        dx[r0:r0 + chunk] = gs * (dP - phi * sg * dS) / Q
        ga = gs / Q                             # d phi / d a_p = x^p / Q
        gb = -gs * phi * sg / Q                 # d phi / d b_q = -phi sign(S) x^q / Q
        for g in range(groups):
            sl = slice(g * cg, (g + 1) * cg)
            xg = xs[:, sl]
            xp = np.ones_like(xg)
            for p in range(m1):
                da[g, p] += float(np.sum(ga[:, sl] * xp))
                xp = xp * xg
            xp = xg.copy()
            for q in range(n):
                db[g, q] += float(np.sum(gb[:, sl] * xp))
                xp = xp * xg
    return dx, da, db

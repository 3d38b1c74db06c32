"""fp64 CPU oracle for the 2-D (tensor-product B-spline surface) KAN layer, forward and backward.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this module.  It shares no code with
the CUDA path and nothing under ``kolmogorov_arnold_network_b200`` imports it.

What it computes (sources):
  - InKAN landing page, "Why InKAN?", item "1D and 2D Splines": besides the
    univariate spline layer, "tensor-product B-spline surfaces for joint
    function approximation".  The page gives no formula; the plainest reading,
    taken here: the inputs are taken in consecutive pairs (u, v) =
    (x[2p], x[2p+1]), p = 0 .. in/2 - 1, and each edge (j, p) carries a
    tensor-product surface on the same knot grid for both coordinates,
        phi_jp(u, v) = sum_{m1, m2} coef[j, p, m1, m2] B_m1(u) B_m2(v),
        y[b, j] = sum_p phi_jp(x[b, 2p], x[b, 2p+1]),
    with the degree-k B-splines of the 1-D layer (G intervals on [lo, hi],
    extended by k knots each side, G + k functions; no SiLU branch).
  - Gradients (calculus):
        dcoef[j, p, m1, m2] = sum_b dY[b, j] B_m1(u_bp) B_m2(v_bp)
        dx[b, 2p]   = sum_j dY[b, j] sum_{m1, m2} coef[j, p, m1, m2] B'_m1(u) B_m2(v)
        dx[b, 2p+1] = sum_j dY[b, j] sum_{m1, m2} coef[j, p, m1, m2] B_m1(u) B'_m2(v)
The univariate B_m and B'_m come from the Cox-de Boor recursion of the 1-D
oracle (kan_oracle.c, pinned on its own); every contraction here is a numpy
einsum in fp64.
"""
from __future__ import annotations

import numpy as np

from . import get as _get_1d


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _bases(x, G, lo, hi, k, o):
    """B and B' of every input: [batch, in, G+k] each."""
    batch, n_in = x.shape
    B, dB = o.basis(x.reshape(-1), G, lo, hi, k=k)
    nb = G + k
    return B.reshape(batch, n_in, nb), dB.reshape(batch, n_in, nb)


def forward(x, coef, G, lo, hi, k=3, o=None):
    """y [batch, out] for coef [out, in/2, G+k, G+k]."""
    o = o or _get_1d()
    x, coef = _f64(x), _f64(coef)
    batch, n_in = x.shape
    assert n_in % 2 == 0 and coef.shape[1:] == (n_in // 2, G + k, G + k), coef.shape
    B, _ = _bases(x, G, lo, hi, k, o)
    Bu, Bv = B[:, 0::2], B[:, 1::2]                    # [batch, pairs, nb]
    return np.einsum("bpm,bpn,jpmn->bj", Bu, Bv, coef, optimize=True)


def backward(x, coef, dY, G, lo, hi, k=3, o=None, want_dx=True, want_dcoef=True):
    """(dx [batch, in], dcoef [out, in/2, G+k, G+k])."""
    o = o or _get_1d()
    x, coef, dY = _f64(x), _f64(coef), _f64(dY)
    batch, n_in = x.shape
    B, dB = _bases(x, G, lo, hi, k, o)
    Bu, Bv, dBu, dBv = B[:, 0::2], B[:, 1::2], dB[:, 0::2], dB[:, 1::2]
    dx = dcoef = None
    if want_dx:
        Gm = np.einsum("bj,jpmn->bpmn", dY, coef, optimize=True)      # dY . coef per pair
        dx = np.empty((batch, n_in))
        dx[:, 0::2] = np.einsum("bpmn,bpm,bpn->bp", Gm, dBu, Bv, optimize=True)
        dx[:, 1::2] = np.einsum("bpmn,bpm,bpn->bp", Gm, Bu, dBv, optimize=True)
    if want_dcoef:
        dcoef = np.einsum("bj,bpm,bpn->jpmn", dY, Bu, Bv, optimize=True)
    return dx, dcoef

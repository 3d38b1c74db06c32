"""fp64 CPU oracle for the UKAN layer: a KAN layer on an unbounded grid whose B-spline
coefficients come from a coefficient-generator (CG) model.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this module.  It shares no code with
the CUDA path and nothing under ``kolmogorov_arnold_network_b200`` imports it.

What it computes (sources: "Want to train KANS at scale? Now UKAN!", Abstract;
readings where the abstract is silent are marked "reading"):
  - An unbounded, symmetric grid: knots t_j = j h for every integer j (reading:
    uniform spacing h, symmetric about 0), cubic B-splines B_m(x) = N(x/h - m)
    for every integer m, N the cardinal cubic B-spline on [0, 4).  There is no
    [lo, hi]: every x has exactly the four basis functions
    m = floor(x/h) - 3 .. floor(x/h), and sum_m B_m(x) = 1 everywhere.
  - "grid groups": group q holds the g consecutive basis indices
    m = q g .. q g + g - 1 (reading: a fixed group size g).
  - "positional encoding of grid groups": the sinusoidal encoding of the
    "Attention Is All You Need" entry of the same page's reference list,
    PE(q)[2l] = sin(q w_l), PE(q)[2l+1] = cos(q w_l), w_l = 10000^(-2l/d).
  - the CG model (reading: a two-layer MLP with a SiLU hidden layer) maps PE(q)
    to the coefficients of group q for every edge:
        hid(q) = silu(W1 PE(q) + b1)                      [H]
        c(q)   = W2 hid(q) + b2                           [out * in * g]
        coef[j, i, m] = c(q)[(j * in + i) * g + (m - q g)],  q = floor(m / g)
    ("produces, on the fly, only the B-spline coefficients required locally":
    only the groups that the batch's inputs reach are evaluated).
  - y[b, j] = sum_i sum_m coef[j, i, m] B_m(x[b, i]).
  - Backward, for upstream gradient dY (calculus): dx, and the gradients of
    W1, b1, W2, b2 through dcoef[j, i, m] = sum_b B_m(x[b, i]) dY[b, j].
The cardinal B-spline is evaluated by its own recursion on the unit grid,
    N_0(v) = [0 <= v < 1],  N_k(v) = (v N_{k-1}(v) + (k + 1 - v) N_{k-1}(v - 1)) / k,
and its derivative N_3'(v) = N_2(v) - N_2(v - 1) (textbook); all in fp64.
"""
from __future__ import annotations

import numpy as np


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def cardinal(v, k):
    """N_k(v), the cardinal B-spline of degree k on [0, k+1], elementwise."""
    v = np.asarray(v, dtype=np.float64)
    if k == 0:
        return ((v >= 0.0) & (v < 1.0)).astype(np.float64)
    return (v * cardinal(v, k - 1) + (k + 1 - v) * cardinal(v - 1.0, k - 1)) / k


def basis(x, m, h):
    """B_m(x) = N_3(x/h - m) and B'_m(x) = (N_2(x/h - m) - N_2(x/h - m - 1)) / h."""
    v = np.asarray(x, dtype=np.float64) / h - m
    return cardinal(v, 3), (cardinal(v, 2) - cardinal(v - 1.0, 2)) / h


def posenc(q, d):
    """Sinusoidal encoding of integer positions q: [len(q), d]."""
    q = np.asarray(q, dtype=np.float64).reshape(-1, 1)
    l = np.arange(d // 2, dtype=np.float64)
    w = 10000.0 ** (-2.0 * l / d)
    pe = np.empty((q.shape[0], d))
    pe[:, 0::2] = np.sin(q * w)
    pe[:, 1::2] = np.cos(q * w)
    return pe


def silu(z):
    return z / (1.0 + np.exp(-z))


def dsilu(z):
    s = 1.0 / (1.0 + np.exp(-z))
    return s * (1.0 + z * (1.0 - s))


def groups_of(x, h, g):
    """The groups whose basis functions the inputs x reach: (q_first, count)."""
    x = _f64(x)
    s = np.floor(x / h)
    return int(np.floor((s.min() - 3) / g)), int(np.floor(s.max() / g) - np.floor((s.min() - 3) / g)) + 1


def cg_coef(W1, b1, W2, b2, n_out, n_in, g, q0, nq):
    """The generated coefficients of groups q0 .. q0+nq-1: coef [out, in, nq * g] (basis m = q0 g + local index),
    and the hidden pre-activations [nq, H] (for the backward)."""
    W1, b1, W2, b2 = _f64(W1), _f64(b1), _f64(W2), _f64(b2)
    pe = posenc(np.arange(q0, q0 + nq), W1.shape[1])
    pre = pe @ W1.T + b1                                   # [nq, H]
    c = silu(pre) @ W2.T + b2                              # [nq, out*in*g]
    coef = c.reshape(nq, n_out, n_in, g).transpose(1, 2, 0, 3).reshape(n_out, n_in, nq * g)
    return coef, pre


def forward(x, W1, b1, W2, b2, n_out, h, g, q0=None, nq=None):
    """y [batch, out] of the UKAN layer (the groups default to those the inputs reach)."""
    x = _f64(x)
    batch, n_in = x.shape
    if q0 is None:
        q0, nq = groups_of(x, h, g)
    coef, _ = cg_coef(W1, b1, W2, b2, n_out, n_in, g, q0, nq)
    y = np.zeros((batch, n_out))
    m0 = q0 * g
    for m_loc in range(nq * g):
        B, _ = basis(x, m0 + m_loc, h)                     # [batch, in]
        y += B @ coef[:, :, m_loc].T
    return y


def backward(x, W1, b1, W2, b2, dY, n_out, h, g, q0=None, nq=None):
    """(dx, dW1, db1, dW2, db2, dcoef) of the UKAN layer."""
    x, dY = _f64(x), _f64(dY)
    W1, b1, W2, b2 = _f64(W1), _f64(b1), _f64(W2), _f64(b2)
    batch, n_in = x.shape
    if q0 is None:
        q0, nq = groups_of(x, h, g)
    coef, pre = cg_coef(W1, b1, W2, b2, n_out, n_in, g, q0, nq)
    m0 = q0 * g
    dx = np.zeros((batch, n_in))
    dcoef = np.zeros_like(coef)
    for m_loc in range(nq * g):
        B, dB = basis(x, m0 + m_loc, h)
        dx += dB * (dY @ coef[:, :, m_loc])                # sum_j dY[b,j] coef[j,i,m] B'_m(x[b,i])
        dcoef[:, :, m_loc] = dY.T @ B                      # sum_b dY[b,j] B_m(x[b,i])
    dW1, db1, dW2, db2 = generator_backward(W1, b1, W2, dcoef, q0, nq)
    return dx, dW1, db1, dW2, db2, dcoef


def generator_backward(W1, b1, W2, dcoef, q0, nq):
    """(dW1, db1, dW2, db2) from the window's dcoef [out, in, nq * g]: back through the generator."""
    W1, b1, W2, dcoef = _f64(W1), _f64(b1), _f64(W2), _f64(dcoef)
    n_out, n_in, ng = dcoef.shape
    g = ng // nq
    pe = posenc(np.arange(q0, q0 + nq), W1.shape[1])
    pre = pe @ W1.T + b1                                   # [nq, H]
    dc = dcoef.reshape(n_out, n_in, nq, g).transpose(2, 0, 1, 3).reshape(nq, -1)   # [nq, out*in*g]
    hid = silu(pre)
    dW2 = dc.T @ hid                                       # [out*in*g, H]
    db2 = dc.sum(0)
    dpre = (dc @ W2) * dsilu(pre)                          # [nq, H]
    dW1 = dpre.T @ pe                                      # [H, d]
    db1 = dpre.sum(0)
    return dW1, db1, dW2, db2

"""Torch-facing calls over the C ABI, and the drop-in ``KANLayer`` module.

``KANLayer(in, out)`` replaces ``nn.Linear(in, out)`` (InKAN landing page,
"Drop-in Replacement" and "Quick Start"); ``KANNetwork([784, 64, 10])`` stacks
layers.  PyTorch provides device memory, the stream and autograd; every step
of the layer itself runs in libkan_b200.so.
"""
from __future__ import annotations

import torch

from . import _native as N

_DT = {torch.float32: N.KAN_F32, torch.bfloat16: N.KAN_BF16}


def _code(t: torch.Tensor) -> int:
    if t.dtype not in _DT:
        raise TypeError(f"dtype {t.dtype} not supported (float32 or bfloat16)")
    return _DT[t.dtype]


def _p(t):
    return None if t is None else t.data_ptr()


def _check(t, name, dtype=None, shape=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def shape_of(x, coef, G, lo, hi, w_base=None, path=N.KAN_PATH_AUTO, degree=3, dims=1) -> N.kan_shape:
    batch, n_in = x.shape
    return N.make_shape(batch, n_in, coef.shape[0], G, lo, hi, _code(x), w_base is not None, path, degree, dims)


def _coef_shape(n_out, n_in, G, degree, dims):
    nb = G + degree
    return (n_out, n_in, nb) if dims == 1 else (n_out, n_in // 2, nb, nb)


def _stream(t):
    return torch.cuda.current_stream(t.device).cuda_stream


def workspace(shape: N.kan_shape, for_backward: bool, device) -> torch.Tensor | None:
    device = torch.device(device)
    if device.type == "cuda":
        with torch.cuda.device(device):
            n = N.kan_workspace_size(shape, for_backward)
    else:
        n = N.kan_workspace_size(shape, for_backward)
    return torch.empty(n, dtype=torch.uint8, device=device) if n else None


def forward(x, coef, G, lo, hi, w_base=None, path=N.KAN_PATH_AUTO, y=None, ws=None, degree=3, dims=1):
    """y[b,j] = sum_i sum_m coef[j,i,m] B_m(x[b,i]) (+ sum_i w_base[j,i] silu(x[b,i])), degree-k B-splines;
    dims=2: sum_p sum_{m1,m2} coef[j,p,m1,m2] B_m1(x[b,2p]) B_m2(x[b,2p+1]) (tensor-product surfaces)."""
    batch, n_in = x.shape
    n_out = coef.shape[0]
    _check(x, "x", None)
    _check(coef, "coef", x.dtype, _coef_shape(n_out, n_in, G, degree, dims))
    _check(w_base, "w_base", x.dtype, (n_out, n_in))
    s = shape_of(x, coef, G, lo, hi, w_base, path, degree, dims)
    if y is None:
        y = torch.empty((batch, n_out), dtype=x.dtype, device=x.device)
    _check(y, "y", x.dtype, (batch, n_out))
    if ws is None:
        ws = workspace(s, False, x.device)
    # the library works on the current device: make it x's
    with torch.cuda.device(x.device):
        N.kan_forward(s, _p(x), _p(coef), _p(w_base), _p(y), _p(ws), 0 if ws is None else ws.numel(), _stream(x))
    return y


def backward(x, coef, dY, G, lo, hi, w_base=None, need_dx=True, need_dcoef=True, need_dw_base=True,
             path=N.KAN_PATH_AUTO, out=None, ws=None, degree=3, dims=1):
    """(dx, dcoef, dw_base) of the layer for upstream gradient dY; dcoef/dw_base are float32."""
    batch, n_in = x.shape
    n_out = coef.shape[0]
    _check(x, "x", None)
    _check(coef, "coef", x.dtype, _coef_shape(n_out, n_in, G, degree, dims))
    _check(w_base, "w_base", x.dtype, (n_out, n_in))
    _check(dY, "dY", x.dtype, (batch, n_out))
    s = shape_of(x, coef, G, lo, hi, w_base, path, degree, dims)
    if out is not None:
        dx, dcoef, dwb = out
    else:
        dx = torch.empty_like(x) if need_dx else None
        dcoef = torch.empty(coef.shape, dtype=torch.float32, device=x.device) if need_dcoef else None
        dwb = (torch.empty(w_base.shape, dtype=torch.float32, device=x.device)
               if (need_dw_base and w_base is not None) else None)
    if ws is None:
        ws = workspace(s, True, x.device)
    with torch.cuda.device(x.device):
        N.kan_backward(s, _p(x), _p(coef), _p(w_base), _p(dY), _p(dx), _p(dcoef), _p(dwb), _p(ws),
                       0 if ws is None else ws.numel(), _stream(x))
    return dx, dcoef, dwb


def basis(x, G, lo, hi, degree=3):
    """(span int32 [.., in], w [.., in, k+1], dw [.., in, k+1]) of the basis step alone."""
    _check(x, "x", None)
    batch, n_in = x.shape
    s = N.make_shape(batch, n_in, 1, G, lo, hi, _code(x), False, degree=degree)
    span = torch.empty((batch, n_in), dtype=torch.int32, device=x.device)
    w = torch.empty((batch, n_in, degree + 1), dtype=torch.float32, device=x.device)
    dw = torch.empty((batch, n_in, degree + 1), dtype=torch.float32, device=x.device)
    with torch.cuda.device(x.device):
        N.kan_basis(s, _p(x), _p(span), _p(w), _p(dw), _stream(x))
    return span, w, dw


class _KANFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, coef, w_base, G, lo, hi, degree):
        x = x.contiguous()
        y = forward(x, coef, G, lo, hi, w_base, degree=degree)
        ctx.save_for_backward(x, coef, w_base)
        ctx.grid = (G, lo, hi, degree)
        return y

    @staticmethod
    def backward(ctx, dY):
        x, coef, w_base = ctx.saved_tensors
        G, lo, hi, degree = ctx.grid
        dx, dcoef, dwb = backward(x, coef, dY.contiguous().to(x.dtype), G, lo, hi, w_base,
                                  need_dx=ctx.needs_input_grad[0], need_dcoef=ctx.needs_input_grad[1],
                                  need_dw_base=w_base is not None and ctx.needs_input_grad[2], degree=degree)
        return (dx, None if dcoef is None else dcoef.to(coef.dtype), None if dwb is None else dwb.to(w_base.dtype),
                None, None, None, None)


class KANLayer(torch.nn.Module):
    """B-spline KAN layer (cubic by default), a drop-in for ``nn.Linear(in, out)``.

    Parameters: ``coef`` [out, in, G+degree] and, with ``base=True``, ``w_base``
    [out, in] for the SiLU base branch.
    """

    def __init__(self, in_features, out_features, G=8, lo=-1.0, hi=1.0, base=False, coef_std=0.1,
                 dtype=torch.float32, device=None, degree=3):
        super().__init__()
        self.in_features, self.out_features = in_features, out_features
        self.G, self.lo, self.hi, self.degree = int(G), float(lo), float(hi), int(degree)
        self.coef = torch.nn.Parameter(
            torch.randn(out_features, in_features, G + degree, dtype=torch.float32, device=device)
            .mul_(coef_std).to(dtype))
        self.w_base = (torch.nn.Parameter(torch.randn(out_features, in_features, dtype=torch.float32, device=device)
                                          .mul_(in_features ** -0.5).to(dtype)) if base else None)

    def forward(self, x):
        lead = x.shape[:-1]
        y = _KANFunction.apply(x.reshape(-1, self.in_features), self.coef, self.w_base, self.G, self.lo, self.hi,
                               self.degree)
        return y.reshape(*lead, self.out_features)


# ---------------------------------------------------------------------------
# GR-KAN: the group-rational activation (safe Pade form per channel group)
def grkan_shape(x, a, b, groups):
    rows, C = x.shape
    return N.make_grkan_shape(rows, C, groups, a.shape[1] - 1, b.shape[1], _code(x))


def grkan_forward(x, a, b, groups, y=None):
    """y = P_g(x) / (1 + |S_g(x)|) per channel, g = channel // (C / groups); a [G, m+1], b [G, n] float32."""
    _check(x, "x", None)
    _check(a, "a", torch.float32)
    _check(b, "b", torch.float32)
    s = grkan_shape(x, a, b, groups)
    if y is None:
        y = torch.empty_like(x)
    _check(y, "y", x.dtype, tuple(x.shape))
    with torch.cuda.device(x.device):
        N.kan_grkan_forward(s, _p(x), _p(a), _p(b), _p(y), _stream(x))
    return y


def grkan_backward(x, a, b, dY, groups, need_dx=True, need_da=True, need_db=True, out=None, ws=None):
    """(dx, da, db) for upstream gradient dY; da, db are float32, reduced without atomics."""
    _check(x, "x", None)
    _check(dY, "dY", x.dtype, tuple(x.shape))
    s = grkan_shape(x, a, b, groups)
    if out is not None:
        dx, da, db = out
    else:
        dx = torch.empty_like(x) if need_dx else None
        da = torch.empty(a.shape, dtype=torch.float32, device=x.device) if need_da else None
        db = torch.empty(b.shape, dtype=torch.float32, device=x.device) if need_db else None
    if ws is None and (da is not None or db is not None):
        with torch.cuda.device(x.device):
            n = N.kan_grkan_workspace_size(s)
        ws = torch.empty(max(n, 16), dtype=torch.uint8, device=x.device)
    with torch.cuda.device(x.device):
        N.kan_grkan_backward(s, _p(x), _p(a), _p(b), _p(dY), _p(dx), _p(da), _p(db), _p(ws),
                             0 if ws is None else ws.numel(), _stream(x))
    return dx, da, db


class _GRKANFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, a, b, groups):
        x = x.contiguous()
        ctx.save_for_backward(x, a, b)
        ctx.groups = groups
        return grkan_forward(x, a, b, groups)

    @staticmethod
    def backward(ctx, dY):
        x, a, b = ctx.saved_tensors
        dx, da, db = grkan_backward(x, a, b, dY.contiguous().to(x.dtype), ctx.groups,
                                    need_dx=ctx.needs_input_grad[0], need_da=ctx.needs_input_grad[1],
                                    need_db=ctx.needs_input_grad[2])
        return dx, da, db, None


class GRKAN(torch.nn.Module):
    """Group-rational activation over the last dimension (channels): ``groups`` coefficient sets of a
    degree-(m, n) safe Pade function, initialised to the identity-like phi(x) = x."""

    def __init__(self, channels, groups=8, num_degree=5, den_degree=4, device=None):
        super().__init__()
        self.channels, self.groups = channels, groups
        a = torch.zeros(groups, num_degree + 1, dtype=torch.float32, device=device)
        a[:, 1] = 1.0
        self.a = torch.nn.Parameter(a)
        self.b = torch.nn.Parameter(torch.zeros(groups, den_degree, dtype=torch.float32, device=device))

    def forward(self, x):
        lead = x.shape[:-1]
        y = _GRKANFunction.apply(x.reshape(-1, self.channels), self.a, self.b, self.groups)
        return y.reshape(*lead, self.channels)


class _KAN2DFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, coef, G, lo, hi):
        x = x.contiguous()
        ctx.save_for_backward(x, coef)
        ctx.grid = (G, lo, hi)
        return forward(x, coef, G, lo, hi, dims=2)

    @staticmethod
    def backward(ctx, dY):
        x, coef = ctx.saved_tensors
        G, lo, hi = ctx.grid
        dx, dcoef, _ = backward(x, coef, dY.contiguous().to(x.dtype), G, lo, hi, need_dx=ctx.needs_input_grad[0],
                                need_dcoef=ctx.needs_input_grad[1], dims=2)
        return dx, None if dcoef is None else dcoef.to(coef.dtype), None, None, None


class KANLayer2D(torch.nn.Module):
    """Layer of cubic tensor-product B-spline surfaces over consecutive input pairs:
    ``coef`` [out, in/2, G+3, G+3]; ``in_features`` must be even."""

    def __init__(self, in_features, out_features, G=8, lo=-1.0, hi=1.0, coef_std=0.1, dtype=torch.float32,
                 device=None):
        super().__init__()
        if in_features % 2:
            raise ValueError("in_features must be even (inputs are taken in pairs)")
        self.in_features, self.out_features = in_features, out_features
        self.G, self.lo, self.hi = int(G), float(lo), float(hi)
        self.coef = torch.nn.Parameter(
            torch.randn(out_features, in_features // 2, G + 3, G + 3, dtype=torch.float32, device=device)
            .mul_(coef_std).to(dtype))

    def forward(self, x):
        lead = x.shape[:-1]
        y = _KAN2DFunction.apply(x.reshape(-1, self.in_features), self.coef, self.G, self.lo, self.hi)
        return y.reshape(*lead, self.out_features)


# ---------------------------------------------------------------------------
# UKAN: unbounded grid, coefficients from a generator of grid-group encodings
_RANGE_WS = 2368


def ukan_window(x, h, group):
    """(q0, nq): the grid groups whose basis functions the inputs reach (basis floor(x/h) - 3 .. floor(x/h)),
    from the inputs' device-side minimum and maximum (one small read-back)."""
    import math
    ws = torch.empty(_RANGE_WS, dtype=torch.uint8, device=x.device)
    mm = torch.empty(2, dtype=torch.float32, device=x.device)
    with torch.cuda.device(x.device):
        N.kan_input_range(x.numel(), _p(x), _code(x), _p(mm), _p(ws), _RANGE_WS, _stream(x))
    lo, hi = mm.tolist()
    if not (math.isfinite(lo) and math.isfinite(hi)):
        raise ValueError("UKAN layers need finite inputs (the window of generated groups is sized from them)")
    s_lo, s_hi = math.floor(lo / h), math.floor(hi / h)
    q0 = math.floor((s_lo - 3) / group)
    nq = math.floor(s_hi / group) - q0 + 1
    while nq * group < 4:
        nq += 1
    return q0, nq


def ukan_shape(n_in, n_out, group, W1, q0, nq, dtype):
    return N.make_ukan_shape(n_in, n_out, group, W1.shape[1], W1.shape[0], q0, nq,
                             N.KAN_F32 if dtype == torch.float32 else N.KAN_BF16)


def ukan_generate(W1, b1, W2, b2, n_in, n_out, group, q0, nq, dtype=torch.float32):
    """(coef [out, in, nq*group] in dtype, pre [nq, hidden] float32): the generator's window."""
    for t, nm in ((W1, "W1"), (b1, "b1"), (W2, "W2"), (b2, "b2")):
        _check(t, nm, torch.float32)
    s = ukan_shape(n_in, n_out, group, W1, q0, nq, dtype)
    coef = torch.empty((n_out, n_in, nq * group), dtype=dtype, device=W1.device)
    pre = torch.empty((nq, W1.shape[0]), dtype=torch.float32, device=W1.device)
    with torch.cuda.device(W1.device):
        N.kan_ukan_generate(s, _p(W1), _p(b1), _p(W2), _p(b2), _p(coef), _p(pre), _stream(W1))
    return coef, pre


def ukan_generate_backward(W1, W2, pre, dcoef, n_in, n_out, group, q0, nq, dtype=torch.float32):
    """(dW1, db1, dW2, db2) from the window's dcoef [out, in, nq*group] (float32)."""
    s = ukan_shape(n_in, n_out, group, W1, q0, nq, dtype)
    dW1, dW2 = torch.empty_like(W1), torch.empty_like(W2)
    db1 = torch.empty(W1.shape[0], dtype=torch.float32, device=W1.device)
    db2 = torch.empty(W2.shape[0], dtype=torch.float32, device=W1.device)
    with torch.cuda.device(W1.device):
        n = N.kan_ukan_workspace_size(s)
        ws = torch.empty(max(n, 16), dtype=torch.uint8, device=W1.device)
        N.kan_ukan_generate_backward(s, _p(W1), _p(W2), _p(pre), _p(dcoef), _p(dW1), _p(db1), _p(dW2), _p(db2),
                                     _p(ws), ws.numel(), _stream(W1))
    return dW1, db1, dW2, db2


class _UKANFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, W1, b1, W2, b2, h, group, n_out):
        x = x.contiguous()
        batch, n_in = x.shape
        q0, nq = ukan_window(x, h, group)
        coef, pre = ukan_generate(W1, b1, W2, b2, n_in, n_out, group, q0, nq, x.dtype)
        ks = N.kan_ukan_layer_shape(ukan_shape(n_in, n_out, group, W1, q0, nq, x.dtype), batch, h)
        y = forward(x, coef, ks.G, ks.lo, ks.hi)
        ctx.save_for_backward(x, W1, W2, coef, pre)
        ctx.meta = (h, group, n_out, q0, nq, ks.G, ks.lo, ks.hi)
        return y

    @staticmethod
    def backward(ctx, dY):
        x, W1, W2, coef, pre = ctx.saved_tensors
        h, group, n_out, q0, nq, G, lo, hi = ctx.meta
        dx, dcoef, _ = backward(x, coef, dY.contiguous().to(x.dtype), G, lo, hi, need_dx=ctx.needs_input_grad[0])
        dW1, db1, dW2, db2 = ukan_generate_backward(W1, W2, pre, dcoef, x.shape[1], n_out, group, q0, nq, x.dtype)
        return dx, dW1, db1, dW2, db2, None, None, None


class UKANLayer(torch.nn.Module):
    """KAN layer on an unbounded grid (spacing h) whose cubic B-spline coefficients come from a generator:
    an MLP of the sinusoidal encodings of grid groups (``group`` basis functions each).  Only the groups that
    the batch's inputs reach are generated; the inputs need no normalisation."""

    def __init__(self, in_features, out_features, h=0.25, group=4, pe_dim=16, hidden=32, device=None):
        super().__init__()
        self.in_features, self.out_features, self.h, self.group = in_features, out_features, float(h), int(group)
        kw = dict(dtype=torch.float32, device=device)
        self.W1 = torch.nn.Parameter(torch.randn(hidden, pe_dim, **kw) * pe_dim ** -0.5)
        self.b1 = torch.nn.Parameter(torch.zeros(hidden, **kw))
        self.W2 = torch.nn.Parameter(torch.randn(out_features * in_features * group, hidden, **kw) * 0.1 * hidden ** -0.5)
        self.b2 = torch.nn.Parameter(torch.zeros(out_features * in_features * group, **kw))

    def forward(self, x):
        lead = x.shape[:-1]
        y = _UKANFunction.apply(x.reshape(-1, self.in_features), self.W1, self.b1, self.W2, self.b2, self.h,
                                self.group, self.out_features)
        return y.reshape(*lead, self.out_features)


class KANNetwork(torch.nn.Module):
    """Stack of KANLayer: ``KANNetwork([784, 64, 10])``."""

    def __init__(self, widths, **kw):
        super().__init__()
        self.layers = torch.nn.ModuleList(KANLayer(a, b, **kw) for a, b in zip(widths[:-1], widths[1:]))

    def forward(self, x):
        for L in self.layers:
            x = L(x)
        return x

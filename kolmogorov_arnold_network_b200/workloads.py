"""Named synthetic workloads and their seeded input generators.

This module holds no arithmetic of the KAN layer: only shapes, grid
parameters and the random draws of the inputs.  The tests, the oracle checks
and the benchmark all take their inputs from here, so that the CUDA path and
the fp64 oracle see the same values.

Recipe (every tensor): a CPU ``torch.Generator`` seeded with
``1000 * family + tensor_id`` (tensor ids: x=0, coef=1, w_base=2, dY=3,
second-layer coef=4), drawn in fp32, then rounded once to the operand dtype.
Distributions: ``N(0, s)`` takes ``s`` as the standard deviation, except the
base weights, drawn with variance ``1/in`` (standard deviation ``1/sqrt(in)``).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Layer:
    """One KAN layer's hyper-parameters (B-splines of degree `degree` on a uniform grid)."""
    inp: int
    out: int
    G: int
    lo: float
    hi: float
    base: bool = False
    degree: int = 3
    dims: int = 1                # 2: tensor-product surfaces over consecutive input pairs

    @property
    def nb(self) -> int:
        """Basis functions per coordinate: G + degree."""
        return self.G + self.degree

    @property
    def units(self) -> int:
        """Edge functions per output: inputs (1-D) or input pairs (2-D)."""
        return self.inp if self.dims == 1 else self.inp // 2

    @property
    def cols(self) -> int:
        """Columns of the dense basis expansion per unit: nb (1-D) or nb^2 (2-D)."""
        return self.nb if self.dims == 1 else self.nb * self.nb


@dataclass(frozen=True)
class Workload:
    name: str
    family: int                  # seed family
    batch: int
    layers: tuple                # tuple[Layer, ...]; >1 only for the FFN block
    dtype: str                   # "f32" or "bf16" (operand dtype; accumulation is fp32)
    x_dist: tuple                # ("uniform", a, b) or ("normal", std)
    coef_std: float
    mode: str = "fwd+bwd"        # "fwd" or "fwd+bwd"
    note: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def edges(self) -> int:
        """Edge evaluations per step: batch * in * out summed over layers (a 2-D surface edge takes an
        input pair: batch * in/2 * out)."""
        return sum(self.batch * L.units * L.out for L in self.layers)


def _grid_sweep():
    out = {}
    for G in (8, 20, 50):
        for dt in ("f32", "bf16"):
            for mode in ("fwd", "fwd+bwd"):
                nm = f"sweep512_g{G}_{dt}_{'fwd' if mode == 'fwd' else 'fwdbwd'}"
                out[nm] = Workload(nm, 4, 65536, (Layer(512, 512, G, -1.0, 1.0),), dt, ("uniform", -1.0, 1.0), 0.1,
                                   mode=mode, note="grid sweep 512x512, batch 65536")
    return out


def _degree_sweep():
    out = {}
    for k in (1, 2, 4, 5):
        nm = f"degree512_k{k}_g20_bf16_fwdbwd"
        out[nm] = Workload(nm, 6, 65536, (Layer(512, 512, 20, -1.0, 1.0, degree=k),), "bf16", ("uniform", -1.0, 1.0),
                           0.1, note=f"spline degree {k}: 512x512, batch 65536, G=20")
    return out


def _surfaces():
    out = {}
    for dt, batch in (("bf16", 65536), ("f32", 16384)):
        nm = f"surface512_g8_{dt}_fwdbwd"
        out[nm] = Workload(nm, 8, batch, (Layer(512, 512, 8, -1.0, 1.0, dims=2),), dt, ("uniform", -1.0, 1.0), 0.1,
                           note=f"2-D tensor-product surfaces: 512 inputs in 256 pairs -> 512, batch {batch}, G=8")
    return out


WORKLOADS = {
    "layer8x4": Workload("layer8x4", 1, 32, (Layer(8, 4, 8, -1.0, 1.0),), "f32", ("uniform", -1.0, 1.0), 0.1,
                         note="KANLayer(8,4) on a [32,8] batch, G=8 on [-1,1]"),
    "layer784x64_silu": Workload("layer784x64_silu", 2, 4096, (Layer(784, 64, 8, -1.0, 1.0, base=True),), "f32",
                                 ("uniform", -1.0, 1.0), 0.1,
                                 note="first layer of KANNetwork([784,64,10]) at batch 4096, SiLU base branch"),
    "layer1024_g20_bf16": Workload("layer1024_g20_bf16", 3, 16384, (Layer(1024, 1024, 20, -1.0, 1.0),), "bf16",
                                   ("uniform", -1.1, 1.1), 0.1,
                                   note="1024x1024, G=20, inputs reach the extended knot intervals"),
    **_grid_sweep(),
    "ffn768_3072_bf16": Workload("ffn768_3072_bf16", 5, 8192,
                                 (Layer(768, 3072, 5, -3.0, 3.0), Layer(3072, 768, 5, -3.0, 3.0)), "bf16",
                                 ("normal", 1.0), 0.05, note="KAN FFN block 768->3072->768, 8192 tokens"),
    **_degree_sweep(),
    **_surfaces(),
}

#: the workload the benchmark times by default: the largest single-GPU one by edge evaluations per step
BENCH_DEFAULT = "ffn768_3072_bf16"


@dataclass(frozen=True)
class GrWorkload:
    """A GR-KAN (group-rational activation) workload: x [rows, channels] in `groups` channel groups,
    numerator degree m, denominator degree n."""
    name: str
    family: int
    rows: int
    channels: int
    groups: int
    m: int
    n: int
    dtype: str
    note: str = ""

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elements(self) -> int:
        return self.rows * self.channels


def _grkan():
    out = {}
    for dt in ("bf16", "f32"):
        nm = f"grkan_vitb_{dt}"
        out[nm] = GrWorkload(nm, 7, 128 * 197, 3072, 8, 5, 4, dt,
                             note="GR-KAN on the 3072-wide hidden activation of a ViT-B MLP, 128 images x 197 tokens")
    return out


GR_WORKLOADS = _grkan()


@dataclass(frozen=True)
class UkWorkload:
    """A UKAN layer workload: x ~ N(0, x_std) [batch, in] (no normalisation to a grid range), knot spacing h,
    `group` basis functions per grid group, generator with pe_dim-wide encodings and `hidden` units."""
    name: str
    family: int
    batch: int
    inp: int
    out: int
    h: float
    group: int
    pe_dim: int
    hidden: int
    dtype: str
    x_std: float
    note: str = ""

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def edges(self) -> int:
        return self.batch * self.inp * self.out


UK_WORKLOADS = {
    "ukan512_bf16": UkWorkload("ukan512_bf16", 9, 65536, 512, 512, 0.25, 4, 16, 32, "bf16", 1.0,
                               note="UKAN layer 512->512, batch 65536, unbounded grid h=0.25, groups of 4"),
    "ukan512_f32": UkWorkload("ukan512_f32", 9, 16384, 512, 512, 0.25, 4, 16, 32, "f32", 1.0,
                              note="UKAN layer 512->512, batch 16384, unbounded grid h=0.25, groups of 4"),
}


def _gen(family: int, tensor_id: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(1000 * family + tensor_id)
    return g


def draw_x(w: Workload, rows: int | None = None) -> torch.Tensor:
    rows = w.batch if rows is None else rows
    g = _gen(w.family, 0)
    shape = (rows, w.layers[0].inp)
    if w.x_dist[0] == "uniform":
        a, b = w.x_dist[1], w.x_dist[2]
        x = torch.rand(shape, generator=g, dtype=torch.float32) * (b - a) + a
    else:
        x = torch.randn(shape, generator=g, dtype=torch.float32) * w.x_dist[1]
    return x.to(w.torch_dtype)


def draw_coef(w: Workload, layer: int = 0) -> torch.Tensor:
    L = w.layers[layer]
    g = _gen(w.family, 1 if layer == 0 else 4)
    shape = (L.out, L.inp, L.nb) if L.dims == 1 else (L.out, L.inp // 2, L.nb, L.nb)
    c = torch.randn(shape, generator=g, dtype=torch.float32) * w.coef_std
    return c.to(w.torch_dtype)


def draw_w_base(w: Workload, layer: int = 0):
    L = w.layers[layer]
    if not L.base:
        return None
    g = _gen(w.family, 2)
    c = torch.randn((L.out, L.inp), generator=g, dtype=torch.float32) * (1.0 / L.inp) ** 0.5
    return c.to(w.torch_dtype)


def draw_dY(w: Workload, rows: int | None = None) -> torch.Tensor:
    rows = w.batch if rows is None else rows
    g = _gen(w.family, 3)
    return torch.randn((rows, w.layers[-1].out), generator=g, dtype=torch.float32).to(w.torch_dtype)


def draw_all(w: Workload, rows: int | None = None) -> dict:
    """All inputs of a workload as CPU tensors in the operand dtype."""
    d = {"x": draw_x(w, rows), "dY": draw_dY(w, rows)}
    for li in range(len(w.layers)):
        d[f"coef{li}"] = draw_coef(w, li)
        d[f"w_base{li}"] = draw_w_base(w, li)
    return d


def draw_grkan(w: GrWorkload, rows: int | None = None) -> dict:
    """x ~ N(0, 1), dY ~ N(0, 1) in the operand dtype; a ~ N(0, 0.5), b ~ N(0, 0.5) float32 (ids 0, 3, 1, 2)."""
    rows = w.rows if rows is None else rows
    x = torch.randn((rows, w.channels), generator=_gen(w.family, 0), dtype=torch.float32).to(w.torch_dtype)
    dY = torch.randn((rows, w.channels), generator=_gen(w.family, 3), dtype=torch.float32).to(w.torch_dtype)
    a = torch.randn((w.groups, w.m + 1), generator=_gen(w.family, 1), dtype=torch.float32) * 0.5
    b = torch.randn((w.groups, w.n), generator=_gen(w.family, 2), dtype=torch.float32) * 0.5
    return {"x": x, "dY": dY, "a": a, "b": b}


def draw_ukan(w: UkWorkload, rows: int | None = None) -> dict:
    """x ~ N(0, x_std), dY ~ N(0, 1) in the operand dtype; generator parameters float32:
    W1 ~ N(0, 1/pe_dim), b1 ~ N(0, 0.1^2), W2 ~ N(0, 0.1^2 / hidden), b2 ~ N(0, 0.1^2) (ids 0, 3, 1, 2, 4, 5)."""
    rows = w.batch if rows is None else rows
    f32 = torch.float32
    x = (torch.randn((rows, w.inp), generator=_gen(w.family, 0), dtype=f32) * w.x_std).to(w.torch_dtype)
    dY = torch.randn((rows, w.out), generator=_gen(w.family, 3), dtype=f32).to(w.torch_dtype)
    E = w.out * w.inp * w.group
    return {"x": x, "dY": dY,
            "W1": torch.randn((w.hidden, w.pe_dim), generator=_gen(w.family, 1), dtype=f32) * w.pe_dim ** -0.5,
            "b1": torch.randn(w.hidden, generator=_gen(w.family, 2), dtype=f32) * 0.1,
            "W2": torch.randn((E, w.hidden), generator=_gen(w.family, 4), dtype=f32) * 0.1 * w.hidden ** -0.5,
            "b2": torch.randn(E, generator=_gen(w.family, 5), dtype=f32) * 0.1}


def custom_ukan(batch, inp, out, h=0.25, group=4, pe_dim=16, hidden=32, dtype="f32", x_std=1.0, family=92):
    return UkWorkload(f"ukan_custom_{batch}x{inp}x{out}_{dtype}", family, batch, inp, out, h, group, pe_dim, hidden,
                      dtype, x_std)


def custom_grkan(rows, channels, groups, m=5, n=4, dtype="f32", family=91):
    """An ad-hoc GR-KAN workload (tests of ragged and edge shapes)."""
    return GrWorkload(f"grkan_custom_{rows}x{channels}_g{groups}_{m}{n}_{dtype}", family, rows, channels, groups, m, n,
                      dtype)


def custom(batch, inp, out, G, lo, hi, dtype="f32", base=False, x_range=None, coef_std=0.1, family=90, degree=3,
           dims=1):
    """An ad-hoc single-layer workload (tests of ragged and edge shapes)."""
    h = (hi - lo) / G
    # reach into the extended intervals (and, for degrees other than 3, a little beyond them)
    ext = 2.0 if degree == 3 else degree - 0.5
    xr = x_range or (lo - ext * h, hi + ext * h)
    return Workload(f"custom_{batch}x{inp}x{out}_g{G}_k{degree}_d{dims}_{dtype}", family, batch,
                    (Layer(inp, out, G, lo, hi, base, degree, dims),), dtype, ("uniform", xr[0], xr[1]), coef_std)

"""Benchmark: KAN layer forward+backward edge evaluations per second on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
    python bench.py --only NAME [--steps K]      # one workload by itself, its own JSON line

Default workload: the KAN FFN block (8192 tokens, 768 -> 3072 -> 768, G = 5 on
[-3, 3], bf16 operands with fp32 accumulation), the largest single-GPU
workload of the method's measurement plan by edge evaluations per step.

A step is one pass of the whole hot path over one batch of synthetic input:
kan_forward of every layer, then one kan_backward per layer (last layer first)
returning dx, dcoef and dw_base together, all through the C ABI of
libkan_b200.so.  Edge evaluations per step = batch * in * out (summed over the
layers of the FFN block).  One JSON line is printed by rank 0.

Timing: W untimed steps, then K timed steps between a barrier and a device
synchronize on both sides.  Each step is bracketed by CUDA events on the
launching stream; a 256 MiB buffer (larger than the 126 MB L2) is rewritten
between steps, outside the events.  Each call carries its own events, and the
library records two more inside it (kan_set_timing_marks) at the boundaries
of its kernel groups, so that every call splits into operand preparation,
dcoef and dx time: the dominant one gives the roofline.  With N > 1
(torchrun), every rank runs an independent replica of the workload (weak
scaling, no collective on the data path) and the time is the maximum over
ranks.

Also in the line: the measured fp32 FMA peak (the library's calibration
kernel), the whole step against its bound, the bilinear adjoint identity per
layer as a parity check that needs no reference, and (one GPU) the same
figures for the other large workloads of the plan ("other_workloads").

--impl reference times the fp64 CPU oracle on the host cores instead (the
only reference this build has), each step a bounded row sample of the same
workload.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from kolmogorov_arnold_network_b200 import workloads as W  # noqa: E402

METRIC = "KAN layer fwd+bwd edge-evals/sec (batch*in*out) and % of roofline, 1xB200"
UNIT = "edge-evals/s"
F16_PER_BF16 = 1.0           # nominal dense fp16 : bf16 tensor-core ratio on B200 (same rate)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm": d["hbm_gbs"], "bf16": d["bf16_tflops"], "bf16_sus": d.get("bf16_tflops_sustained"),
                "src": "measured"}
    return {"hbm": 6650.0, "bf16": 1590.0, "bf16_sus": 1400.0, "src": "fallback"}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(v: float, world: int, device=None) -> float:
    """The maximum of a per-rank time over all ranks (identity with one rank)."""
    if world <= 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(units_per_rank_step: float, steps: int, world: int, t_max_ms: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return world * units_per_rank_step * steps / (t_max_ms / 1000.0)


def csrc_hash() -> str:
    """Hash of the kernel sources (names and bytes), to match ncu figures to the kernels they were taken on."""
    import glob
    import hashlib
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "kolmogorov_arnold_network_b200", "csrc", "*"))):
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


# ---------------------------------------------------------------------------
# FLOP / byte accounting (per call, algorithmic)
def layer_dense_flops(batch, L):
    """Dense-expanded FLOPs of one layer GEMM: 2 * batch * out * (units * columns per unit [+ in for SiLU])."""
    k = L.units * L.cols + (L.inp if L.base else 0)
    return 2.0 * batch * L.out * k


def layer_alg_flops(batch, L):
    """Algorithmic FLOPs of one layer GEMM: (k+1)^dims FMAs per edge (4 for cubic splines, 16 for cubic
    surfaces; +1 with SiLU), 2 FLOPs each."""
    return (2.0 * (L.degree + 1) ** L.dims + (2.0 if L.base else 0.0)) * batch * L.units * L.out


def layer_bytes(batch, L, esz, call):
    """Algorithmic HBM bytes of one call: operands read once, outputs written once."""
    x = batch * L.inp * esz
    dy = batch * L.out * esz
    coef = L.out * L.units * L.cols * esz + (L.out * L.inp * esz if L.base else 0)
    if call == "fwd":
        return x + coef + batch * L.out * esz
    if call == "dcoef":
        return x + dy + (L.out * L.units * L.cols + (L.out * L.inp if L.base else 0)) * 4
    return x + dy + coef + batch * L.inp * esz          # dx


def measured_counters(workload: str, call: str):
    """The committed ncu figures of a call's main kernel (profiles/traffic.json, keyed by segment: "fwd1",
    "dcoef1", "dx1" for layer index 1, "bwd" for GR-KAN): DRAM bytes per launch and tensor-pipe activity,
    or None when there are none or the kernel sources changed since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    if d.get("csrc_hash") != csrc_hash():
        return None
    return d.get("workloads", {}).get(workload, {}).get(call)


def measured_traffic(workload: str, call: str):
    """DRAM bytes per launch of a call's main kernel from the committed ncu capture, or None."""
    e = measured_counters(workload, call)
    return None if e is None else e.get("dram_bytes")


# ---------------------------------------------------------------------------
def result_keys(li: int, n_layers: int, mode: str):
    """The step's results among layer li's tensors (what the end-to-end variant copies to the host): the
    last layer's y, the first layer's dx and every layer's dcoef and dw_base (without a backward, y only)."""
    keys = ["y"] if li == n_layers - 1 else []
    if mode != "fwd":
        keys += (["dx"] if li == 0 else []) + ["dcoef", "dwb"]
    return keys


class Runner:
    """Pre-allocated buffers and the step's C-ABI calls for one workload.

    A step is the forward of every layer, then one kan_backward per layer (last
    layer first) that returns dx, dcoef and dw_base together: the call pattern
    of training through the library."""

    def __init__(self, w: W.Workload, dev):
        from kolmogorov_arnold_network_b200 import _native as N
        from kolmogorov_arnold_network_b200 import layer as LY
        self.N, self.LY, self.w, self.dev = N, LY, w, dev
        d = W.draw_all(w)
        self.host = d
        dt = w.torch_dtype
        self.x = d["x"].to(dev)
        self.dY = d["dY"].to(dev)
        self.layers = []
        act = self.x
        for li, L in enumerate(w.layers):
            coef = d[f"coef{li}"].to(dev)
            wb = None if d[f"w_base{li}"] is None else d[f"w_base{li}"].to(dev)
            s = LY.shape_of(act, coef, L.G, L.lo, L.hi, wb, degree=L.degree, dims=L.dims)
            ws_f = LY.workspace(s, False, dev)
            ws_b = LY.workspace(s, True, dev)
            y = torch.empty((w.batch, L.out), dtype=dt, device=dev)
            dx = torch.empty((w.batch, L.inp), dtype=dt, device=dev)
            dcoef = torch.empty(coef.shape, dtype=torch.float32, device=dev)
            dwb = None if wb is None else torch.empty(wb.shape, dtype=torch.float32, device=dev)
            self.layers.append(dict(L=L, s=s, x=act, coef=coef, wb=wb, y=y, dx=dx, dcoef=dcoef, dwb=dwb,
                                    ws_f=ws_f, ws_b=ws_b))
            act = y
        self.h_x = self.h_dY = None

    def pin_host(self):
        """Pinned host mirrors of the inputs and of the step's results (the end-to-end variant): the last
        layer's y, the first layer's dx and every layer's dcoef (and dw_base); the activations and
        gradients between the layers stay on the device."""
        self.h_x = self.host["x"].pin_memory()
        self.h_dY = self.host["dY"].pin_memory()
        pin = lambda t: None if t is None else torch.empty_like(t, device="cpu").pin_memory()
        self.h_out = []
        for li, l in enumerate(self.layers):
            keys = result_keys(li, len(self.layers), self.w.mode)
            self.h_out.append({k: pin(l[k]) if k in keys else None for k in ("y", "dx", "dcoef", "dwb")})

    def results_of(self, name):
        """(host, device) pairs of the step's results that call `name` completes."""
        kind, li = name.rstrip("0123456789"), int(name[len(name.rstrip("0123456789")):])
        l, h = self.layers[li], self.h_out[li]
        keys = ("y",) if kind == "fwd" else ("dx", "dcoef", "dwb")
        return [(h[k], l[k]) for k in keys if h[k] is not None]

    def dy_of(self, li):
        return self.dY if li == len(self.layers) - 1 else self.layers[li + 1]["dx"]

    def calls(self):
        """The step as a list of (name, kind, callable(marks)), in launch order; kind is "fwd" or "bwd".
        marks = (after_prep, after_dcoef) event handles or None, set for the duration of the call."""
        N, P = self.N, lambda t: None if t is None else t.data_ptr()
        st = torch.cuda.current_stream(self.dev).cuda_stream
        out = []
        for li, l in enumerate(self.layers):
            def fwd(marks=None, l=l):
                if marks is not None:
                    N.kan_set_timing_marks(marks[0], None)
                N.kan_forward(l["s"], P(l["x"]), P(l["coef"]), P(l["wb"]), P(l["y"]), P(l["ws_f"]),
                              0 if l["ws_f"] is None else l["ws_f"].numel(), st)
                if marks is not None:
                    N.kan_set_timing_marks(None, None)
            out.append((f"fwd{li}", "fwd", fwd))
        if self.w.mode == "fwd":
            return out
        for li in reversed(range(len(self.layers))):
            l = self.layers[li]
            dy = self.dy_of(li)

            def bwd(marks=None, l=l, dy=dy):
                if marks is not None:
                    N.kan_set_timing_marks(marks[0], marks[1])
                N.kan_backward(l["s"], P(l["x"]), P(l["coef"]), P(l["wb"]), P(dy), P(l["dx"]), P(l["dcoef"]),
                               P(l["dwb"]), P(l["ws_b"]), 0 if l["ws_b"] is None else l["ws_b"].numel(), st)
                if marks is not None:
                    N.kan_set_timing_marks(None, None)
            out.append((f"bwd{li}", "bwd", bwd))
        return out

    def h2d(self):
        self.x.copy_(self.h_x, non_blocking=True)
        n = self.h_x.numel() * self.h_x.element_size()
        if self.w.mode != "fwd":
            self.dY.copy_(self.h_dY, non_blocking=True)
            n += self.h_dY.numel() * self.h_dY.element_size()
        return n

    def d2h_after(self, name, stream, copy_stream):
        """Copy the results of call `name` to pinned host memory on the copy stream, once `stream` has
        produced them (they leave while the next calls compute); returns the bytes copied."""
        n = 0
        pairs = self.results_of(name)
        if pairs:
            copy_stream.wait_stream(stream)
            with torch.cuda.stream(copy_stream):
                for h, d in pairs:
                    h.copy_(d, non_blocking=True)
                    n += h.numel() * h.element_size()
        return n

    def adjoint_errors(self):
        """Bilinear adjoint identity per layer (y is linear in coef and w_base):
        <dY, y> = <dcoef, coef> + <dw_base, w_base>, relative to sum |dY * y|.  Holds at any size,
        needs no reference implementation."""
        out = {}
        for li, l in enumerate(self.layers):
            dy = self.dy_of(li).double()
            y = l["y"].double()
            lhs = (dy * y).sum().item()
            rhs = (l["dcoef"].double() * l["coef"].double()).sum().item()
            if l["wb"] is not None:
                rhs += (l["dwb"].double() * l["wb"].double()).sum().item()
            scale = (dy * y).abs().sum().item()
            out[f"layer{li}"] = abs(lhs - rhs) / scale if scale > 0 else abs(lhs - rhs)
        return out


def _ev():
    return torch.cuda.Event(enable_timing=True)


def time_steps(R: Runner, K: int, warmup: int, flush, barrier=lambda: None):
    """W untimed steps, then K steps each bracketed by events on the launching stream, with the L2 flush
    buffer rewritten between steps (outside the events).  Every call records its own events and the
    library's timing marks, which split it into segments: "prep<li>" (fp32 operand preparation),
    "fwd<li>", "dcoef<li>", "dx<li>".  Returns (total ms, {segment: total ms}, launches)."""
    N = R.N
    calls = R.calls()
    stream = torch.cuda.current_stream(R.dev)
    for _ in range(warmup):
        flush.zero_()
        for _, _, c in calls:
            c()
    torch.cuda.synchronize(R.dev)
    st = N.kan_sync_status(None)
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {N.STATUS.get(st, st)}")
    # per call: start, after_prep (layer calls), after_dcoef (backward only), end
    evs = [[dict(start=_ev(), prep=_ev() if kind in ("fwd", "bwd") else None, mid=_ev() if kind == "bwd" else None,
                 end=_ev()) for _, kind, _ in calls] for _ in range(K)]
    step_ev = [(_ev(), _ev()) for _ in range(K)]
    # torch creates an event's CUDA handle at its first record: record every mark event once now, so that
    # the handles passed to the library exist
    for row in evs:
        for e in row:
            for v in e.values():
                if v is not None:
                    v.record(stream)
    barrier()
    torch.cuda.synchronize(R.dev)
    n0 = N.kan_launch_count()
    for k in range(K):
        flush.zero_()
        step_ev[k][0].record(stream)
        for e, (_, kind, c) in zip(evs[k], calls):
            e["start"].record(stream)
            if e["prep"] is None:
                c()
            else:
                c((e["prep"].cuda_event, None if e["mid"] is None else e["mid"].cuda_event))
            e["end"].record(stream)
        step_ev[k][1].record(stream)
    torch.cuda.synchronize(R.dev)
    barrier()
    launches = N.kan_launch_count() - n0
    total = sum(a.elapsed_time(b) for a, b in step_ev)
    seg = {}
    for k in range(K):
        for e, (nm, kind, _) in zip(evs[k], calls):
            if kind not in ("fwd", "bwd"):
                seg[nm] = seg.get(nm, 0.0) + e["start"].elapsed_time(e["end"])
                continue
            li = nm[3:]
            parts = [(f"prep{li}", e["start"], e["prep"])]
            if kind == "fwd":
                parts.append((f"fwd{li}", e["prep"], e["end"]))
            else:
                parts += [(f"dcoef{li}", e["prep"], e["mid"]), (f"dx{li}", e["mid"], e["end"])]
            for key, e0, e1 in parts:
                seg[key] = seg.get(key, 0.0) + e0.elapsed_time(e1)
    return total, seg, launches


def ffma_peak(dev, sms):
    """The fp32 FMA rate of this GPU, measured with the library's calibration kernel (best of 3 launches
    of about 50 ms each), in TFLOP/s."""
    from kolmogorov_arnold_network_b200 import _native as N
    blocks = sms * 4
    sink = torch.empty(blocks * 256, dtype=torch.float32, device=dev)
    st = torch.cuda.current_stream(dev)
    iters = 2000
    N.kan_ffma_probe(blocks, iters, sink.data_ptr(), st.cuda_stream)      # warm-up
    torch.cuda.synchronize(dev)
    best = 0.0
    for _ in range(3):
        a, b = _ev(), _ev()
        a.record(st)
        fl = N.kan_ffma_probe(blocks, iters * 25, sink.data_ptr(), st.cuda_stream)
        b.record(st)
        torch.cuda.synchronize(dev)
        best = max(best, fl / (a.elapsed_time(b) / 1000.0) / 1e12)
    return best


def step_roofline(w: W.Workload, ms_per_step: float, pk: dict, ffma_tflops: float):
    """The whole step against its bound: bf16, dense-expanded FLOPs of every GEMM at the bf16 tensor
    peak; fp32, algorithmic FLOPs at the fp32 FMA peak (3 GEMMs per layer for forward + backward)."""
    gemms = 1 if w.mode == "fwd" else 3
    if w.dtype == "bf16":
        fl = gemms * sum(layer_dense_flops(w.batch, L) for L in w.layers)
        t = fl / (pk["bf16"] * 1e12)
    else:
        fl = gemms * sum(layer_alg_flops(w.batch, L) for L in w.layers)
        t = fl / (ffma_tflops * 1e12)
    return {"t_roof_ms": t * 1000.0, "frac": t * 1000.0 / ms_per_step,
            "bound": "bf16 tensor, dense-expanded" if w.dtype == "bf16" else "fp32 FMA, algorithmic"}


def roofline_of(w: W.Workload, seg: dict, K: int, pk: dict, ffma_tflops: float):
    """Roofline of the dominant kernel segment (fwd, dcoef or dx of one layer).

    bf16: dense-expanded FLOPs of the GEMM at the measured bf16 tensor peak.  fp32: the fp32 bound of
    the method's measurement plan, algorithmic FLOPs (4 FMAs per edge, +1 with SiLU) at the measured
    fp32 FMA peak; the dense-expanded fraction at the fp16 tensor peak is reported beside it."""
    gemm = {k: v for k, v in seg.items() if k.rstrip("0123456789") in ("fwd", "dcoef", "dx")}
    dom = max(gemm, key=gemm.get)
    kind, li = dom.rstrip("0123456789"), int(dom[len(dom.rstrip("0123456789")):])
    L = w.layers[li]
    avg_s = gemm[dom] / K / 1000.0
    dense = layer_dense_flops(w.batch, L)
    counters = measured_counters(w.name, dom) or {}
    if w.dtype == "bf16":
        achieved = dense / avg_s / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": pk["bf16"], "unit": "TFLOP/s",
                "frac": achieved / pk["bf16"], "peak_note": f"bf16 dense, {pk['src']} burst (of {pk['src']})",
                "frac_of_sustained": achieved / pk["bf16_sus"] if pk.get("bf16_sus") else None,
                "flops_per_launch": dense, "flops_kind": "dense-expanded"}
    else:
        alg = layer_alg_flops(w.batch, L)
        achieved = alg / avg_s / 1e12
        tens = dense / avg_s / 1e12
        roof = {"bound": "alu", "achieved": achieved, "peak": ffma_tflops, "unit": "TFLOP/s",
                "frac": achieved / ffma_tflops,
                "peak_note": "fp32 FMA peak measured in this run by the library's calibration kernel",
                "flops_per_launch": alg, "flops_kind": "algorithmic (4 FMA per edge, +1 with SiLU)",
                "tensor_dense_achieved": tens, "tensor_dense_frac": tens / (pk["bf16"] * F16_PER_BF16),
                "note": ("the kernel runs on fp16 tensor cores (3 products of hi/lo splits); tensor_dense_frac is "
                         "its dense-expanded FLOPs at the fp16 tensor peak, at most 1/3 by construction")}
    roof.update({"traffic": counters.get("dram_bytes"), "tensor_pipe_active": counters.get("tensor_pipe_active"),
                 "kernel": f"{kind} of layer {li}", "launch_ms": avg_s * 1000.0,
                 "algorithmic_bytes_per_launch": layer_bytes(w.batch, L, 4 if w.dtype == "f32" else 2, kind),
                 "segment_ms": {k: v / K for k, v in seg.items()}})
    return roof


class ClockSampler:
    def __init__(self, dev_index):
        self.proc = None
        self.path = None
        try:
            uuid = str(torch.cuda.get_device_properties(dev_index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            uuid = None
        q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
        cmd = ["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits", "-lms", "50"]
        if uuid:
            cmd += ["-i", uuid]
        self.first = ""
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            # wait for the first sample, so that even a timed region shorter than
            # nvidia-smi's start-up is covered by the stream that follows
            self.first = self.proc.stdout.readline()
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in (self.first + out).strip().splitlines():
            f = [t.strip() for t in line.split(",")]
            if len(f) >= 8:
                try:
                    rows.append((float(f[0]), float(f[1]), f[3:], float(f[2])))
                except ValueError:
                    pass
        if not rows:
            return None
        # "under load": samples drawing at least half the peak power seen
        pmax = max(r[3] for r in rows)
        loaded = [r for r in rows if r[3] >= 0.5 * pmax] or rows
        sm = sorted(r[0] for r in loaded)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for nm, v in zip(names, r[2][1:]):
                if v.lower() == "active":
                    reasons.add(nm)
        res = {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": max(r[1] for r in rows), "reasons": sorted(reasons),
               "samples": len(rows), "samples_under_load": len(loaded), "power_w_max": pmax}
        if len(rows) < 3:
            res["note"] = "timed region about as short as the 50 ms sampling interval: few samples"
        return res


# ---------------------------------------------------------------------------
def _oracle_step(o, d, w: W.Workload, rows: int, cores: int):
    """The whole hot path of the workload on the first `rows` rows, by the fp64 oracle (forward through
    every layer, then the backward of every layer, last first)."""
    from oracle import kan2d
    act = d["x"][:rows]
    acts = []
    for li, L in enumerate(w.layers):
        acts.append(act)
        if L.dims == 2:
            act = kan2d.forward(act, d[f"coef{li}"], L.G, L.lo, L.hi, k=L.degree, o=o)
        else:
            act = o.forward(act, d[f"coef{li}"], L.G, L.lo, L.hi, w_base=d[f"w_base{li}"], k=L.degree,
                            nthreads=cores)
    g = d["dY"][:rows]
    for li in (reversed(range(len(w.layers))) if w.mode != "fwd" else ()):
        L = w.layers[li]
        if L.dims == 2:
            g, _ = kan2d.backward(acts[li], d[f"coef{li}"], g, L.G, L.lo, L.hi, k=L.degree, o=o)
        else:
            g, _, _ = o.backward(acts[li], d[f"coef{li}"], g, L.G, L.lo, L.hi, w_base=d[f"w_base{li}"], k=L.degree,
                                 nthreads=cores)


def cpu_baseline(w: W.Workload, target_s=12.0):
    """The fp64 oracle, as it stands, on a row sample of the workload (host cores)."""
    import oracle
    o = oracle.get()
    cores = oracle.default_threads()
    d = W.draw_all(w)

    def run(rows):
        t0 = time.perf_counter()
        _oracle_step(o, d, w, rows, cores)
        return time.perf_counter() - t0

    probe = max(cores, 8)
    t = run(probe)
    rows = int(min(w.batch, max(probe, probe * target_s / max(t, 1e-6))))
    # the whole batch may take well under target_s: repeat it until about target_s
    passes, t, t_first = 0, 0.0, None
    while True:
        dt = run(rows)
        t_first = dt if t_first is None else t_first
        t += dt
        passes += 1
        if t >= 0.8 * target_s or passes >= 100:
            break
    edges = passes * sum(rows * L.units * L.out for L in w.layers)
    return {"value": edges / t, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{passes} pass(es) over {rows} of {w.batch} rows of {w.name}, fp64 Cox-de Boor "
                      f"{'forward' if w.mode == 'fwd' else 'forward+backward'}, {t:.1f} s"}


def run_reference(args, world, rank):
    w = W.WORKLOADS[args.workload]
    if rank != 0:
        return
    import oracle
    o = oracle.get()
    cores = oracle.default_threads()
    d = W.draw_all(w)

    def step(rows):
        _oracle_step(o, d, w, rows, cores)

    # size the per-step sample so that warmup + steps end within ~2 minutes
    probe = max(cores, 8)
    t0 = time.perf_counter()
    step(probe)
    per_row = (time.perf_counter() - t0) / probe
    budget = 120.0 / max(1, args.steps + args.warmup)
    rows = int(max(1, min(w.batch, budget / max(per_row, 1e-9))))
    for _ in range(args.warmup):
        step(rows)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step(rows)
    dt = time.perf_counter() - t0
    edges = sum(rows * L.units * L.out for L in w.layers) * args.steps
    value = edges / dt
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"{rows} of {w.batch} rows per step of {w.name}"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_of(w: W.Workload):
    L0 = w.layers[0]
    c = {"workload": w.name, "batch": w.batch, "layers": [[L.inp, L.out] for L in w.layers], "G": L0.G,
         "degree": L0.degree, "dims": L0.dims, "grid": [L0.lo, L0.hi], "silu_base": L0.base, "mode": w.mode,
         "l2": "256 MiB flush between steps",
         "note": w.note}
    if w.dtype == "f32":
        c["compute"] = ("fp32 operands as fp16 hi/lo splits (power-of-two scaled), 3 fp16 tensor-core products, "
                        "fp32 accumulation")
    else:
        c["compute"] = "bf16 operands, fp32 accumulation"
    return c


class UkRunner(Runner):
    """A UKAN layer step: the generator's window, the layer's forward and backward on it, and the
    generator's backward.  The window (the groups the fixed synthetic batch reaches) is sized once, before
    the timed steps, from the inputs' device-side range."""

    def __init__(self, w: W.UkWorkload, dev):
        from kolmogorov_arnold_network_b200 import _native as N
        from kolmogorov_arnold_network_b200 import layer as LY
        self.N, self.LY, self.uk, self.dev = N, LY, w, dev
        d = W.draw_ukan(w)
        self.host = d
        self.x, self.dY = d["x"].to(dev), d["dY"].to(dev)
        self.W1, self.b1, self.W2, self.b2 = (d[k].to(dev) for k in ("W1", "b1", "W2", "b2"))
        self.q0, self.nq = LY.ukan_window(self.x, w.h, w.group)
        self.us = LY.ukan_shape(w.inp, w.out, w.group, self.W1, self.q0, self.nq, w.torch_dtype)
        self.ks = N.kan_ukan_layer_shape(self.us, w.batch, w.h)
        self.coef = torch.empty((w.out, w.inp, self.nq * w.group), dtype=w.torch_dtype, device=dev)
        self.pre = torch.empty((self.nq, w.hidden), dtype=torch.float32, device=dev)
        self.y = torch.empty((w.batch, w.out), dtype=w.torch_dtype, device=dev)
        self.dx = torch.empty_like(self.x)
        self.dcoef = torch.empty(self.coef.shape, dtype=torch.float32, device=dev)
        self.g = [torch.empty_like(t) for t in (self.W1, self.b1, self.W2, self.b2)]
        self.ws_f = LY.workspace(self.ks, False, dev)
        self.ws_b = LY.workspace(self.ks, True, dev)
        self.ws_g = torch.empty(max(16, N.kan_ukan_workspace_size(self.us)), dtype=torch.uint8, device=dev)
        self.w = W.Workload(w.name, w.family, w.batch, (W.Layer(w.inp, w.out, self.ks.G, self.ks.lo, self.ks.hi),),
                            w.dtype, ("normal", w.x_std), 0.0, note=w.note)

    def calls(self):
        N, P = self.N, lambda t: None if t is None else t.data_ptr()
        st = torch.cuda.current_stream(self.dev).cuda_stream
        ks, us = self.ks, self.us

        def gen():
            N.kan_ukan_generate(us, P(self.W1), P(self.b1), P(self.W2), P(self.b2), P(self.coef), P(self.pre), st)

        def fwd(marks=None):
            if marks is not None:
                N.kan_set_timing_marks(marks[0], None)
            N.kan_forward(ks, P(self.x), P(self.coef), None, P(self.y), P(self.ws_f),
                          0 if self.ws_f is None else self.ws_f.numel(), st)
            if marks is not None:
                N.kan_set_timing_marks(None, None)

        def bwd(marks=None):
            if marks is not None:
                N.kan_set_timing_marks(marks[0], marks[1])
            N.kan_backward(ks, P(self.x), P(self.coef), None, P(self.dY), P(self.dx), P(self.dcoef), None,
                           P(self.ws_b), 0 if self.ws_b is None else self.ws_b.numel(), st)
            if marks is not None:
                N.kan_set_timing_marks(None, None)

        def gen_bwd():
            N.kan_ukan_generate_backward(us, P(self.W1), P(self.W2), P(self.pre), P(self.dcoef), *(P(t) for t in self.g),
                                         P(self.ws_g), self.ws_g.numel(), st)
        return [("gen0", "gen", gen), ("fwd0", "fwd", fwd), ("bwd0", "bwd", bwd), ("genbwd0", "gen", gen_bwd)]


class GrRunner:
    """Buffers and the two C-ABI calls of one GR-KAN workload: the forward (y) and one backward that
    returns dx, da and db."""

    def __init__(self, w: W.GrWorkload, dev):
        from kolmogorov_arnold_network_b200 import _native as N
        self.N, self.w, self.dev = N, w, dev
        d = W.draw_grkan(w)
        self.x, self.dY = d["x"].to(dev), d["dY"].to(dev)
        self.a, self.b = d["a"].to(dev), d["b"].to(dev)
        self.y = torch.empty_like(self.x)
        self.dx = torch.empty_like(self.x)
        self.da = torch.empty_like(self.a)
        self.db = torch.empty_like(self.b)
        code = N.KAN_F32 if w.dtype == "f32" else N.KAN_BF16
        self.s = N.make_grkan_shape(w.rows, w.channels, w.groups, w.m, w.n, code)
        self.ws = torch.empty(max(16, N.kan_grkan_workspace_size(self.s)), dtype=torch.uint8, device=dev)

    def calls(self):
        N, st = self.N, torch.cuda.current_stream(self.dev).cuda_stream

        def fwd():
            N.kan_grkan_forward(self.s, self.x.data_ptr(), self.a.data_ptr(), self.b.data_ptr(), self.y.data_ptr(), st)

        def bwd():
            N.kan_grkan_backward(self.s, self.x.data_ptr(), self.a.data_ptr(), self.b.data_ptr(), self.dY.data_ptr(),
                                 self.dx.data_ptr(), self.da.data_ptr(), self.db.data_ptr(), self.ws.data_ptr(),
                                 self.ws.numel(), st)
        return [("fwd", fwd), ("bwd", bwd)]


def time_grkan(w: W.GrWorkload, dev, K, flush, pk):
    """GR-KAN forward + backward: K steps, events around each call, L2 flushed between steps; the
    backward (the larger call) against the HBM roofline."""
    R = GrRunner(w, dev)
    calls = R.calls()
    stream = torch.cuda.current_stream(dev)
    for _ in range(3):
        flush.zero_()
        for _, c in calls:
            c()
    torch.cuda.synchronize(dev)
    ev = [[(_ev(), _ev()) for _ in calls] for _ in range(K)]
    for k in range(K):
        flush.zero_()
        for (a, b), (_, c) in zip(ev[k], calls):
            a.record(stream)
            c()
            b.record(stream)
    torch.cuda.synchronize(dev)
    seg = {nm: sum(ev[k][i][0].elapsed_time(ev[k][i][1]) for k in range(K)) / K for i, (nm, _) in enumerate(calls)}
    esz = 4 if w.dtype == "f32" else 2
    n = w.elements
    bytes_ = {"fwd": 2.0 * n * esz, "bwd": 3.0 * n * esz}      # fwd: x in, y out; bwd: x, dY in, dx out
    gbs = {k: bytes_[k] / (seg[k] / 1000.0) / 1e9 for k in seg}
    ms = seg["fwd"] + seg["bwd"]
    out = {"ms_per_step": ms, "value": n / (ms / 1000.0), "unit": "elements/s", "steps": K, "dtype": w.dtype,
           "dominant": "bwd", "bound": "hbm", "achieved": gbs["bwd"], "peak": pk["hbm"], "peak_unit": "GB/s",
           "frac": gbs["bwd"] / pk["hbm"], "fwd_frac": gbs["fwd"] / pk["hbm"], "segment_ms": seg,
           "traffic": (measured_counters(w.name, "bwd") or {}).get("dram_bytes"),
           "algorithmic_bytes_per_launch": bytes_,
           "step_roofline": {"t_roof_ms": (bytes_["fwd"] + bytes_["bwd"]) / (pk["hbm"] * 1e9) * 1000.0,
                             "frac": (bytes_["fwd"] + bytes_["bwd"]) / (pk["hbm"] * 1e9) * 1000.0 / ms,
                             "bound": "HBM, algorithmic bytes"},
           "config": {"rows": w.rows, "channels": w.channels, "groups": w.groups, "m": w.m, "n": w.n,
                      "note": w.note}}
    # bitwise reproducibility of the atomic-free gradient reduction
    d1 = (R.da.clone(), R.db.clone())
    calls[1][1]()
    torch.cuda.synchronize(dev)
    out["deterministic"] = bool(torch.equal(d1[0], R.da) and torch.equal(d1[1], R.db))
    del R
    torch.cuda.empty_cache()
    return out


#: workloads timed beside the headline one (each in the same JSON line, with the adjoint-identity check)
EXTRA_WORKLOADS = ["layer784x64_silu", "layer1024_g20_bf16"] + \
    [f"sweep512_g{G}_{dt}_fwdbwd" for G in (8, 20, 50) for dt in ("bf16", "f32")] + \
    [f"degree512_k{k}_g20_bf16_fwdbwd" for k in (1, 2, 4, 5)] + \
    [f"surface512_g8_{dt}_fwdbwd" for dt in ("bf16", "f32")]


def time_other(nm: str, dev, K: int, flush, pk: dict, ffma: float) -> dict:
    """One workload beside the headline one: K steps after 3 warm-up steps, L2 flushed between steps."""
    if nm in W.GR_WORKLOADS:
        return time_grkan(W.GR_WORKLOADS[nm], dev, K, flush, pk)
    if nm in W.UK_WORKLOADS:
        wu = W.UK_WORKLOADS[nm]
        Ru = UkRunner(wu, dev)
        tu, segu, _ = time_steps(Ru, K, 3, flush)
        msu = tu / K
        ru = roofline_of(Ru.w, segu, K, pk, ffma)
        out = {"ms_per_step": msu, "value": wu.edges / (msu / 1000.0), "unit": UNIT, "steps": K,
               "dtype": wu.dtype, "dominant": ru["kernel"], "bound": ru["bound"], "frac": ru["frac"],
               "segment_ms": ru["segment_ms"], "step_roofline": step_roofline(Ru.w, msu, pk, ffma),
               "window": {"q0": Ru.q0, "nq": Ru.nq, "G": Ru.ks.G, "basis_per_input": Ru.nq * wu.group},
               "note": "generator window sized once before the timed steps; step = generate + layer "
                       "forward + layer backward + generator backward"}
        del Ru
        torch.cuda.empty_cache()
        return out
    wx = W.WORKLOADS[nm]
    Rx = Runner(wx, dev)
    tx, segx, _ = time_steps(Rx, K, 3, flush)
    msx = tx / K
    rx = roofline_of(wx, segx, K, pk, ffma)
    ax = Rx.adjoint_errors()
    tolx = 1e-5 if wx.dtype == "f32" else 2e-2
    out = {"ms_per_step": msx, "value": wx.edges / (msx / 1000.0), "unit": UNIT, "steps": K,
           "dtype": wx.dtype, "dominant": rx["kernel"], "bound": rx["bound"], "frac": rx["frac"],
           "tensor_dense_frac": rx.get("tensor_dense_frac"),
           "segment_ms": rx["segment_ms"], "step_roofline": step_roofline(wx, msx, pk, ffma),
           "adjoint_rel_err": ax, "adjoint_ok": all(v <= tolx for v in ax.values())}
    del Rx
    torch.cuda.empty_cache()
    return out


def run_only(args, local):
    """``--only NAME``: one workload of the measurement plan by itself (one GPU, no headline line); used to
    profile a kernel that the headline workload does not run."""
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    res = time_other(args.only, dev, args.steps, flush, peaks(), ffma_peak(dev, sms))
    st = R_status()
    if st != 0:
        raise RuntimeError(f"device status after timing: {st}")
    print(json.dumps({"workload": args.only, **res}), flush=True)


def run_ours(args, world, rank, local):
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = W.WORKLOADS[args.workload]
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    R = Runner(w, dev)
    sampler = ClockSampler(local)   # started before the warm-up so that it is sampling by the timed region
    wall0 = time.perf_counter()
    K = args.steps
    total, seg, launches = time_steps(R, K, args.warmup, flush, barrier)
    wall = time.perf_counter() - wall0
    clocks = sampler.stop()
    t_max = max_over_ranks(total, world, dev)
    value = aggregate_rate(w.edges, K, world, t_max)
    adj = R.adjoint_errors()
    tol = 1e-5 if w.dtype == "f32" else 2e-2
    ffma = ffma_peak(dev, sms)
    pk = peaks()
    roof = roofline_of(w, seg, K, pk, ffma)

    # ---- end to end: pinned host inputs in, results out, every step ----
    e2e = None
    if not args.no_e2e:
        R.pin_host()
        calls = R.calls()
        e2e_ev = [(_ev(), _ev()) for _ in range(K)]
        hb = db = 0
        copy_stream = torch.cuda.Stream(dev)
        barrier()
        torch.cuda.synchronize(dev)
        for k in range(K):
            flush.zero_()
            e2e_ev[k][0].record(stream)
            hb = R.h2d()
            db = 0
            for nm, _, c in calls:
                c()
                db += R.d2h_after(nm, stream, copy_stream)
            stream.wait_stream(copy_stream)   # the step ends when its results are on the host
            e2e_ev[k][1].record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in e2e_ev), world, dev)
        e2e = {"value": aggregate_rate(w.edges, K, world, e_ms), "unit": UNIT, "h2d_bytes_per_step": hb,
               "d2h_bytes_per_step": db}
    del R

    # ---- the other workloads of the method's measurement plan, one GPU only ----
    others = {}
    if world == 1 and not args.no_extras:
        for nm in EXTRA_WORKLOADS + sorted(W.GR_WORKLOADS) + sorted(W.UK_WORKLOADS):
            if nm != w.name:
                others[nm] = time_other(nm, dev, min(K, args.extra_steps), flush, pk, ffma)

    st = R_status()
    if st != 0:
        raise RuntimeError(f"device status after timing: {st}")
    if rank == 0:
        ms = t_max / K
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
                "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": w.dtype, "data": "synthetic", "config": config_of(w), "roofline": roof,
                "step_roofline": step_roofline(w, ms, pk, ffma),
                "parity": {"check": "adjoint identity <dY,y> = <dcoef,coef> (+<dw_base,w_base>) per layer, "
                                    "relative to sum|dY*y|", "rel_err": adj, "tol": tol,
                           "ok": all(v <= tol for v in adj.values())},
                "e2e": e2e, "gpu_launches": launches, "clocks": clocks, "wall_s": wall,
                "ffma_peak_tflops": ffma, "peaks": pk}
        if others:
            line["other_workloads"] = others
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w)
        print(json.dumps(line), flush=True)


def R_status():
    from kolmogorov_arnold_network_b200 import _native as N
    return N.kan_sync_status(None)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--extra-steps", type=int, default=30)
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--workload", default=W.BENCH_DEFAULT, choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", default=None,
                    choices=sorted(set(W.WORKLOADS) | set(W.GR_WORKLOADS) | set(W.UK_WORKLOADS)),
                    help="time one workload by itself (one GPU) and print its own JSON line")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_setup() if args.impl == "ours" else (int(os.environ.get("WORLD_SIZE", "1")),
                                                                    int(os.environ.get("RANK", "0")), 0)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        elif args.only:
            if world > 1:
                raise SystemExit("--only runs on one GPU")
            run_only(args, local)
        else:
            run_ours(args, world, rank, local)
    finally:
        if args.impl == "ours" and world > 1 and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()

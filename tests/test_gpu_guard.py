"""Out-of-bounds stores, detected without a memory checker.

Every output buffer (y, dx, dcoef, dw_base) and the workspace are carved out
of a larger allocation with guard bands of a known bit pattern on both sides.
After a forward and a backward on the ragged shapes of the parity suite (odd
M-tile counts, N not a multiple of the tile, unaligned x rows, CTA pairs with
a padding tile), on both kernel families, the guard bands must be untouched
and no element inside an output may still hold the pattern (every element
written).  A store that lands just past the end of a row block, or a skipped
tile, fails here even when parity, which reads only in-bounds elements, would
pass.
"""
import numpy as np
import pytest
import torch

from kolmogorov_arnold_network_b200 import _native as N
from kolmogorov_arnold_network_b200 import layer as L
from kolmogorov_arnold_network_b200 import workloads as W

from gpu_util import workload_inputs
from test_gpu_parity import SMALL

pytestmark = pytest.mark.gpu

GUARD_BYTES = 512          # each side; a multiple of 16 keeps the carved buffers 16-byte aligned
PATTERN = {torch.float32: (torch.int32, 0x7FA5A5A5), torch.bfloat16: (torch.int16, 0x7FA5),
           torch.uint8: (torch.uint8, 0xA5)}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


class Guarded:
    """A tensor of `shape` inside a buffer with pattern-filled guard bands on both sides."""

    def __init__(self, shape, dtype):
        self.dtype = dtype
        esz = torch.empty((), dtype=dtype).element_size()
        self.g = GUARD_BYTES // esz
        self.n = int(np.prod(shape))
        self.buf = torch.empty(self.n + 2 * self.g, dtype=dtype, device="cuda")
        idt, pat = PATTERN[dtype]
        signed = idt != torch.uint8
        self.buf.view(idt).fill_(pat if not signed or pat < 2 ** (8 * esz - 1) else pat - 2 ** (8 * esz))
        self.t = self.buf[self.g:self.g + self.n].view(shape)
        assert self.t.data_ptr() % 16 == 0

    def check(self, name, all_written=True):
        idt, pat = PATTERN[self.dtype]
        bits = self.buf.view(idt).cpu().numpy().astype(np.int64) & ((1 << (8 * self.buf.element_size())) - 1)
        assert np.all(bits[:self.g] == pat), f"{name}: guard band before the buffer was written"
        assert np.all(bits[self.g + self.n:] == pat), f"{name}: guard band after the buffer was written"
        if all_written:
            assert not np.any(bits[self.g:self.g + self.n] == pat), f"{name}: elements left unwritten"


CASES = [c + (3,) for c in SMALL] + [
    # other spline degrees: k+1 weights per input in the producers and the dx gather
    (300, 16, 256, 8, -1.0, 1.0, True, 1), (800, 24, 296, 20, -1.0, 1.0, False, 5),
    (300, 40, 296, 8, -1.0, 1.0, False, 2), (257, 24, 64, 20, -1.0, 1.0, True, 4),
    # bf16: dcoef with the outputs on M (DCB, TMA-stored), a ragged last M tile / a ragged last N tile and
    # rows of x that are not 16-byte aligned
    (300, 1536, 648, 5, -3.0, 3.0, False, 3), (257, 1532, 768, 5, -3.0, 3.0, False, 3)]


@pytest.mark.parametrize("path", [N.KAN_PATH_TENSOR, N.KAN_PATH_SIMT], ids=["tensor", "simt"])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "b{}_i{}_o{}_g{}{}_k{}".format(c[0], c[1], c[2], c[3],
                                                                                         "_silu" if c[6] else "", c[7]))
def test_no_store_outside_the_outputs(path, dt, case):
    batch, n_in, n_out, G, lo, hi, base, k = case
    w = W.custom(batch, n_in, n_out, G, lo, hi, dtype=dt, base=base, degree=k)
    x, coef, wb, dY = (None if t is None else t.cuda() for t in workload_inputs(w))
    tdt = x.dtype
    s = L.shape_of(x, coef, G, lo, hi, wb, path, degree=k)
    y = Guarded((batch, n_out), tdt)
    dx = Guarded((batch, n_in), tdt)
    dc = Guarded(tuple(coef.shape), torch.float32)
    dwb = Guarded(tuple(wb.shape), torch.float32) if wb is not None else None
    wsf = Guarded((max(1, N.kan_workspace_size(s, False)),), torch.uint8)
    wsb = Guarded((max(1, N.kan_workspace_size(s, True)),), torch.uint8)
    L.forward(x, coef, G, lo, hi, wb, path=path, y=y.t, ws=wsf.t, degree=k)
    L.backward(x, coef, dY, G, lo, hi, wb, path=path, out=(dx.t, dc.t, None if dwb is None else dwb.t), ws=wsb.t,
               degree=k)
    torch.cuda.synchronize()
    assert N.kan_sync_status(None) == 0
    y.check("y")
    dx.check("dx")
    dc.check("dcoef")
    if dwb is not None:
        dwb.check("dw_base")
    # the workspace need not be written everywhere, but nothing may land outside it
    wsf.check("forward workspace", all_written=False)
    wsb.check("backward workspace", all_written=False)

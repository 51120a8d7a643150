"""Out-of-bounds write checks: every output (y, dx, dA, dB) and the workspace sit
between sentinel regions inside larger device buffers, and every kernel path
(TMA-pipelined with lane stores or TMA tensor stores, generic; both element
types; ragged row tiles; boxes that do not fill every lane slot; the one-pass
forward + backward; the host-buffer step's device scratch is covered by its own
exact-equality test) must leave the sentinels and the inputs untouched. The
sentinels sit right against each region, so a store one element past either end
is caught."""
import numpy as np
import pytest
import torch

import group_rational_kan_b200 as grk
import synth
from parity import to_torch

pytestmark = pytest.mark.gpu

GUARD = 512          # sentinel bytes on each side
FILL = 0xA5          # sentinel byte


def _custom(name, rows, d, n_g, dtype):
    return synth.Workload(name=name, B=rows, N=1, d=d, n_g=n_g, m=5, n=4, dtype=dtype,
                          x_kind=synth.KIND_NORMAL, x_scale=1.0, x_clip=8.0, dy_scale=1.0,
                          coef_base="zero", coef_lo=-0.5, coef_hi=0.5)


CASES = [
    synth.workload("kat_b").with_rows(333),       # bf16, lane stores, ragged last tile
    synth.workload("kat_t").with_rows(301),       # float32, TMA tensor stores, ragged
    synth.workload("stress", n_g=64).with_rows(77),
    _custom("box_partial_f32", 301, 160, 4, synth.F32),   # boxes not filling every slot
    _custom("box_partial_bf16", 301, 160, 4, synth.BF16),
    _custom("generic_f32", 77, 30, 3, synth.F32),         # 40-byte groups: generic path
    _custom("dg1_f32", 45, 16, 16, synth.F32),             # one channel per group
]


class Guarded:
    """A region of `nbytes` at byte offset GUARD (+ shift) inside a buffer filled
    with the sentinel; check() verifies both sides."""

    def __init__(self, nbytes, shift=0):
        self.nbytes, self.shift = nbytes, shift
        self.buf = torch.full((GUARD + shift + nbytes + GUARD,), FILL, dtype=torch.uint8,
                              device="cuda")

    def view(self, dtype, shape):
        off = GUARD + self.shift
        return self.buf[off:off + self.nbytes].view(dtype).view(shape)

    def check(self, what):
        b = self.buf.cpu().numpy()
        lo = b[:GUARD + self.shift]
        hi = b[GUARD + self.shift + self.nbytes:]
        assert np.all(lo == FILL), "%s: write before the region" % what
        assert np.all(hi == FILL), "%s: write after the region" % what


def _tdt(w):
    return torch.float32 if w.dtype == synth.F32 else torch.bfloat16


@pytest.mark.parametrize("flags", [0, grk.FLAG_GENERIC], ids=["auto", "generic"])
@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_outputs_stay_inside_their_regions(w, flags):
    x, dy = w.x(), w.dy()
    a, b = w.coefficients()
    tx, tdy = to_torch(x), to_torch(dy)
    x0, dy0 = tx.clone(), tdy.clone()
    ta, tb = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
    es = 4 if w.dtype == synth.F32 else 2
    nb = w.rows * w.d * es
    shape = (w.rows, w.d)
    args = (w.rows, 1, w.d, w.n_g, w.m, w.n, w.dtype)
    wsb = grk.grkan_backward_workspace_bytes(*args)

    gy, gdx, gfy, gfdx = (Guarded(nb) for _ in range(4))
    gA, gB = Guarded(w.n_g * (w.m + 1) * 4), Guarded(w.n_g * w.n * 4)
    gws = Guarded(max(wsb, 16))
    y, dx = gy.view(_tdt(w), shape), gdx.view(_tdt(w), shape)
    dA = gA.view(torch.float32, (w.n_g, w.m + 1))
    dB = gB.view(torch.float32, (w.n_g, w.n))
    ws = gws.view(torch.uint8, (max(wsb, 16),))

    assert grk.grkan_forward_ex(tx, y, ta, tb, *args, flags) == 0
    assert grk.grkan_backward_ex(tx, tdy, ta, tb, dx, dA, dB, *args, ws, wsb, flags) == 0
    torch.cuda.synchronize()
    for g, nm in ((gy, "y"), (gdx, "dx"), (gA, "dA"), (gB, "dB"), (gws, "workspace")):
        g.check("%s %s" % (w.name, nm))
    # the outputs are the library's own results, not sentinel bytes
    ry = grk.forward(tx, ta, tb, w.n_g, flags=flags)
    rdx, rdA, rdB = grk.backward(tx, tdy, ta, tb, w.n_g, flags=flags)
    assert torch.equal(y, ry) and torch.equal(dx, rdx)
    assert torch.equal(dA, rdA) and torch.equal(dB, rdB)

    # the one-pass forward + backward
    fy, fdx = gfy.view(_tdt(w), shape), gfdx.view(_tdt(w), shape)
    assert grk.grkan_forward_backward(tx, tdy, ta, tb, fy, fdx, dA, dB, *args, ws, wsb,
                                      flags) == 0
    torch.cuda.synchronize()
    for g, nm in ((gfy, "one-pass y"), (gfdx, "one-pass dx"), (gA, "one-pass dA"),
                  (gB, "one-pass dB"), (gws, "one-pass workspace")):
        g.check("%s %s" % (w.name, nm))
    assert torch.equal(fy, ry) and torch.equal(fdx, rdx)

    # the inputs are read, never written
    assert torch.equal(tx, x0) and torch.equal(tdy, dy0)
    assert grk.grkan_device_error()[1] == 0


@pytest.mark.parametrize("dtype", [synth.F32, synth.BF16])
def test_unaligned_outputs_stay_inside_their_regions(dtype):
    """Outputs shifted off the 16-byte grid (the generic kernels take them)."""
    w = (synth.workload("kat_t") if dtype == synth.F32 else synth.workload("kat_b")).with_rows(70)
    x, dy = w.x(), w.dy()
    a, b = w.coefficients()
    tx, tdy = to_torch(x), to_torch(dy)
    ta, tb = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
    es = 4 if dtype == synth.F32 else 2
    nb = w.rows * w.d * es
    args = (w.rows, 1, w.d, w.n_g, w.m, w.n, w.dtype)
    gy, gdx = Guarded(nb, shift=es), Guarded(nb, shift=es)
    y, dx = gy.view(_tdt(w), (w.rows, w.d)), gdx.view(_tdt(w), (w.rows, w.d))
    assert grk.grkan_backward_path(tx, tdy, dx, *args) == 0
    wsb = grk.grkan_backward_workspace_bytes(*args)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device="cuda")
    dA = torch.empty(w.n_g, w.m + 1, device="cuda")
    dB = torch.empty(w.n_g, w.n, device="cuda")
    assert grk.grkan_forward(tx, y, ta, tb, *args) == 0
    assert grk.grkan_backward(tx, tdy, ta, tb, dx, dA, dB, *args, ws, wsb) == 0
    torch.cuda.synchronize()
    gy.check("unaligned y")
    gdx.check("unaligned dx")
    assert torch.equal(y, grk.forward(tx, ta, tb, w.n_g))

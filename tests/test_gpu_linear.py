"""GR-KAN fused into the following linear layer (grkan_linear_forward) against
the fp64 oracle's activation times the weight in fp64, and against the same
product taken from the library's own forward output. The shapes reach both
kernels behind the call (one CTA per 128 x 512 tile for n_out up to 512, CTA
clusters of four for wider outputs) and span several row and column tiles, a
ragged last tile in both, more K steps than any ring has stages, more tiles than
resident clusters, groups that straddle a 64-channel K step, bias and no bias.
The output is written inside its region only."""
import numpy as np
import pytest
import torch

import group_rational_kan_b200 as grk
import oracle
import synth
from parity import to_f64, to_torch

pytestmark = pytest.mark.gpu


def _case(rows, d, n_g, nout, seed=0, dy_scale=1.0):
    w = synth.Workload(name="lin", B=rows, N=1, d=d, n_g=n_g, m=5, n=4, dtype=synth.BF16,
                       x_kind=synth.KIND_NORMAL, x_scale=1.0, x_clip=8.0, dy_scale=dy_scale,
                       coef_base="zero", coef_lo=-0.5, coef_hi=0.5, seed=seed)
    x = w.x()
    a, b = w.coefficients()
    # the weight: seeded bf16 from the same generator (the dy stream, scaled)
    wt = synth.Workload(name="lin_w", B=nout, N=1, d=d, n_g=n_g, m=5, n=4, dtype=synth.BF16,
                        x_kind=synth.KIND_NORMAL, x_scale=1.0, x_clip=8.0,
                        dy_scale=1.0 / np.sqrt(d), coef_base="zero", coef_lo=-0.5,
                        coef_hi=0.5, seed=seed + 1).dy()
    bias = np.linspace(-0.25, 0.25, nout).astype(np.float32)
    return w, x, a, b, wt, bias


def _reference(w, x, a, b, wt, bias):
    y = oracle.forward(x, a, b, w.n_g)  # fp64
    W = synth.bf16_bits_to_f32(wt).astype(np.float64)
    ref = y @ W.T
    scale = np.abs(y) @ np.abs(W).T
    if bias is not None:
        ref = ref + bias.astype(np.float64)[None, :]
    return ref, scale


@pytest.mark.parametrize("rows,d,n_g,nout,with_bias", [
    (300, 768, 8, 576, True),     # d_g 96: ragged rows and columns; second tile half-empty
    (128, 256, 4, 256, False),    # one tile, first half only
    (256, 512, 4, 1024, True),    # two full 512-column tiles
    (1000, 3072, 8, 768, True),   # the KAT-B second-linear shape, ragged rows
    (200, 1536, 16, 200, False),  # n_out not a multiple of 64: the store box is clipped
    (130, 160, 20, 520, True),    # d_g 8 (many groups per K step), n_out just past a tile
    (300, 1536, 8, 384, True),    # second half 128 wide (narrower MMA)
    (200, 512, 8, 296, False),    # second half 40 wide: MMA width 48, store clipped at 296
    (20000, 512, 8, 768, True),   # more 256-row tiles than resident CTAs: persistent walk
    (700, 256, 4, 1536, False),   # n_out past 1024: two column tiles of a cluster
    (600, 1024, 16, 2048, True),  # two column tiles of 1024
    (300, 768, 8, 3072, True),    # the KAT second-linear's transpose: three column tiles
    (100, 512, 8, 640, False),    # one ragged 256-row tile: half of it past the last row
])
def test_fused_linear_matches_oracle(rows, d, n_g, nout, with_bias):
    w, x, a, b, wt, bias = _case(rows, d, n_g, nout)
    tx = to_torch(x)
    tw = to_torch(wt)
    ta = torch.from_numpy(a).cuda()
    tb = torch.from_numpy(b).cuda()
    tbias = torch.from_numpy(bias).cuda() if with_bias else None
    out = grk.linear_forward(tx, ta, tb, n_g, tw, tbias)
    torch.cuda.synchronize()
    assert grk.grkan_device_error()[1] == 0
    got = to_f64(out)
    ref, scale = _reference(w, x, a, b, wt, bias if with_bias else None)
    # y rounded to bf16 (2^-9 relative per term), float32 sums, bf16 output (2^-9)
    lim = 2.0 ** -8 * scale + 2.0 ** -8 * np.abs(ref) + 1e-6
    err = np.abs(got - ref)
    assert np.all(err <= lim), "worst %.3g of limit" % float(np.max(err / lim))

    # the unfused composition: the library's forward (same y bits), then the
    # product in float32 on the device
    y = grk.forward(tx, ta, tb, n_g)
    ref2 = y.float() @ tw.float().T
    if with_bias:
        ref2 += tbias
    ref2 = ref2.double().cpu().numpy()
    err2 = np.abs(got - ref2)
    lim2 = 2.0 ** -8 * np.abs(ref2) + 1e-5 * scale + 1e-6
    assert np.all(err2 <= lim2), "worst %.3g of limit" % float(np.max(err2 / lim2))


def test_fused_linear_rejects_unsupported():
    t = torch.empty(64, dtype=torch.bfloat16, device="cuda")
    f = torch.empty(16, device="cuda")
    args = (1, 1, 64, 8, 5, 4, 64)
    assert grk.grkan_linear_forward(t, f, f, t, None, t, *args, grk.F32) == 4  # dtype
    assert grk.grkan_linear_forward(t, f, f, t, None, t, 1, 1, 64, 8, 3, 3, 64,
                                    grk.BF16) == 3  # degree
    assert grk.grkan_linear_forward(t, f, f, t, None, t, 1, 1, 48, 6, 5, 4, 64,
                                    grk.BF16) == 2  # d % 32
    assert grk.grkan_linear_forward(t, f, f, t, None, t, 0, 1, 64, 8, 5, 4, 64,
                                    grk.BF16) == 0  # empty: nothing to do
    assert grk.grkan_linear_forward(t, f, f, t, None, t, 1, 1, 0, 8, 5, 4, 64,
                                    grk.BF16) == 2  # d == 0


@pytest.mark.parametrize("rows,d,nout", [(333, 512, 296), (333, 512, 768), (77, 768, 2048)])
def test_fused_linear_writes_only_its_output(rows, d, nout):
    """out sits between sentinel bytes; both kernels' clipped TMA stores (ragged
    rows and columns) leave them untouched."""
    n_g = 8
    w, x, a, b, wt, bias = _case(rows, d, n_g, nout)
    guard = 4096
    nb = rows * nout * 2
    buf = torch.full((guard + nb + guard,), 0xA5, dtype=torch.uint8, device="cuda")
    out = buf[guard:guard + nb].view(torch.bfloat16).view(rows, nout)
    tx, tw = to_torch(x), to_torch(wt)
    ta, tb = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
    assert grk.grkan_linear_forward(tx, ta, tb, tw, None, out, rows, 1, d, n_g, 5, 4, nout,
                                    grk.BF16) == 0
    torch.cuda.synchronize()
    host = buf.cpu().numpy()
    assert np.all(host[:guard] == 0xA5) and np.all(host[guard + nb:] == 0xA5)
    ref = grk.linear_forward(tx, ta, tb, n_g, tw, None)
    assert torch.equal(out, ref)
    assert grk.grkan_device_error()[1] == 0


@pytest.mark.parametrize("rows,d,with_bias", [(1000, 3072, True), (333, 512, False)])
def test_fused_linear_kernels_agree(rows, d, with_bias):
    """n_out = 768 takes the cluster kernel, n_out <= 512 the one-CTA kernel. Every
    output element is the same bf16 y row times one W row, summed over K in the
    same 16-wide slices in the same order, so the 768 columns equal, bit for bit,
    the one-CTA kernel's results for the column slices [0, 512) and [512, 768)."""
    n_g, nout = 8, 768
    w, x, a, b, wt, bias = _case(rows, d, n_g, nout)
    tx, tw = to_torch(x), to_torch(wt)
    ta, tb = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
    tbias = torch.from_numpy(bias).cuda() if with_bias else None
    full = grk.linear_forward(tx, ta, tb, n_g, tw, tbias)
    lo = grk.linear_forward(tx, ta, tb, n_g, tw[:512].contiguous(),
                            tbias[:512].contiguous() if with_bias else None)
    hi = grk.linear_forward(tx, ta, tb, n_g, tw[512:].contiguous(),
                            tbias[512:].contiguous() if with_bias else None)
    torch.cuda.synchronize()
    assert torch.equal(full[:, :512], lo) and torch.equal(full[:, 512:], hi)
    assert grk.grkan_device_error()[1] == 0

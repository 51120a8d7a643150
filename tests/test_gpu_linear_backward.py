"""GR-KAN backward fused into the linear layer's data-gradient product
(grkan_linear_backward) against the fp64 oracle.

The reference gradient of the activation's output is dy = dout W in fp64 from
the same bf16 operands, rounded to float32 for the oracle (x widened exactly).
The kernel's dy is the tensor cores' float32 sum of nout products, so the
tolerances add that sum's rounding to the oracle tolerances of grkan_backward:
  dx: n_out 2^-24 sum_o |dout W| times the oracle's bound on |dy/dx| (its
      kappa_dx at dy = 1), element by element;
  dA, dB: the random part of the same rounding over the group's elements,
      6 sqrt(n_out) 2^-24 sqrt(sum_e (sum_o |dout W| |term_e / dy_e|)^2).
Shapes span several 128-row and 192-channel tiles, ragged last tiles in rows,
channels and output features, more K steps than the three-stage ring, more
tiles than SMs (each CTA loops), one-group-per-block and many-blocks-per-group
layouts."""
import numpy as np
import pytest
import torch

import group_rational_kan_b200 as grk
import oracle
import synth
from parity import check_coef, check_dx, to_f64, to_torch

pytestmark = pytest.mark.gpu

U = 2.0 ** -24


def _case(rows, d, n_g, nout, seed=0):
    w = synth.Workload(name="lin_bwd", B=rows, N=1, d=d, n_g=n_g, m=5, n=4, dtype=synth.BF16,
                       x_kind=synth.KIND_NORMAL, x_scale=1.0, x_clip=8.0, dy_scale=1.0,
                       coef_base="zero", coef_lo=-0.5, coef_hi=0.5, seed=seed)
    x = w.x()
    a, b = w.coefficients()
    # dout (rows x nout) and W (nout x d): seeded bf16 from the same generator
    dout = synth.Workload(name="lin_dout", B=rows, N=1, d=max(nout, 8), n_g=1, m=5, n=4,
                          dtype=synth.BF16, x_kind=synth.KIND_NORMAL, x_scale=1.0, x_clip=8.0,
                          dy_scale=1e-2, coef_base="zero", coef_lo=-0.5, coef_hi=0.5,
                          seed=seed + 2).dy()[:, :nout]
    W = synth.Workload(name="lin_w", B=max(nout, 1), N=1, d=d, n_g=n_g, m=5, n=4,
                       dtype=synth.BF16, x_kind=synth.KIND_NORMAL, x_scale=1.0, x_clip=8.0,
                       dy_scale=1.0 / np.sqrt(max(nout, 1)), coef_base="zero", coef_lo=-0.5,
                       coef_hi=0.5, seed=seed + 1).dy()[:nout]
    return w, x, a, b, np.ascontiguousarray(dout), np.ascontiguousarray(W)


def _run(x, dout, W, a, b, n_g):
    tx, tdo, tw = to_torch(x), to_torch(dout), to_torch(W)
    ta = torch.from_numpy(a).cuda()
    tb = torch.from_numpy(b).cuda()
    dx, dA, dB = grk.linear_backward(tx, tdo, tw, ta, tb, n_g)
    torch.cuda.synchronize()
    assert grk.grkan_device_error()[1] == 0
    return dx, dA, dB


def _check(x, dout, W, a, b, n_g, got_dx, dA, dB):
    nout = W.shape[0]
    do64 = synth.bf16_bits_to_f32(dout).astype(np.float64)
    w64 = synth.bf16_bits_to_f32(W).astype(np.float64)
    dy64 = do64 @ w64
    S = np.abs(do64) @ np.abs(w64)  # sum_o |dout W| per element
    x32 = synth.bf16_bits_to_f32(x)
    dy32 = dy64.astype(np.float32)
    ref, ex = oracle.backward_elem(x32, dy32, a, b, n_g, extras=True)
    # the oracle's bound on |dy/dx| per element: kappa_dx at dy = 1
    _, ex1 = oracle.backward_elem(x32, np.ones_like(x32), a, b, n_g, extras=True)
    extra_dx = nout * U * S * ex1["kappa_dx"] + 2.0 * U * np.abs(dy64) * ex1["kappa_dx"]
    got = to_f64(got_dx).reshape(ref.shape)
    err = np.abs(got - ref)
    kap = ex["kappa_dx"]
    ok = err <= 1e-2 * (np.abs(ref) + kap) + extra_dx
    if not ok.all():  # elements at the kink of |Q|: check_dx also takes the other branches
        ex = dict(ex)
        ex["kappa_dx"] = kap + extra_dx / 1e-2
        check_dx(got, ref, ex, 1e-2, what="dx")

    coef = oracle.coef_grads(x32, dy32, a, b, n_g)
    # random rounding of dy: per-term weights |x|^i / D and |y| |x|^j / D
    d = x.shape[1]
    dg = d // n_g
    xa = np.abs(x32.astype(np.float64))
    q = ex["q"]
    D = 1.0 + np.abs(q)
    y = oracle.forward(x32, a, b, n_g)
    extra_A = np.zeros((n_g, 6))
    extra_B = np.zeros((n_g, 4))
    for g in range(n_g):
        sl = slice(g * dg, (g + 1) * dg)
        s = S[:, sl] / D[:, sl]
        xs = xa[:, sl]
        ys = np.abs(y[:, sl])
        for i in range(6):
            extra_A[g, i] = np.sqrt(np.sum((s * xs ** i) ** 2))
        for j in range(1, 5):
            extra_B[g, j - 1] = np.sqrt(np.sum((s * ys * xs ** j) ** 2))
    k = 6.0 * np.sqrt(max(nout, 1)) * U
    coef = dict(coef)
    coef["c2_a"] = (np.sqrt(coef["c2_a"]) + k * extra_A / 2e-6) ** 2
    coef["c2_b"] = (np.sqrt(coef["c2_b"]) + k * extra_B / 2e-6) ** 2
    check_coef(dA.cpu().numpy(), dB.cpu().numpy(), coef, what="linear backward")


@pytest.mark.parametrize("rows,d,n_g,nout", [
    (300, 768, 4, 576),     # d_g 192: ragged rows (a quarter with no rows), 9 K steps
    (128, 192, 1, 64),      # one tile, one K step
    (1000, 3072, 8, 768),   # the KAT-B layer shape, ragged rows
    (4000, 3072, 8, 256),   # 512 tiles: every CTA loops over several
    (200, 320, 5, 128),     # d_g 64: last column tile 128 wide (N 128, one warp column idle)
    (260, 448, 7, 200),     # last column tile 64 wide, last K step partly past nout
    (130, 1536, 8, 8),      # nout 8: one K step, mostly zero-filled
    (300, 6144, 96, 64),    # 96 groups: coefficients from global memory, not the table
    (1, 384, 2, 64),        # one row: the pair's second CTA and 127 rows are past the end
    (256, 384, 2, 4096),    # 64 K steps through the ring
])
def test_fused_linear_backward_matches_oracle(rows, d, n_g, nout):
    w, x, a, b, dout, W = _case(rows, d, n_g, nout)
    dx, dA, dB = _run(x, dout, W, a, b, n_g)
    _check(x, dout, W, a, b, n_g, dx, dA, dB)


def test_fused_linear_backward_is_deterministic():
    w, x, a, b, dout, W = _case(2000, 1536, 8, 384, seed=5)
    r1 = _run(x, dout, W, a, b, 8)
    r2 = _run(x, dout, W, a, b, 8)
    for u, v in zip(r1, r2):
        assert torch.equal(u, v)


def test_fused_linear_backward_degenerate_sizes():
    n_g, d = 4, 256
    a = torch.from_numpy(np.linspace(-0.5, 0.5, n_g * 6).astype(np.float32)).cuda().view(n_g, 6)
    b = torch.from_numpy(np.linspace(-0.5, 0.5, n_g * 4).astype(np.float32)).cuda().view(n_g, 4)
    # no output features: dy = 0, so dx = 0 and the gradients are 0
    x = torch.randn(64, d, device="cuda").to(torch.bfloat16)
    dout = torch.empty(64, 0, device="cuda", dtype=torch.bfloat16)
    W = torch.empty(0, d, device="cuda", dtype=torch.bfloat16)
    dx = torch.full_like(x, 3.0)
    dA = torch.full((n_g, 6), 7.0, device="cuda")
    dB = torch.full((n_g, 4), 7.0, device="cuda")
    grk.linear_backward(x, dout, W, a, b, n_g, dx=dx, dA=dA, dB=dB)
    torch.cuda.synchronize()
    assert torch.count_nonzero(dx).item() == 0
    assert torch.count_nonzero(dA).item() == 0 and torch.count_nonzero(dB).item() == 0
    # no rows: zero gradients
    x0 = torch.empty(0, d, device="cuda", dtype=torch.bfloat16)
    dout0 = torch.empty(0, 64, device="cuda", dtype=torch.bfloat16)
    W0 = torch.randn(64, d, device="cuda").to(torch.bfloat16)
    dA.fill_(7.0)
    dB.fill_(7.0)
    grk.linear_backward(x0, dout0, W0, a, b, n_g, dA=dA, dB=dB)
    torch.cuda.synchronize()
    assert torch.count_nonzero(dA).item() == 0 and torch.count_nonzero(dB).item() == 0


def test_fused_linear_backward_rejects():
    n_g, d, rows, nout = 4, 256, 64, 64
    a = torch.zeros(n_g, 6, device="cuda")
    b = torch.zeros(n_g, 4, device="cuda")
    x = torch.zeros(rows, d, device="cuda", dtype=torch.bfloat16)
    dout = torch.zeros(rows, nout, device="cuda", dtype=torch.bfloat16)
    W = torch.zeros(nout, d, device="cuda", dtype=torch.bfloat16)
    dx = torch.empty_like(x)
    dA = torch.empty(n_g, 6, device="cuda")
    dB = torch.empty(n_g, 4, device="cuda")
    wsb = grk.grkan_linear_backward_workspace_bytes(1, rows, d, n_g, 5, 4, nout, grk.BF16)
    assert wsb == (rows + 127) // 128 * (d // n_g // 64) * 4 * n_g * 10 * 4
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")

    def call(x=x, dout=dout, W=W, dx=dx, d=d, n_g=n_g, nout=nout, dtype=grk.BF16, m=5, n=4,
             ws=ws, wsb=wsb):
        return grk.grkan_linear_backward(x, dout, W, a, b, dx, dA, dB, 1, rows, d, n_g, m, n, nout,
                                         dtype, ws, wsb)

    assert call() == 0
    assert call(dtype=grk.F32) == 4                    # bf16 only
    assert call(m=4, n=4) == 3                         # (5, 4) only
    assert call(n_g=8) == 2                            # d_g 32: not a multiple of 64
    assert call(nout=60) == 2                          # nout % 8
    assert call(wsb=wsb - 4) == 5                      # workspace too small
    assert call(dx=dout) == 7                          # dx overlaps dout
    assert call(ws=dx, wsb=wsb) == 7                   # workspace overlaps dx
    assert grk.grkan_linear_backward_workspace_bytes(1, rows, d, 8, 5, 4, nout, grk.BF16) == 0
    torch.cuda.synchronize()
    assert grk.grkan_device_error()[1] == 0

"""CUDA path vs the fp64 oracle, element by element, on seeded inputs that span
several tiles and a ragged tail; both kernel paths (TMA-pipelined and generic),
both dtypes, other degrees, odd shapes and the edge cases. Calls go through the
C ABI (via the thin binding)."""
import numpy as np
import pytest
import torch

import group_rational_kan_b200 as grk
import oracle
import synth
from parity import RTOL, check_coef, check_dx, check_y, to_f64, to_torch

pytestmark = pytest.mark.gpu


def _custom(name, rows, d, n_g, m, n, dtype, x_kind=synth.KIND_NORMAL, dy_scale=1.0, lo=-0.5,
            hi=0.5):
    return synth.Workload(name=name, B=rows, N=1, d=d, n_g=n_g, m=m, n=n, dtype=dtype,
                          x_kind=x_kind, x_scale=1.0, x_clip=8.0, dy_scale=dy_scale,
                          coef_base="zero", coef_lo=lo, coef_hi=hi)


CASES = {
    "tiny": synth.workload("tiny"),
    "kat_t_ragged": synth.workload("kat_t").with_rows(700),
    "kat_s_ragged": synth.workload("kat_s").with_rows(333),
    "kat_b_ragged": synth.workload("kat_b").with_rows(333),
    "stress_ng1": synth.workload("stress", n_g=1).with_rows(150),
    "stress_ng8": synth.workload("stress", n_g=8).with_rows(150),
    "stress_ng64": synth.workload("stress", n_g=64).with_rows(150),
    "one_row_bf16": synth.workload("kat_b").with_rows(1),
    "odd_f32_dg10": _custom("odd_f32", 77, 30, 3, 5, 4, synth.F32),
    "odd_bf16_dg6": _custom("odd_bf16", 91, 24, 4, 5, 4, synth.BF16),
    # TMA-pipelined boxes that do not fill every lane's vector slots (40-channel
    # groups: 9-row float32 / 38-row bf16 backward boxes), through the staged
    # TMA stores (float32) and the buffered guarded stores (bf16)
    "box_partial_f32_dg40": _custom("box_f32_dg40", 301, 160, 4, 5, 4, synth.F32),
    "box_partial_bf16_dg40": _custom("box_bf16_dg40", 301, 160, 4, 5, 4, synth.BF16),
    # one channel per group (d_g = 1): every channel its own coefficients
    "dg1_f32": _custom("dg1_f32", 45, 16, 16, 5, 4, synth.F32),
    "dg1_bf16": _custom("dg1_bf16", 45, 16, 16, 5, 4, synth.BF16),
    "deg_3_2": _custom("deg_3_2", 100, 384, 4, 3, 2, synth.BF16),
    "deg_0_0": _custom("deg_0_0", 60, 64, 2, 0, 0, synth.F32),
    "deg_8_8": _custom("deg_8_8", 60, 64, 4, 8, 8, synth.F32, x_kind=synth.KIND_NORMAL,
                       lo=-0.2, hi=0.2),
    "deg_5_0": _custom("deg_5_0", 60, 128, 8, 5, 0, synth.BF16),
    "deg_2_6": _custom("deg_2_6", 60, 96, 3, 2, 6, synth.F32),
    # degrees with TMA-pipelined kernels besides (5, 4): several tiles and a ragged tail
    "deg_3_3_bf16": _custom("deg_3_3", 530, 256, 4, 3, 3, synth.BF16),
    "deg_4_4_f32": _custom("deg_4_4", 410, 256, 4, 4, 4, synth.F32),
    "deg_5_5_bf16": _custom("deg_5_5", 530, 256, 4, 5, 5, synth.BF16),
    "deg_6_6_f32": _custom("deg_6_6", 410, 256, 4, 6, 6, synth.F32, lo=-0.3, hi=0.3),
    "deg_7_7_bf16": _custom("deg_7_7", 530, 256, 4, 7, 7, synth.BF16, lo=-0.3, hi=0.3),
    "deg_8_8_bf16": _custom("deg_8_8b", 530, 256, 4, 8, 8, synth.BF16, lo=-0.2, hi=0.2),
    # more groups than the kernels' shared coefficient table holds (64)
    "ng96_bf16": _custom("ng96", 200, 3072, 96, 5, 4, synth.BF16),
    "ng128_f32_deg66": _custom("ng128", 120, 3072, 128, 6, 6, synth.F32, lo=-0.3, hi=0.3),
}

_cache = {}


def case_data(name):
    if name not in _cache:
        w = CASES[name]
        x, dy = w.x(), w.dy()
        a, b = w.coefficients()
        y_ref, ky = oracle.forward(x, a, b, w.n_g, kappa=True)
        dx_ref, ex = oracle.backward_elem(x, dy, a, b, w.n_g, extras=True)
        g_ref = oracle.coef_grads(x, dy, a, b, w.n_g)
        _cache[name] = (w, x, dy, a, b, y_ref, ky, dx_ref, ex, g_ref)
    return _cache[name]


def _dev(w, x, dy, a, b):
    return (to_torch(x), to_torch(dy), torch.from_numpy(a).cuda(),
            torch.from_numpy(b.reshape(w.n_g, w.n)).cuda())


@pytest.mark.parametrize("flags", [0, grk.FLAG_GENERIC], ids=["auto", "generic"])
@pytest.mark.parametrize("name", list(CASES))
def test_forward_backward_parity(name, flags):
    w, x, dy, a, b, y_ref, ky, dx_ref, ex, g_ref = case_data(name)
    tx, tdy, ta, tb = _dev(w, x, dy, a, b)
    y = grk.forward(tx, ta, tb, w.n_g, flags=flags)
    dx, dA, dB = grk.backward(tx, tdy, ta, tb, w.n_g, flags=flags)
    torch.cuda.synchronize()
    rtol = RTOL[w.dtype]
    check_y(to_f64(y), y_ref, ky, rtol, "%s y" % name)
    check_dx(to_f64(dx), dx_ref, ex, rtol, "%s dx" % name)
    check_coef(dA.cpu().numpy(), dB.cpu().numpy(), g_ref, what=name)
    assert grk.grkan_device_error()[1] == 0


def test_fast_path_is_taken_where_expected():
    for name in ("tiny", "kat_t_ragged", "kat_s_ragged", "kat_b_ragged", "stress_ng1",
                 "stress_ng8", "stress_ng64", "one_row_bf16", "deg_8_8", "deg_3_3_bf16",
                 "deg_4_4_f32", "deg_5_5_bf16", "deg_6_6_f32", "deg_7_7_bf16", "deg_8_8_bf16",
                 "ng96_bf16", "ng128_f32_deg66", "box_partial_f32_dg40", "box_partial_bf16_dg40"):
        w = CASES[name]
        t = torch.empty((w.rows, w.d), dtype=torch.float32 if w.dtype == synth.F32
                        else torch.bfloat16, device="cuda")
        args = (w.rows, 1, w.d, w.n_g, w.m, w.n, w.dtype)
        assert grk.grkan_forward_path(t, t, *args) == 1, name
        assert grk.grkan_backward_path(t, t, t, *args) == 1, name
    for name in ("odd_f32_dg10", "odd_bf16_dg6", "deg_3_2", "deg_0_0", "deg_5_0", "deg_2_6",
                 "dg1_f32", "dg1_bf16"):
        w = CASES[name]
        t = torch.empty((w.rows, w.d), dtype=torch.float32, device="cuda")
        assert grk.grkan_backward_path(t, t, t, w.rows, 1, w.d, w.n_g, w.m, w.n, w.dtype) == 0


@pytest.mark.parametrize("name", ["kat_b_ragged", "stress_ng64", "kat_t_ragged", "odd_f32_dg10",
                                  "ng96_bf16", "deg_7_7_bf16", "box_partial_f32_dg40"])
def test_bitwise_determinism(name):
    w, x, dy, a, b = case_data(name)[:5]
    tx, tdy, ta, tb = _dev(w, x, dy, a, b)
    first = grk.backward(tx, tdy, ta, tb, w.n_g)
    for _ in range(10):
        again = grk.backward(tx, tdy, ta, tb, w.n_g)
        for u, v in zip(first, again):
            assert torch.equal(u, v)
    # another stream, other launches in between: same bits
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        grk.forward(tx, ta, tb, w.n_g)
        other = grk.backward(tx, tdy, ta, tb, w.n_g)
    s.synchronize()
    for u, v in zip(first, other):
        assert torch.equal(u, v)


@pytest.mark.parametrize("flags", [0, grk.FLAG_GENERIC], ids=["auto", "generic"])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_identity_is_exact(dtype, flags):
    """a = (0,1,0,0,0,0), b = 0: y = x and dx = dy bit for bit, dB = 0."""
    rows, d, n_g = 300, 768, 8
    g = torch.Generator().manual_seed(0)
    x = torch.randn(rows, d, generator=g).to(dtype).cuda()
    dy = torch.randn(rows, d, generator=g).to(dtype).cuda()
    a = torch.zeros(n_g, 6, device="cuda")
    a[:, 1] = 1
    b = torch.zeros(n_g, 4, device="cuda")
    y = grk.forward(x, a, b, n_g, flags=flags)
    dx, dA, dB = grk.backward(x, dy, a, b, n_g, flags=flags)
    assert torch.equal(y, x) and torch.equal(dx, dy)
    assert torch.all(dB == 0)
    xs = x.double().cpu().view(rows, n_g, d // n_g)
    gs = dy.double().cpu().view(rows, n_g, d // n_g)
    want = torch.stack([(gs * xs ** i).sum(dim=(0, 2)) for i in range(6)], dim=1)
    c2 = torch.stack([((gs * xs ** i) ** 2).sum(dim=(0, 2)) for i in range(6)], dim=1)
    err = (dA.double().cpu() - want).abs()
    assert torch.all(err <= 1e-4 * want.abs() + 2e-6 * c2.sqrt())


@pytest.mark.parametrize("flags", [0, grk.FLAG_GENERIC], ids=["auto", "generic"])
def test_x_zero(flags):
    """x = 0: sign(0) = 0, so dx = dy * a_1 (one float32 rounding) and y = a_0."""
    rows, d, n_g = 64, 384, 4
    x = torch.zeros(rows, d, device="cuda")
    dy = torch.randn(rows, d, device="cuda")
    a = torch.randn(n_g, 6, device="cuda")
    b = torch.randn(n_g, 4, device="cuda")
    y = grk.forward(x, a, b, n_g, flags=flags)
    dx, dA, dB = grk.backward(x, dy, a, b, n_g, flags=flags)
    a_per_col = a.repeat_interleave(d // n_g, dim=0)
    assert torch.equal(y, a_per_col[:, 0].expand(rows, d))
    assert torch.equal(dx, dy * a_per_col[:, 1])
    assert torch.all(dB == 0) and torch.all(dA[:, 1:] == 0)


def test_empty_input_zeroes_gradients():
    x = torch.empty(0, 197, 768, device="cuda")
    a = torch.randn(8, 6, device="cuda")
    b = torch.randn(8, 4, device="cuda")
    y = grk.forward(x, a, b, 8)
    dA = torch.full((8, 6), float("nan"), device="cuda")
    dB = torch.full((8, 4), float("nan"), device="cuda")
    dx, dA, dB = grk.backward(x, x, a, b, 8, dA=dA, dB=dB)
    assert y.numel() == 0 and dx.numel() == 0
    assert torch.all(dA == 0) and torch.all(dB == 0)


@pytest.mark.parametrize("name", ["kat_b_ragged", "kat_t_ragged", "odd_bf16_dg6",
                                  "box_partial_f32_dg40"])
def test_in_place(name):
    w, x, dy, a, b, y_ref, ky, dx_ref, ex, g_ref = case_data(name)
    tx, tdy, ta, tb = _dev(w, x, dy, a, b)
    y = grk.forward(tx.clone(), ta, tb, w.n_g)
    buf = tx.clone()
    grk.forward(buf, ta, tb, w.n_g, out=buf)  # y written over x
    assert torch.equal(buf, y)
    ref = grk.backward(tx, tdy, ta, tb, w.n_g)
    g2 = tdy.clone()
    dx, dA, dB = grk.backward(tx, g2, ta, tb, w.n_g, dx=g2)  # dx written over dy
    assert torch.equal(dx, ref[0]) and torch.equal(dA, ref[1]) and torch.equal(dB, ref[2])


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_unaligned_pointers_take_generic_path(dtype):
    w = synth.workload("kat_b").with_rows(40)
    if dtype == torch.float32:
        w = synth.workload("kat_t").with_rows(40)
    x, dy = w.x(), w.dy()
    a, b = w.coefficients()
    tx, tdy, ta, tb = _dev(w, x, dy, a, b)
    n = tx.numel()
    big = torch.empty(n + 8, dtype=tx.dtype, device="cuda")
    gbig = torch.empty(n + 8, dtype=tx.dtype, device="cuda")
    ux = big[1:n + 1].view(tx.shape)
    ug = gbig[1:n + 1].view(tx.shape)
    ux.copy_(tx)
    ug.copy_(tdy)
    args = (w.rows, 1, w.d, w.n_g, w.m, w.n, w.dtype)
    assert grk.grkan_backward_path(ux, ug, ug, *args) == 0
    dx, dA, dB = grk.backward(ux, ug, ta, tb, w.n_g)
    dx_ref, ex = oracle.backward_elem(x, dy, a, b, w.n_g, extras=True)
    check_dx(to_f64(dx), dx_ref, ex, RTOL[w.dtype])
    check_coef(dA.cpu().numpy(), dB.cpu().numpy(), oracle.coef_grads(x, dy, a, b, w.n_g))


def test_abi_errors_on_gpu():
    x = torch.randn(4, 12, device="cuda")
    a = torch.randn(3, 6, device="cuda")
    b = torch.randn(3, 4, device="cuda")
    with pytest.raises(grk.GrkanError):
        grk.forward(x, a, b, 5)  # 12 % 5 != 0
    ws = torch.empty(4, dtype=torch.uint8, device="cuda")
    with pytest.raises(grk.GrkanError):
        grk.backward(x, x, a, b, 3, workspace=ws)
    assert grk.grkan_device_error()[1] == 0


def test_partials_merge_and_sums64():
    w, x, dy, a, b, y_ref, ky, dx_ref, ex, g_ref = case_data("kat_b_ragged")
    tx, tdy, ta, tb = _dev(w, x, dy, a, b)
    wsb = grk.grkan_backward_workspace_bytes(w.rows, 1, w.d, w.n_g, w.m, w.n, w.dtype)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    dx = torch.empty_like(tx)
    dA = torch.empty(w.n_g, 6, device="cuda")
    dB = torch.empty(w.n_g, 4, device="cuda")
    s64 = torch.empty(w.n_g, 10, dtype=torch.float64, device="cuda")
    args = (w.rows, 1, w.d, w.n_g, w.m, w.n, w.dtype)
    assert grk.grkan_backward_partials(tx, tdy, ta, tb, dx, *args, ws, wsb) == 0
    assert grk.grkan_backward_merge(ws, wsb, dA, dB, s64, *args) == 0
    ref = grk.backward(tx, tdy, ta, tb, w.n_g)
    assert torch.equal(dx, ref[0]) and torch.equal(dA, ref[1]) and torch.equal(dB, ref[2])
    assert torch.equal(s64[:, :6].float(), dA) and torch.equal(s64[:, 6:].float(), dB)


@pytest.mark.parametrize("flags", [0, grk.FLAG_GENERIC], ids=["auto", "generic"])
@pytest.mark.parametrize("name", ["tiny", "kat_t_ragged", "kat_b_ragged", "stress_ng64",
                                  "one_row_bf16", "odd_f32_dg10", "deg_3_2",
                                  "box_partial_f32_dg40", "box_partial_bf16_dg40"])
def test_fused_recompute_parity(name, flags):
    """grkan_forward_backward (y recomputed inside the backward pass): y against
    the oracle, and dx, dA, dB the same bits as the separate backward call."""
    w, x, dy, a, b, y_ref, ky, dx_ref, ex, g_ref = case_data(name)
    tx, tdy, ta, tb = _dev(w, x, dy, a, b)
    y, dx, dA, dB = grk.forward_backward(tx, tdy, ta, tb, w.n_g, flags=flags)
    sdx, sdA, sdB = grk.backward(tx, tdy, ta, tb, w.n_g, flags=flags)
    torch.cuda.synchronize()
    rtol = RTOL[w.dtype]
    check_y(to_f64(y), y_ref, ky, rtol, "%s fused y" % name)
    check_dx(to_f64(dx), dx_ref, ex, rtol, "%s fused dx" % name)
    check_coef(dA.cpu().numpy(), dB.cpu().numpy(), g_ref, what=name)
    assert torch.equal(dx, sdx) and torch.equal(dA, sdA) and torch.equal(dB, sdB)
    # the recomputed y is the forward's, bit for bit
    assert torch.equal(y, grk.forward(tx, ta, tb, w.n_g, flags=flags))
    assert grk.grkan_device_error()[1] == 0


def test_fused_recompute_rejects_overlapping_y():
    w, x, dy, a, b = case_data("kat_t_ragged")[:5]
    tx, tdy, ta, tb = _dev(w, x, dy, a, b)
    dx = torch.empty_like(tx)
    dA = torch.empty(w.n_g, w.m + 1, device="cuda")
    dB = torch.empty(w.n_g, w.n, device="cuda")
    wsb = grk.grkan_backward_workspace_bytes(w.rows, 1, w.d, w.n_g, w.m, w.n, w.dtype)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    for y in (tx, tdy, dx):
        st = grk.grkan_forward_backward(tx, tdy, ta, tb, y, dx, dA, dB, w.rows, 1, w.d, w.n_g,
                                        w.m, w.n, w.dtype, ws, wsb)
        assert st == 7  # GRKAN_ERR_ALIAS


def test_concurrent_calls_on_two_streams():
    """Two backward calls with their own workspaces, enqueued on two streams so
    that the kernels may run at the same time, give the bits of the same calls
    made one after the other (the kernels share no state besides the error
    word)."""
    cases = [case_data("kat_b_ragged"), case_data("stress_ng64")]
    devs = [_dev(c[0], *c[1:5]) for c in cases]
    ref = [grk.backward(tx, tdy, ta, tb, c[0].n_g) for c, (tx, tdy, ta, tb) in zip(cases, devs)]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    for _ in range(3):
        outs = []
        for s, c, (tx, tdy, ta, tb) in zip(streams, cases, devs):
            with torch.cuda.stream(s):
                outs.append(grk.backward(tx, tdy, ta, tb, c[0].n_g))
        for s in streams:
            s.synchronize()
        for got, want in zip(outs, ref):
            for u, v in zip(got, want):
                assert torch.equal(u, v)
    assert grk.grkan_device_error()[1] == 0

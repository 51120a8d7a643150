"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError on
a mismatch. ``test_oracle_pins.py`` runs them on the committed oracle;
``test_oracle_mutants.py`` plants plausible mistakes in a copy of the oracle's
source and checks that every planted mistake trips at least one pin.

What pins what:
  y      identity closed form, b = 0 polynomial (exact rationals), exact dyadic
         brute force, x = 0, bf16 widening, fp64 autograd witness, numpy's
         polyval for P and Q with the bound |y| <= |P| (D >= 1)
  dx     identity closed form, x = 0 (dx = dy a_1 under sign(0) = 0), central
         differences of the forward (Richardson), exact dual-number brute force,
         autograd witness
  dA     identity closed form (sum dy x^i), central differences of
         L = sum dy y (exact: L is linear in a), brute force, linearity in dy
  dB     b = 0 gives 0, central differences (Richardson), brute force,
         autograd witness, group relabelling
  error scales (which widen every y / dx comparison and pick the elements
  whose sign of Q is undecidable in float32):
         kappa_q  = max over the 2^n sign patterns of b of |Q| (brute force)
         kappa_y  = the largest first-order change of y under relative
                    coefficient perturbations of size one, over every sign
                    pattern (exact dual numbers); closed form (P + yQ) / D at
                    nonnegative x, a, b (exact rationals)
         kappa_dx = closed form at nonnegative x, a, b, dy (exact rationals);
                    invariant under a -> -a, b -> -b, dy -> -dy; bounds the
                    first-order change of dx under relative coefficient
                    perturbations (with the |dx| kappa_q / D part that the
                    relative tolerance term covers)
         c2       = closed forms at nonnegative inputs with b != 0
"""
from fractions import Fraction

import numpy as np

import exact


def _close(got, want, rtol, atol=0.0, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    err = np.abs(got - want)
    lim = rtol * np.abs(want) + atol
    bad = err > lim
    assert not bad.any(), "%s: %d mismatches, worst err %.3e at want %.6e" % (
        what, int(bad.sum()), float(err.max()), float(want.flat[int(np.argmax(err))]))


def _rand_case(rng, rows, d, n_g, m, n, xs=1.0, coef=0.5, dys=1.0):
    x = (rng.standard_normal((rows, d)) * xs).astype(np.float32)
    dy = (rng.standard_normal((rows, d)) * dys).astype(np.float32)
    a = rng.uniform(-coef, coef, (n_g, m + 1)).astype(np.float32)
    b = rng.uniform(-coef, coef, (n_g, n)).astype(np.float32)
    return x, dy, a, b


def _dyadic(rng, shape, den, kmax):
    return (rng.integers(-kmax, kmax + 1, shape) / den).astype(np.float32)


# --- y ----------------------------------------------------------------------

def pin_identity(orc):
    """a = (0,1,0,...), b = 0: y = x, dx = dy, dA_i = sum dy x^i, dB = 0."""
    rng = np.random.default_rng(1)
    rows, d, n_g, m, n = 5, 12, 3, 5, 4
    x = _dyadic(rng, (rows, d), 8, 24)
    dy = _dyadic(rng, (rows, d), 8, 24)
    a = np.zeros((n_g, m + 1), np.float32)
    a[:, 1] = 1.0
    b = np.zeros((n_g, n), np.float32)
    y = orc.forward(x, a, b, n_g)
    assert np.array_equal(y, x.astype(np.float64)), "identity: y != x"
    dx = orc.backward_elem(x, dy, a, b, n_g)
    assert np.array_equal(dx, dy.astype(np.float64)), "identity: dx != dy"
    g = orc.coef_grads(x, dy, a, b, n_g)
    assert np.all(g["dB"] == 0.0), "identity: dB != 0"
    dg = d // n_g
    for gi in range(n_g):
        xs = [Fraction(float(v)) for v in x[:, gi * dg:(gi + 1) * dg].ravel()]
        gs = [Fraction(float(v)) for v in dy[:, gi * dg:(gi + 1) * dg].ravel()]
        for i in range(m + 1):
            want = float(sum(gv * xv ** i for xv, gv in zip(xs, gs)))
            _close(g["dA"][gi, i], want, 1e-13, 1e-13, "identity dA")


def pin_polynomial_b0(orc):
    """b = 0: y is the plain polynomial P(x), compared with exact rationals."""
    rng = np.random.default_rng(2)
    rows, d, n_g, m, n = 4, 16, 4, 7, 3
    x = rng.uniform(-3, 3, (rows, d)).astype(np.float32)
    a = rng.uniform(-1, 1, (n_g, m + 1)).astype(np.float32)
    b = np.zeros((n_g, n), np.float32)
    y, ky = orc.forward(x, a, b, n_g, kappa=True)
    dg = d // n_g
    for r in range(rows):
        for c in range(d):
            xv = Fraction(float(x[r, c]))
            want = sum(Fraction(float(a[c // dg, i])) * xv ** i for i in range(m + 1))
            assert abs(Fraction(float(y[r, c])) - want) <= Fraction(1e-14) * Fraction(
                float(ky[r, c])), "b=0 polynomial mismatch at %d,%d" % (r, c)


def pin_dyadic_exact(orc):
    """Exact brute force (dual numbers over rationals) on dyadic inputs."""
    rng = np.random.default_rng(3)
    for (m, n, n_g, d) in [(5, 4, 2, 8), (3, 2, 1, 6), (0, 0, 2, 4), (1, 3, 3, 6), (2, 0, 1, 3),
                           (6, 5, 2, 4)]:
        rows = 3
        x = _dyadic(rng, (rows, d), 4, 12)
        x[0, 0] = 0.0  # the kink: Q(0) = 0
        dy = _dyadic(rng, (rows, d), 4, 12)
        a = _dyadic(rng, (n_g, m + 1), 8, 8)
        b = _dyadic(rng, (n_g, n), 8, 8)
        ey, edx, edA, edB = exact.forward_backward(x.tolist(), dy.tolist(), a.tolist(),
                                                   b.tolist(), n_g)
        y = orc.forward(x, a, b, n_g)
        dx = orc.backward_elem(x, dy, a, b, n_g)
        g = orc.coef_grads(x, dy, a, b, n_g)
        fy = np.array([[float(v) for v in row] for row in ey])
        fdx = np.array([[float(v) for v in row] for row in edx])
        _close(y, fy, 1e-14, 1e-300, "dyadic y (m=%d n=%d)" % (m, n))
        _close(dx, fdx, 1e-13, 1e-13 * np.abs(fdx).max(), "dyadic dx (m=%d n=%d)" % (m, n))
        sabs_a = g["sabs_a"]
        sabs_b = g["sabs_b"]
        _close(g["dA"], np.array([[float(v) for v in r] for r in edA]).reshape(n_g, m + 1), 0,
               1e-13 * (sabs_a + 1e-300), "dyadic dA")
        if n:
            _close(g["dB"], np.array([[float(v) for v in r] for r in edB]).reshape(n_g, n), 0,
                   1e-13 * (sabs_b + 1e-300), "dyadic dB")


def pin_x_zero(orc):
    """x = 0: Q = 0 so D = 1 and sign(0) = 0, hence y = a_0 and dx = dy a_1."""
    rng = np.random.default_rng(4)
    n_g, m, n, d = 4, 5, 4, 8
    x = np.zeros((2, d), np.float32)
    dy = rng.standard_normal((2, d)).astype(np.float32)
    a = rng.uniform(-1, 1, (n_g, m + 1)).astype(np.float32)
    b = rng.uniform(-1, 1, (n_g, n)).astype(np.float32)
    y = orc.forward(x, a, b, n_g)
    dx = orc.backward_elem(x, dy, a, b, n_g)
    dg = d // n_g
    for c in range(d):
        g = c // dg
        assert np.all(y[:, c] == np.float64(a[g, 0])), "x=0: y != a0"
        want = dy[:, c].astype(np.float64) * np.float64(a[g, 1])
        assert np.all(dx[:, c] == want), "x=0: dx != dy*a1"
    gr = orc.coef_grads(x, dy, a, b, n_g)
    assert np.all(gr["dB"] == 0.0), "x=0: dB != 0"
    assert np.all(gr["dA"][:, 1:] == 0.0), "x=0: dA_i (i>0) != 0"


def pin_bf16_widening(orc):
    """bf16 inputs equal to float32 inputs with the same values give the same results."""
    rng = np.random.default_rng(5)
    rows, d, n_g, m, n = 6, 16, 2, 5, 4
    xf, dyf, a, b = _rand_case(rng, rows, d, n_g, m, n)
    xb = (xf.view(np.uint32) >> 16).astype(np.uint16)
    dyb = (dyf.view(np.uint32) >> 16).astype(np.uint16)
    xf = (xb.astype(np.uint32) << 16).view(np.float32)
    dyf = (dyb.astype(np.uint32) << 16).view(np.float32)
    assert np.array_equal(orc.forward(xb, a, b, n_g), orc.forward(xf, a, b, n_g)), "bf16 y"
    assert np.array_equal(orc.backward_elem(xb, dyb, a, b, n_g),
                          orc.backward_elem(xf, dyf, a, b, n_g)), "bf16 dx"
    gb = orc.coef_grads(xb, dyb, a, b, n_g)
    gf = orc.coef_grads(xf, dyf, a, b, n_g)
    assert np.array_equal(gb["dA"], gf["dA"]) and np.array_equal(gb["dB"], gf["dB"]), "bf16 dA/dB"


# --- derivatives ------------------------------------------------------------

def _richardson(f, h):
    d1 = (f(h) - f(-h)) / (2 * h)
    d2 = (f(h / 2) - f(-h / 2)) / h
    return (4 * d2 - d1) / 3


def pin_fd_dx(orc):
    """dx against Richardson-extrapolated central differences of the forward."""
    rng = np.random.default_rng(6)
    rows, d, n_g, m, n = 8, 16, 4, 5, 4
    h = 2.0 ** -8
    x = (rng.integers(-2048, 2049, (rows, d)) / 1024.0).astype(np.float32)
    dy = rng.standard_normal((rows, d)).astype(np.float32)
    a = rng.uniform(-0.5, 0.5, (n_g, m + 1)).astype(np.float32)
    b = rng.uniform(-0.5, 0.5, (n_g, n)).astype(np.float32)
    dx, ex = orc.backward_elem(x, dy, a, b, n_g, extras=True)

    def yat(off):
        return orc.forward((x.astype(np.float64) + off).astype(np.float32), a, b, n_g)

    fd = dy.astype(np.float64) * _richardson(yat, h)
    # exclude elements where Q changes sign inside [x - h, x + h]
    qs = [orc.backward_elem((x.astype(np.float64) + o).astype(np.float32), dy, a, b, n_g,
                            extras=True)[1]["q"] for o in (-h, h)]
    smooth = (np.sign(qs[0]) == np.sign(ex["q"])) & (np.sign(qs[1]) == np.sign(ex["q"])) & (
        ex["q"] != 0)
    assert smooth.mean() > 0.8
    _close(dx[smooth], fd[smooth], 1e-6, 1e-7 * (1 + np.abs(dy[smooth])), "fd dx")


def pin_fd_dA(orc):
    """dA against central differences of L = sum dy*y (L is linear in a: exact)."""
    rng = np.random.default_rng(7)
    rows, d, n_g, m, n = 16, 12, 3, 5, 4
    x, dy, a, b = _rand_case(rng, rows, d, n_g, m, n)
    a = (rng.integers(-512, 513, a.shape) / 1024.0).astype(np.float32)  # a +- h stays exact
    g = orc.coef_grads(x, dy, a, b, n_g)
    h = 2.0 ** -6
    for gi in range(n_g):
        for i in range(m + 1):
            def L(off):
                aa = a.astype(np.float64).copy()
                aa[gi, i] += off
                return float(np.sum(dy.astype(np.float64) * orc.forward(x, aa.astype(np.float32),
                                                                         b, n_g)))
            fd = (L(h) - L(-h)) / (2 * h)
            _close(g["dA"][gi, i], fd, 1e-9, 1e-12, "fd dA[%d,%d]" % (gi, i))


def pin_fd_dB(orc):
    """dB against Richardson central differences of L = sum dy*y. The data keep
    sign(Q) = sign(x) under the perturbation, so L is smooth in b."""
    rng = np.random.default_rng(8)
    rows, d, n_g, m, n = 16, 12, 3, 5, 4
    x = (rng.integers(-2048, 2049, (rows, d)) / 1024.0).astype(np.float32)
    dy = rng.standard_normal((rows, d)).astype(np.float32)
    a = rng.uniform(-0.5, 0.5, (n_g, m + 1)).astype(np.float32)
    # dyadic b (multiples of 2^-12) so that b +- h and b +- h/2 stay exact in float32
    b = (rng.integers(-204, 205, (n_g, n)) / 4096.0).astype(np.float32)
    b[:, 0] = (rng.choice([-1.0, 1.0], n_g) * (1.0 + rng.integers(0, 819, n_g) / 4096.0)).astype(
        np.float32)
    g = orc.coef_grads(x, dy, a, b, n_g)
    h = 2.0 ** -10
    for gi in range(n_g):
        for j in range(n):
            def L(off):
                bb = b.astype(np.float64).copy()
                bb[gi, j] += off
                return float(np.sum(dy.astype(np.float64) * orc.forward(x, a,
                                                                         bb.astype(np.float32),
                                                                         n_g)))
            fd = _richardson(L, h)
            _close(g["dB"][gi, j], fd, 1e-7, 1e-8 * g["sabs_b"][gi, j], "fd dB[%d,%d]" % (gi, j))


def pin_autograd(orc):
    """An fp64 torch autograd witness on random data with both signs of Q."""
    import torch
    rng = np.random.default_rng(9)
    rows, d, n_g, m, n = 10, 24, 4, 5, 4
    x, dy, a, b = _rand_case(rng, rows, d, n_g, m, n, coef=0.7)
    x[0, :3] = 0.0
    dg = d // n_g
    tx = torch.tensor(x, dtype=torch.float64, requires_grad=True)
    ta = torch.tensor(a, dtype=torch.float64, requires_grad=True)
    tb = torch.tensor(b, dtype=torch.float64, requires_grad=True)
    ga = ta.repeat_interleave(dg, dim=0)  # (d, m+1): row c holds group c // dg
    gb = tb.repeat_interleave(dg, dim=0)
    P = ga[:, m].expand(rows, d)
    for i in range(m - 1, -1, -1):
        P = P * tx + ga[:, i]
    Q = torch.zeros_like(tx)
    for j in range(n, 0, -1):
        Q = (Q + gb[:, j - 1]) * tx
    y = P / (1 + Q.abs())
    L = (torch.tensor(dy, dtype=torch.float64) * y).sum()
    L.backward()
    _close(orc.forward(x, a, b, n_g), y.detach().numpy(), 1e-13, 1e-15, "autograd y")
    _close(orc.backward_elem(x, dy, a, b, n_g), tx.grad.numpy(), 1e-12, 1e-14, "autograd dx")
    g = orc.coef_grads(x, dy, a, b, n_g)
    _close(g["dA"], ta.grad.numpy(), 0, 1e-12 * g["sabs_a"], "autograd dA")
    _close(g["dB"], tb.grad.numpy(), 0, 1e-12 * g["sabs_b"], "autograd dB")


# --- structure --------------------------------------------------------------

def pin_linearity(orc):
    """Scaling dy by 2^k scales dx, dA, dB by exactly 2^k."""
    rng = np.random.default_rng(10)
    x, dy, a, b = _rand_case(rng, 8, 16, 4, 5, 4)
    g1 = orc.coef_grads(x, dy, a, b, 4)
    g4 = orc.coef_grads(x, dy * np.float32(4), a, b, 4)
    assert np.array_equal(g4["dA"], 4 * g1["dA"]) and np.array_equal(g4["dB"], 4 * g1["dB"]), \
        "linearity dA/dB"
    assert np.array_equal(orc.backward_elem(x, dy * np.float32(4), a, b, 4),
                          4 * orc.backward_elem(x, dy, a, b, 4)), "linearity dx"


def pin_group_relabel(orc):
    """Permuting the channel groups together with their coefficients permutes
    the outputs the same way."""
    rng = np.random.default_rng(11)
    rows, d, n_g, m, n = 6, 20, 5, 5, 4
    dg = d // n_g
    x, dy, a, b = _rand_case(rng, rows, d, n_g, m, n)
    perm = rng.permutation(n_g)
    cols = np.concatenate([np.arange(p * dg, (p + 1) * dg) for p in perm])
    xp, dyp, ap, bp = x[:, cols], dy[:, cols], a[perm], b[perm]
    assert np.array_equal(orc.forward(xp, ap, bp, n_g), orc.forward(x, a, b, n_g)[:, cols])
    assert np.array_equal(orc.backward_elem(xp, dyp, ap, bp, n_g),
                          orc.backward_elem(x, dy, a, b, n_g)[:, cols])
    g = orc.coef_grads(x, dy, a, b, n_g)
    gp = orc.coef_grads(xp, dyp, ap, bp, n_g)
    _close(gp["dA"], g["dA"][perm], 1e-14, 1e-300, "relabel dA")
    _close(gp["dB"], g["dB"][perm], 1e-14, 1e-300, "relabel dB")


def pin_thread_invariance(orc):
    """Reductions run in fixed chunks: the thread count cannot change a bit."""
    rng = np.random.default_rng(12)
    x, dy, a, b = _rand_case(rng, 300, 32, 4, 5, 4)
    g1 = orc.coef_grads(x, dy, a, b, 4, nthreads=1)
    g3 = orc.coef_grads(x, dy, a, b, 4, nthreads=3)
    for k in ("dA", "dB", "sabs_a", "sabs_b"):
        assert np.array_equal(g1[k], g3[k]), k


def pin_sampled_and_extras(orc):
    """Per-index evaluation equals the full evaluation; the extras are
    consistent: dx_sign at s = sign(Q) is dx, and for a, b >= 0, x >= 0 the
    error scales equal the values."""
    rng = np.random.default_rng(13)
    rows, d, n_g, m, n = 7, 12, 3, 5, 4
    x, dy, a, b = _rand_case(rng, rows, d, n_g, m, n)
    idx = rng.choice(rows * d, 20, replace=False)
    assert np.array_equal(orc.forward(x, a, b, n_g, idx=idx), orc.forward(x, a, b, n_g).ravel()[idx])
    dx, ex = orc.backward_elem(x, dy, a, b, n_g, extras=True)
    dxi = orc.backward_elem(x, dy, a, b, n_g, idx=idx)
    assert np.array_equal(dxi, dx.ravel()[idx])
    s = np.sign(ex["q"]).astype(int) + 1
    pick = np.take_along_axis(ex["dx_sign"], s[..., None], axis=-1)[..., 0]
    assert np.array_equal(pick, dx)
    # with b = 0 and a, x >= 0 the error scale of y is y itself
    y, ky = orc.forward(np.abs(x), np.abs(a), np.zeros_like(b), n_g, kappa=True)
    _close(ky, y, 1e-14, 0, "kappa_y positive case")
    assert np.all(ex["kappa_q"] >= np.abs(ex["q"]) * (1 - 1e-12))


def pin_ambiguity(orc):
    """Elements with Q exactly 0 away from x = 0 are counted as sign-ambiguous and
    the dB allowance there is 2 |dy y x^j / D| (D = 1 at a root)."""
    n_g, m, n = 1, 2, 2
    # Q(x) = x/2 - x^2/4 vanishes at x = 2
    a = np.array([[0.5, 0.25, 0.125]], np.float32)
    b = np.array([[0.5, -0.25]], np.float32)
    x = np.array([[2.0, 1.0, -1.0, 0.0]], np.float32)
    dy = np.array([[0.5, 0.5, 0.5, 0.5]], np.float32)
    g = orc.coef_grads(x, dy, a, b, n_g)
    assert g["amb_count"] == 1, g["amb_count"]
    y2 = 0.5 + 0.25 * 2 + 0.125 * 4
    want = np.array([2 * 0.5 * y2 * 2.0, 2 * 0.5 * y2 * 4.0])
    _close(g["amb_b"][0], want, 1e-15, 0, "ambiguity allowance")


def pin_noise_scales(orc):
    """c2 (the conditioned sums of squares used as the float32 noise scale of
    dA / dB): with b = 0 the denominator is exactly 1 and Q is exactly 0, so
    c2_a = sum (dy x^i)^2 and c2_b = sum (|dy x^j| sum_i |a_i||x|^i)^2; in general
    c2 >= sabs^2 / n_terms (Cauchy-Schwarz, the weights being >= 1)."""
    rng = np.random.default_rng(14)
    rows, d, n_g, m, n = 9, 12, 3, 5, 4
    x, dy, a, b = _rand_case(rng, rows, d, n_g, m, n)
    dg = d // n_g
    g0 = orc.coef_grads(x, dy, a, np.zeros_like(b), n_g)
    xs = x.astype(np.float64).reshape(rows, n_g, dg)
    gs = dy.astype(np.float64).reshape(rows, n_g, dg)
    kp = sum(np.abs(a.astype(np.float64))[None, :, i, None] * np.abs(xs) ** i for i in range(m + 1))
    for i in range(m + 1):
        _close(g0["c2_a"][:, i], ((gs * xs ** i) ** 2).sum(axis=(0, 2)), 1e-13, 0, "c2_a b=0")
    for j in range(1, n + 1):
        _close(g0["c2_b"][:, j - 1], ((np.abs(gs * xs ** j) * kp) ** 2).sum(axis=(0, 2)), 1e-13,
               0, "c2_b b=0")
    g = orc.coef_grads(x, dy, a, b, n_g)
    nt = rows * dg
    assert np.all(g["c2_a"] >= g["sabs_a"] ** 2 / nt * (1 - 1e-12))
    assert np.all(g["c2_b"] >= g["sabs_b"] ** 2 / nt * (1 - 1e-12))


def pin_library_polyval(orc):
    """y against numpy's own polynomial evaluator for P and Q (b != 0, several
    degrees, values of x up to 4), and the bound that D = 1 + |Q| >= 1 gives:
    |y| <= |P(x)|, with equality exactly where Q = 0."""
    from numpy.polynomial import polynomial as npp
    rng = np.random.default_rng(21)
    for (m, n) in ((5, 4), (3, 3), (2, 6), (8, 1)):
        rows, d, n_g = 7, 12, 3
        x, dy, a, b = _rand_case(rng, rows, d, n_g, m, n, xs=1.5)
        x[0, :3] = 0.0
        y = orc.forward(x, a, b, n_g)
        dg = d // n_g
        for g in range(n_g):
            xs = x[:, g * dg:(g + 1) * dg].astype(np.float64)
            P = npp.polyval(xs, a[g].astype(np.float64))
            Q = npp.polyval(xs, np.concatenate([[0.0], b[g].astype(np.float64)]))
            want = P / (1.0 + np.abs(Q))
            _close(y[:, g * dg:(g + 1) * dg], want, 1e-13, 1e-300, "y vs polyval (%d,%d)" % (m, n))
            yg = np.abs(y[:, g * dg:(g + 1) * dg])
            assert np.all(yg <= np.abs(P) * (1 + 1e-15) + 1e-300), "|y| <= |P|"
            eq = Q == 0.0
            assert np.all(yg[eq] == np.abs(P[eq])), "|y| = |P| where Q = 0"


# --- error scales -------------------------------------------------------------
#
# kappa_y, kappa_dx and kappa_q widen the y / dx tolerances and decide which
# elements count as sign-ambiguous, so an inflated scale would silently loosen
# every parity check. They are pinned here to what they mean, not to their
# formulas.

def _fpoly(coefs, x):
    """sum_k coefs[k] x^k over Fractions (plain power sum)."""
    return sum((c * x ** k for k, c in enumerate(coefs)), Fraction(0))


def _nonneg_case(rng, rows, d, n_g, m, n):
    x = _dyadic(rng, (rows, d), 8, 24)
    x = np.abs(x)
    x[0, 0] = 0.0
    dy = np.abs(_dyadic(rng, (rows, d), 8, 16))
    a = np.abs(_dyadic(rng, (n_g, m + 1), 8, 8))
    b = np.abs(_dyadic(rng, (n_g, n), 8, 8))
    b[:, 0] = np.maximum(b[:, 0], 0.125)  # Q > 0 wherever x > 0
    return x, dy, a, b


def _pqs(xv, ga, gb):
    """Exact P, P', Q, Q' at a Fraction x for group coefficients (floats)."""
    fa = [Fraction(float(v)) for v in ga]
    fb = [Fraction(0)] + [Fraction(float(v)) for v in gb]  # Q has no constant term
    P = _fpoly(fa, xv)
    Q = _fpoly(fb, xv)
    dP = _fpoly([k * c for k, c in enumerate(fa)][1:], xv)
    dQ = _fpoly([k * c for k, c in enumerate(fb)][1:], xv)
    return P, dP, Q, dQ


def pin_kappa_q_brute_force(orc):
    """kappa_q = sum_j |b_j||x|^j is the largest |Q(x)| over the 2^n sign
    patterns of (b_1..b_n) (numpy's polynomial evaluator), the scale that
    float32 rounding of Q is measured against."""
    from numpy.polynomial import polynomial as npp
    import itertools
    rng = np.random.default_rng(31)
    for (m, n) in ((5, 4), (2, 6), (3, 1)):
        rows, d, n_g = 5, 8, 2
        x, dy, a, b = _rand_case(rng, rows, d, n_g, m, n, xs=1.5, coef=0.8)
        x[0, 0] = 0.0
        _, ex = orc.backward_elem(x, dy, a, b, n_g, extras=True)
        dg = d // n_g
        for g in range(n_g):
            xs = x[:, g * dg:(g + 1) * dg].astype(np.float64)
            best = np.zeros_like(xs)
            for signs in itertools.product((-1.0, 1.0), repeat=n):
                cb = np.concatenate([[0.0], np.abs(b[g].astype(np.float64)) * signs])
                best = np.maximum(best, np.abs(npp.polyval(xs, cb)))
            _close(ex["kappa_q"][:, g * dg:(g + 1) * dg], best, 1e-14, 1e-300,
                   "kappa_q (m=%d n=%d)" % (m, n))


def pin_kappa_y_nonneg_closed_form(orc):
    """With x, a, b >= 0 every term is nonnegative, so the absolute-value
    evaluation is the evaluation itself: kappa_y = (P + y Q) / D
    = P (1 + 2Q) / (1 + Q)^2, in exact rationals."""
    rng = np.random.default_rng(32)
    for (m, n, n_g, d) in ((5, 4, 2, 8), (3, 3, 1, 4), (7, 2, 2, 4)):
        x, dy, a, b = _nonneg_case(rng, 3, d, n_g, m, n)
        _, ky = orc.forward(x, a, b, n_g, kappa=True)
        dg = d // n_g
        for r in range(x.shape[0]):
            for c in range(d):
                P, _, Q, _ = _pqs(Fraction(float(x[r, c])), a[c // dg], b[c // dg])
                want = P * (1 + 2 * Q) / (1 + Q) ** 2
                assert abs(Fraction(float(ky[r, c])) - want) <= Fraction(1, 10 ** 13) * want, \
                    "kappa_y closed form at (%d,%d), m=%d n=%d" % (r, c, m, n)


def pin_kappa_y_max_sensitivity(orc):
    """kappa_y is the largest first-order change of y when every coefficient
    takes a relative perturbation of size one (a_i -> a_i (1 + t s_i),
    b_j -> b_j (1 + t r_j), s, r = +-1): brute force over all 2^(m+1+n) sign
    patterns with exact dual numbers, at points with Q != 0 and both signs of
    x, y and the coefficients."""
    import itertools
    rng = np.random.default_rng(33)
    for (m, n, cnt) in ((3, 2, 10), (5, 4, 4)):
        x = _dyadic(rng, (cnt,), 8, 24)
        x[x == 0] = 0.625
        a = _dyadic(rng, (m + 1,), 8, 8)
        b = _dyadic(rng, (n,), 8, 8)
        b[0] = 0.375 if b[0] == 0 else b[0]
        _, ky = orc.forward(x.reshape(1, -1), a.reshape(1, -1), b.reshape(1, -1), 1, kappa=True)
        fa = [Fraction(float(v)) for v in a]
        fb = [Fraction(float(v)) for v in b]
        seen_neg_y = False
        for e in range(cnt):
            xv = exact.Dual(Fraction(float(x[e])))
            if exact.activation(xv, fa, fb).v < 0:
                seen_neg_y = True
            best = Fraction(0)
            for signs in itertools.product((-1, 1), repeat=m + 1 + n):
                aa = [exact.Dual(v, signs[i] * v) for i, v in enumerate(fa)]
                bb = [exact.Dual(v, signs[m + 1 + j] * v) for j, v in enumerate(fb)]
                out = exact.activation(xv, aa, bb)
                best = max(best, abs(out.d))
            assert abs(Fraction(float(ky[0, e])) - best) <= Fraction(1, 10 ** 13) * best, \
                "kappa_y vs max sensitivity at x=%g (m=%d n=%d): %r vs %r" % (
                    float(x[e]), m, n, float(ky[0, e]), float(best))
        assert seen_neg_y


def pin_kappa_dx_nonneg_closed_form(orc):
    """With x, a, b, dy >= 0 (so Q >= 0, s = 1 where x > 0): kappa_dx
    = dy (P' + y Q' + kappa_y Q') / D = dy (P' + Q' P (2 + 3Q) / (1 + Q)^2) / (1 + Q),
    in exact rationals."""
    rng = np.random.default_rng(34)
    for (m, n, n_g, d) in ((5, 4, 2, 8), (3, 3, 1, 4), (7, 2, 2, 4)):
        x, dy, a, b = _nonneg_case(rng, 3, d, n_g, m, n)
        _, ex = orc.backward_elem(x, dy, a, b, n_g, extras=True)
        dg = d // n_g
        for r in range(x.shape[0]):
            for c in range(d):
                P, dP, Q, dQ = _pqs(Fraction(float(x[r, c])), a[c // dg], b[c // dg])
                g = Fraction(float(dy[r, c]))
                want = g * (dP + dQ * P * (2 + 3 * Q) / (1 + Q) ** 2) / (1 + Q)
                got = Fraction(float(ex["kappa_dx"][r, c]))
                assert abs(got - want) <= Fraction(1, 10 ** 13) * want, \
                    "kappa_dx closed form at (%d,%d), m=%d n=%d: %r vs %r" % (
                        r, c, m, n, float(got), float(want))


def pin_kappa_dx_sign_invariance(orc):
    """kappa_dx is a sum of absolute values: negating every a_i (which negates
    P, P', y), every b_j (which negates Q, Q') or dy leaves it unchanged bit for
    bit."""
    rng = np.random.default_rng(35)
    rows, d, n_g, m, n = 6, 12, 3, 5, 4
    x, dy, a, b = _rand_case(rng, rows, d, n_g, m, n, xs=1.5)
    x[0, :2] = 0.0
    base = orc.backward_elem(x, dy, a, b, n_g, extras=True)[1]
    for what, args in (("-a", (x, dy, -a, b)), ("-b", (x, dy, a, -b)), ("-dy", (x, -dy, a, b))):
        ex = orc.backward_elem(*args, n_g, extras=True)[1]
        assert np.array_equal(ex["kappa_dx"], base["kappa_dx"]), "kappa_dx changes under " + what
        assert np.array_equal(ex["kappa_q"], base["kappa_q"]), "kappa_q changes under " + what
    _, ky0 = orc.forward(x, a, b, n_g, kappa=True)
    for aa, bb in ((-a, b), (a, -b)):
        assert np.array_equal(orc.forward(x, aa, bb, n_g, kappa=True)[1], ky0), "kappa_y sign"


def pin_kappa_dx_bounds_perturbation(orc):
    """Relative coefficient perturbations of size eta change dx by at most
    eta (kappa_dx + |dx| kappa_q / D) to first order (the second part is the
    effect of D's error on the 1/D factor, covered by the relative part of the
    tolerance), and over the elements the largest change seen under random
    sign patterns reaches that bound (an inflated kappa_dx fails there)."""
    rng = np.random.default_rng(36)
    rows, d, n_g, m, n = 6, 16, 2, 5, 4
    x, dy, a, b = _rand_case(rng, rows, d, n_g, m, n, xs=1.5, coef=0.7)
    dx, ex = orc.backward_elem(x, dy, a, b, n_g, extras=True)
    q = ex["q"]
    Dv = 1.0 + np.abs(q)
    bound = ex["kappa_dx"] + np.abs(dx) * ex["kappa_q"] / Dv
    eta = 2.0 ** -26
    a64, b64 = a.astype(np.float64), b.astype(np.float64)
    reach = np.zeros_like(dx)
    for _ in range(48):
        sa = rng.choice([-1.0, 1.0], a.shape)
        sb = rng.choice([-1.0, 1.0], b.shape)
        # the oracle widens float32 coefficients exactly; feed it the perturbed
        # values through its double-precision arrays
        o_p = _backward_f64(orc, x, dy, a64 * (1 + eta * sa), b64 * (1 + eta * sb), n_g)
        o_m = _backward_f64(orc, x, dy, a64 * (1 - eta * sa), b64 * (1 - eta * sb), n_g)
        change = np.abs(o_p - o_m) / (2 * eta)
        smooth = np.abs(q) > 1e-6
        assert np.all(change[smooth] <= bound[smooth] * (1 + 1e-5) + 1e-12), "dx moves beyond kappa"
        reach = np.maximum(reach, change)
    # No element-wise lower bound exists (one coefficient moves P' and y in
    # ways that can cancel), but over the elements the bound is reached and
    # typically nearly so: an inflated kappa_dx fails both.
    sm = np.abs(q) > 1e-6
    assert np.max(reach[sm] / bound[sm]) >= 0.95, "no element reaches the bound"
    assert np.median(reach[sm] / ex["kappa_dx"][sm]) >= 0.6, "kappa_dx far above dx's sensitivity"


def _backward_f64(orc, x, dy, a64, b64, n_g):
    """dx with float64 coefficients (bypassing the float32 widening)."""
    rows, d = x.shape
    m = a64.shape[1] - 1
    n = b64.shape[1]
    out = np.empty(rows * d, np.float64)
    a64 = np.ascontiguousarray(a64)
    b64 = np.ascontiguousarray(b64)
    rc = orc.lib.gro_backward_elem(x.ctypes.data, np.ascontiguousarray(dy).ctypes.data, 0, rows,
                                   d, n_g, m, n, a64.ctypes.data, b64.ctypes.data, None,
                                   rows * d, out.ctypes.data, None, None, None, None)
    assert rc == 0
    return out.reshape(rows, d)


def pin_noise_scales_nonneg(orc):
    """c2 with b != 0, at x, a, b, dy >= 0 (Q >= 0, s = 1 where x > 0): the dA
    weight is |t x^i| (1 + Q/D) = dy x^i (1 + 2Q) / (1 + Q)^2 and the dB weight
    |t y x^j| + |dy x^j / D^2| (P + 2 P Q / D) = 2 dy x^j P (1 + 2Q) / (1 + Q)^3,
    summed in squares over the group (exact rationals)."""
    rng = np.random.default_rng(37)
    rows, d, n_g, m, n = 4, 8, 2, 5, 4
    x, dy, a, b = _nonneg_case(rng, rows, d, n_g, m, n)
    x[x == 0] = 0.25  # s = 1 everywhere
    g = orc.coef_grads(x, dy, a, b, n_g)
    dg = d // n_g
    for gi in range(n_g):
        wa = [Fraction(0)] * (m + 1)
        wb = [Fraction(0)] * n
        for r in range(rows):
            for c in range(gi * dg, (gi + 1) * dg):
                xv = Fraction(float(x[r, c]))
                gv = Fraction(float(dy[r, c]))
                P, _, Q, _ = _pqs(xv, a[gi], b[gi])
                for i in range(m + 1):
                    wa[i] += (gv * xv ** i * (1 + 2 * Q) / (1 + Q) ** 2) ** 2
                for j in range(1, n + 1):
                    wb[j - 1] += (2 * gv * xv ** j * P * (1 + 2 * Q) / (1 + Q) ** 3) ** 2
        _close(g["c2_a"][gi], [float(v) for v in wa], 1e-13, 0, "c2_a nonneg")
        _close(g["c2_b"][gi], [float(v) for v in wb], 1e-13, 0, "c2_b nonneg")


ALL_PINS = [pin_identity, pin_polynomial_b0, pin_dyadic_exact, pin_x_zero, pin_bf16_widening,
            pin_fd_dx, pin_fd_dA, pin_fd_dB, pin_autograd, pin_linearity, pin_group_relabel,
            pin_thread_invariance, pin_sampled_and_extras, pin_ambiguity, pin_noise_scales,
            pin_library_polyval, pin_kappa_q_brute_force, pin_kappa_y_nonneg_closed_form,
            pin_kappa_y_max_sensitivity, pin_kappa_dx_nonneg_closed_form,
            pin_kappa_dx_sign_invariance, pin_kappa_dx_bounds_perturbation,
            pin_noise_scales_nonneg]

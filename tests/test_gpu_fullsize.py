"""Full-size workloads (KAT-T/S/B-shaped activations and the accumulation /
group stress sweep), in the launch configuration the benchmark times: y and dx
on sampled elements against the oracle evaluated one by one, dA and dB against
the oracle's reduction over every element, and bitwise determinism."""
import numpy as np
import pytest
import torch

import group_rational_kan_b200 as grk
import oracle
import synth
from parity import RTOL, check_dx, check_y, coef_report, to_f64, to_torch

pytestmark = pytest.mark.gpu

FULL = [("kat_t", None), ("kat_s", None), ("kat_b", None), ("stress", 1), ("stress", 8),
        ("stress", 64)]


def _sample(w, k=60000, seed=0):
    """Random elements plus the first and last rows and tile-boundary rows."""
    rng = np.random.default_rng(seed)
    idx = rng.choice(w.elems, size=k, replace=False)
    rows = [0, w.rows - 1] + list(range(63, w.rows, 4096))
    extra = np.concatenate([r * w.d + np.arange(w.d) for r in rows[:12]])
    return np.unique(np.concatenate([idx, extra])).astype(np.int64)


@pytest.mark.parametrize("name,n_g", FULL, ids=["%s%s" % (n, "" if g is None else g)
                                                for n, g in FULL])
def test_fullsize(name, n_g):
    w = synth.workload(name, n_g=n_g)
    x, dy = w.x(), w.dy()
    a, b = w.coefficients()
    tx, tdy = to_torch(x), to_torch(dy)
    ta, tb = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
    shape = (w.B, w.N, w.d)
    tx = tx.view(shape)
    tdy = tdy.view(shape)
    assert grk.grkan_backward_path(tx, tdy, tdy, w.B, w.N, w.d, w.n_g, w.m, w.n, w.dtype) == 1
    y = grk.forward(tx, ta, tb, w.n_g)
    dx, dA, dB = grk.backward(tx, tdy, ta, tb, w.n_g)
    torch.cuda.synchronize()

    idx = _sample(w)
    tidx = torch.from_numpy(idx).cuda()
    y_s = to_f64(y.reshape(-1)[tidx])
    dx_s = to_f64(dx.reshape(-1)[tidx])
    y_ref, ky = oracle.forward(x, a, b, w.n_g, idx=idx, kappa=True)
    dx_ref, ex = oracle.backward_elem(x, dy, a, b, w.n_g, idx=idx, extras=True)
    rtol = RTOL[w.dtype]
    check_y(y_s, y_ref, ky, rtol, "%s y" % w.name)
    check_dx(dx_s, dx_ref, ex, rtol, "%s dx" % w.name)

    g_ref = oracle.coef_grads(x, dy, a, b, w.n_g)
    # The KAT-shaped workloads meet the plain 1e-4 relative bound on every entry
    # whose sum does not cancel below 1e-8 of its terms' magnitudes; the noise
    # floor is needed only for the heavy-tailed stress sweep.
    rep = coef_report(dA.cpu().numpy(), dB.cpu().numpy(), g_ref, what=w.name,
                      plain=name != "stress")
    print("%s: dA/dB max plain relative error %.3g (graded entries %.3g), %d of %d entries "
          "pass only through the noise floor or the sign allowance, %d ungraded; ambiguous "
          "signs %d" % (w.name, rep["max_rel"], rep["max_rel_graded"], rep["floor_only"],
                        rep["entries"], rep["ungraded"], g_ref["amb_count"]))

    for _ in range(2):
        again = grk.backward(tx, tdy, ta, tb, w.n_g)
        assert torch.equal(again[1], dA) and torch.equal(again[2], dB)
        assert torch.equal(again[0], dx)
    assert grk.grkan_device_error()[1] == 0

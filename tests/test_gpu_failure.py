"""Failure detection without a GPU fault: a bounded wait on an mbarrier phase
that nothing completes runs out after its limit, the kernel records the error in
the device error word and returns, and the context stays usable (a forward and a
backward afterwards match the oracle)."""
import time

import numpy as np
import pytest
import torch

import group_rational_kan_b200 as grk
import oracle
import synth
from parity import check_coef, check_dx, check_y, to_f64, to_torch

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_context_stays_usable():
    assert grk.grkan_clear_device_error() == 0
    assert grk.grkan_device_error()[1] == 0
    t0 = time.perf_counter()
    assert grk.grkan_selftest_wait_timeout(20000) == 0  # 20 ms
    st, code = grk.grkan_device_error()  # synchronises the stream
    dt = time.perf_counter() - t0
    assert st == 0
    assert code & grk.DEVICE_ERROR_SELFTEST
    assert 0.015 < dt < 1.5, dt
    assert grk.grkan_clear_device_error() == 0
    assert grk.grkan_device_error()[1] == 0

    # the context still works: the pipelined path against the oracle
    w = synth.workload("tiny")
    x = w.x()
    dy = w.dy()
    a, b = w.coefficients()
    tx, tdy = to_torch(x), to_torch(dy)
    ta, tb = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
    y = grk.forward(tx, ta, tb, w.n_g)
    dx, dA, dB = grk.backward(tx, tdy, ta, tb, w.n_g)
    torch.cuda.synchronize()
    assert grk.grkan_device_error()[1] == 0
    x2 = x.reshape(w.rows, w.d)
    dy2 = dy.reshape(w.rows, w.d)
    ref_y, ky = oracle.forward(x2, a, b, w.n_g, kappa=True)
    check_y(to_f64(y).reshape(ref_y.shape), ref_y, ky, 1e-5)
    ref_dx, ex = oracle.backward_elem(x2, dy2, a, b, w.n_g, extras=True)
    check_dx(to_f64(dx).reshape(ref_dx.shape), ref_dx, ex, 1e-5)
    check_coef(dA.cpu().numpy(), dB.cpu().numpy(), oracle.coef_grads(x2, dy2, a, b, w.n_g))

"""More than 2^31 elements in one call (KAT-B channel width, 700,000 rows of
bf16: 2.15e9 elements, 4.3 GB per tensor): every index past 32 bits, in the
kernels the benchmark times. y and dx on sampled elements (including the last
rows) against the oracle one by one, dA and dB against the oracle's reduction
over every element."""
import numpy as np
import pytest
import torch

import group_rational_kan_b200 as grk
import oracle
import synth
from parity import RTOL, check_coef, check_dx, check_y, to_f64, to_torch

pytestmark = pytest.mark.gpu


def test_beyond_32_bit_element_count():
    w = synth.workload("kat_b").with_rows(700_000)
    w.B, w.N = 700_000, 1
    w.rows_override = None
    assert w.elems > 2 ** 31
    free, _ = torch.cuda.mem_get_info()
    if free < 5 * w.elems * 2:
        pytest.skip("needs about 22 GB of free device memory")
    x, dy = w.x(), w.dy()
    a, b = w.coefficients()
    tx, tdy = to_torch(x), to_torch(dy)
    ta, tb = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
    assert grk.grkan_forward_path(tx, tx, w.rows, 1, w.d, w.n_g, w.m, w.n, w.dtype) == 1
    assert grk.grkan_backward_path(tx, tdy, tdy, w.rows, 1, w.d, w.n_g, w.m, w.n, w.dtype) == 1
    y = grk.forward(tx, ta, tb, w.n_g)
    dx, dA, dB = grk.backward(tx, tdy, ta, tb, w.n_g)
    torch.cuda.synchronize()
    assert grk.grkan_device_error()[1] == 0

    rng = np.random.default_rng(7)
    last = np.arange((w.rows - 3) * w.d, w.elems, dtype=np.int64)
    idx = np.unique(np.concatenate([rng.choice(w.elems, 40000, replace=False), last,
                                    np.arange(2 ** 31 - 4096, 2 ** 31 + 4096)])).astype(np.int64)
    tidx = torch.from_numpy(idx).cuda()
    y_ref, ky = oracle.forward(x, a, b, w.n_g, idx=idx, kappa=True)
    dx_ref, ex = oracle.backward_elem(x, dy, a, b, w.n_g, idx=idx, extras=True)
    check_y(to_f64(y.reshape(-1)[tidx]), y_ref, ky, RTOL[w.dtype], "huge y")
    check_dx(to_f64(dx.reshape(-1)[tidx]), dx_ref, ex, RTOL[w.dtype], "huge dx")
    del y, dx
    g_ref = oracle.coef_grads(x, dy, a, b, w.n_g)
    check_coef(dA.cpu().numpy(), dB.cpu().numpy(), g_ref, what="huge")

"""The accumulation schemes that the FlashKAT paper compares (paper notes,
section "Ablation": gradient rounding error of KAT's per-element atomic adds
against FlashKAT's per-block accumulation), measured against the fp64 oracle on
the same inputs, next to this library's two-stage fixed-order reduction.

Pinned here: dx of both atomic schemes is the generic backward's, bit for bit;
the per-element scheme's mean absolute error is well above the per-block
scheme's (at least four times: the ratio depends on the order in which the
atomics land and was measured between 9.9 and about 15) and at least ten times
the two-stage reduction's, and the per-block scheme's is above the two-stage
reduction's (the direction of the paper's table); the two-stage result stays
within the library's tolerance and is identical from run to run."""
import numpy as np
import pytest
import torch

import group_rational_kan_b200 as grk
import oracle
import synth
from parity import check_coef, to_torch

pytestmark = pytest.mark.gpu


def _setup(w):
    x, dy = w.x(), w.dy()
    a, b = w.coefficients()
    tx, tdy = to_torch(x), to_torch(dy)
    ta = torch.from_numpy(a).cuda()
    tb = torch.from_numpy(b.reshape(w.n_g, w.n)).cuda()
    ref = oracle.coef_grads(x, dy, a, b, w.n_g)
    return tx, tdy, ta, tb, ref


def _atomic(w, tx, tdy, ta, tb, mode, block_rows=0):
    dx = torch.empty_like(tx)
    dA = torch.empty(w.n_g, w.m + 1, device="cuda")
    dB = torch.empty(w.n_g, w.n, device="cuda")
    st = grk.grkan_backward_atomic(tx, tdy, ta, tb, dx, dA, dB, w.rows, 1, w.d, w.n_g, w.m, w.n,
                                   w.dtype, mode, block_rows)
    assert st == 0, grk.grkan_status_string(st)
    return dx, dA, dB


def _errors(dA, dB, ref):
    got = np.concatenate([dA.cpu().numpy().ravel(), dB.cpu().numpy().ravel()]).astype(np.float64)
    want = np.concatenate([ref["dA"].ravel(), ref["dB"].ravel()])
    err = np.abs(got - want)
    return float(err.mean()), float(err.var()), float(np.max(err / np.maximum(np.abs(want), 1e-30)))


@pytest.mark.parametrize("name,rows", [("kat_t", 20000), ("stress", 8000)])
def test_atomic_schemes_against_the_two_stage_reduction(name, rows):
    w = synth.workload(name, n_g=8 if name == "stress" else None).with_rows(rows)
    tx, tdy, ta, tb, ref = _setup(w)
    gdx, _, _ = grk.backward(tx, tdy, ta, tb, w.n_g, flags=grk.FLAG_GENERIC)
    runs = {}
    for label, mode in (("per_element", grk.ATOMIC_PER_ELEMENT), ("per_block", grk.ATOMIC_PER_BLOCK)):
        outs = [_atomic(w, tx, tdy, ta, tb, mode) for _ in range(3)]
        for dx, _, _ in outs:
            assert torch.equal(dx, gdx), label
        runs[label] = outs
    runs["two_stage"] = [grk.backward(tx, tdy, ta, tb, w.n_g) for _ in range(3)]
    torch.cuda.synchronize()
    table = {}
    for label, outs in runs.items():
        errs = [_errors(dA, dB, ref) for _, dA, dB in outs]
        same = all(torch.equal(o[1], outs[0][1]) and torch.equal(o[2], outs[0][2]) for o in outs)
        table[label] = (np.mean([e[0] for e in errs]), np.mean([e[1] for e in errs]),
                        max(e[2] for e in errs), same)
    print("\n%s, %d rows: scheme, MAE, error variance, max relative error, identical runs" %
          (w.name, w.rows))
    for label, (mae, var, rel, same) in table.items():
        print("  %-12s %.3e %.3e %.3e %s" % (label, mae, var, rel, same))
    assert table["per_element"][0] > 4 * table["per_block"][0]
    assert table["per_element"][0] > 10 * table["two_stage"][0]
    assert table["per_block"][0] > table["two_stage"][0]
    assert table["two_stage"][3]
    _, dA, dB = runs["two_stage"][0]
    check_coef(dA.cpu().numpy(), dB.cpu().numpy(), ref, what=w.name)


def test_atomic_entry_point_rejects_bad_mode_and_zeroes_on_empty():
    w = synth.workload("tiny")
    t = torch.empty(16, device="cuda")
    dA = torch.full((w.n_g, w.m + 1), 7.0, device="cuda")
    dB = torch.full((w.n_g, w.n), 7.0, device="cuda")
    assert grk.grkan_backward_atomic(t, t, t, t, t, dA, dB, 1, 1, w.d, w.n_g, w.m, w.n, w.dtype,
                                     3) == 8  # GRKAN_ERR_FLAGS
    assert grk.grkan_backward_atomic(t, t, t, t, t, dA, dB, 0, 1, w.d, w.n_g, w.m, w.n, w.dtype,
                                     grk.ATOMIC_PER_BLOCK) == 0
    torch.cuda.synchronize()
    assert torch.count_nonzero(dA) == 0 and torch.count_nonzero(dB) == 0

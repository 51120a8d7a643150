"""grkan_backward_noalloc: the backward entry point for callers that cannot
allocate device memory per call (for example a plugin whose host framework owns
all device memory and forbids allocation while enqueueing, or a process that must
keep its device footprint fixed after start-up). It uses the library's static
scratch array instead of a caller workspace; its results must match the regular
grkan_backward entry point's, call after call, whatever the array held before.

This file is collected last on purpose; it must pass alone in a fresh process
and after the rest of the suite."""
import numpy as np
import pytest
import torch

import group_rational_kan_b200 as grk
import synth

pytestmark = pytest.mark.gpu



def _inputs(w):
    x, dy = w.x(), w.dy()
    a, b = w.coefficients()

    def dev(arr):
        if arr.dtype == np.uint16:
            return torch.from_numpy(arr.view(np.int16)).view(torch.bfloat16).cuda()
        return torch.from_numpy(arr).cuda()

    return dev(x), dev(dy), torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()


def _via_workspace(w, tx, tdy, ta, tb):
    return grk.backward(tx, tdy, ta, tb, w.n_g)


def _via_noalloc(w, tx, tdy, ta, tb):
    dx = torch.empty_like(tx)
    dA = torch.empty(w.n_g, w.m + 1, device="cuda")
    dB = torch.empty(w.n_g, w.n, device="cuda")
    st = grk.grkan_backward_noalloc(tx, tdy, ta, tb, dx, dA, dB, w.rows, 1, w.d, w.n_g, w.m,
                                    w.n, w.dtype)
    assert st == 0, grk.grkan_status_string(st)
    return dx, dA, dB


def _same(got, ref):
    # the same plan, kernels, partial layout and merge order as grkan_backward:
    # the results must be the same bits (a leftover partial from an earlier call
    # or a skipped tile would show up here, however small)
    for u, v in zip(got, ref):
        assert torch.equal(u, v)


def test_noalloc_matches_workspace_entry_point_call_after_call():
    cases = [synth.workload("kat_b").with_rows(2000), synth.workload("kat_t").with_rows(1500),
             synth.workload("stress", n_g=64).with_rows(300)]
    prepared = [(w,) + _inputs(w) for w in cases]
    refs = [_via_workspace(*p) for p in prepared]
    # two rounds in a row: the scratch keeps the previous call's partials, which
    # must not leak into the next result
    for _ in range(2):
        for p, ref in zip(prepared, refs):
            _same(_via_noalloc(*p), ref)
    st, code = grk.grkan_device_error()
    assert st == 0 and code == 0


def test_noalloc_rejects_shapes_beyond_the_scratch():
    B = 16384  # a KAT-B-width activation 32 times the size of the workload's batch
    need = grk.grkan_backward_workspace_bytes(B, 197, 3072, 8, 5, 4, grk.BF16)
    assert need > grk.NOALLOC_WORKSPACE_BYTES
    x = torch.empty(8, device="cuda")
    st = grk.grkan_backward_noalloc(x, x, x, x, x, x, x, B, 197, 3072, 8, 5, 4, grk.BF16)
    assert st == 5  # GRKAN_ERR_WORKSPACE, nothing launched

"""grkan_step_host: forward + backward of host-resident tensors streamed in row
chunks through device scratch on three streams. The results must be the same
bits as grkan_forward + grkan_backward on device copies of the same data,
whatever the chunking (chunks are whole reduction tiles)."""
import numpy as np
import pytest
import torch

import group_rational_kan_b200 as grk
import synth

pytestmark = pytest.mark.gpu


def _host(arr):
    t = torch.from_numpy(arr.view(np.int16) if arr.dtype == np.uint16 else arr)
    if arr.dtype == np.uint16:
        t = t.view(torch.bfloat16)
    return t.pin_memory()


@pytest.mark.parametrize("name,rows,chunk", [("kat_b", 333, 96), ("kat_b", 333, 0),
                                             ("kat_t", 700, 64), ("stress", 150, 16),
                                             ("tiny", 32, 0)])
def test_host_step_matches_device_calls(name, rows, chunk):
    w = synth.workload(name).with_rows(rows)
    x, dy = w.x(), w.dy()
    a_np, b_np = w.coefficients()
    a, b = torch.from_numpy(a_np).cuda(), torch.from_numpy(b_np).cuda()
    xh, dyh = _host(x), _host(dy)
    yh, dxh = torch.empty_like(xh).pin_memory(), torch.empty_like(xh).pin_memory()
    dAh = torch.empty(w.n_g, w.m + 1).pin_memory()
    dBh = torch.empty(w.n_g, w.n).pin_memory()
    need = grk.grkan_step_host_scratch_bytes(w.rows, 1, w.d, w.n_g, w.m, w.n, w.dtype, chunk)
    scratch = torch.empty(need, dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    for _ in range(2):  # a second call reuses streams, events and staging slots
        sums = torch.empty(w.n_g, w.m + 1 + w.n, dtype=torch.float64, device="cuda")
        st = grk.grkan_step_host(xh, dyh, a, b, yh, dxh, dAh, dBh, sums, w.rows, 1, w.d, w.n_g,
                                 w.m, w.n, w.dtype, scratch, need, chunk, stream=s)
        assert st == 0, grk.grkan_last_error()
        s.synchronize()
        xd, dyd = xh.cuda(), dyh.cuda()
        y = grk.forward(xd, a, b, w.n_g)
        dx, dA, dB = grk.backward(xd, dyd, a, b, w.n_g)
        torch.cuda.synchronize()
        assert torch.equal(yh, y.cpu()) and torch.equal(dxh, dx.cpu())
        assert torch.equal(dAh, dA.cpu()) and torch.equal(dBh, dB.cpu())
        # the float64 sums are the ones grkan_backward_merge gives for the batch
        wsb = grk.grkan_backward_workspace_bytes(w.rows, 1, w.d, w.n_g, w.m, w.n, w.dtype)
        ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device="cuda")
        dx2 = torch.empty_like(xd)
        ref = torch.empty_like(sums)
        assert grk.grkan_backward_partials(xd, dyd, a, b, dx2, w.rows, 1, w.d, w.n_g, w.m, w.n,
                                           w.dtype, ws, wsb, 0) == 0
        assert grk.grkan_backward_merge(ws, wsb, dA, dB, ref, w.rows, 1, w.d, w.n_g, w.m, w.n,
                                        w.dtype) == 0
        torch.cuda.synchronize()
        assert torch.equal(sums, ref)


def test_host_step_rejects_small_scratch():
    x = torch.empty(4, 64).pin_memory()
    a = torch.zeros(8, 6, device="cuda")
    b = torch.zeros(8, 4, device="cuda")
    need = grk.grkan_step_host_scratch_bytes(4, 1, 64, 8, 5, 4, grk.F32, 0)
    scratch = torch.empty(need, dtype=torch.uint8, device="cuda")
    dA = torch.empty(8, 6).pin_memory()
    dB = torch.empty(8, 4).pin_memory()
    st = grk.grkan_step_host(x, x, a, b, x, x, dA, dB, None, 4, 1, 64, 8, 5, 4, grk.F32, scratch,
                             need - 256, 0)
    assert st == 5

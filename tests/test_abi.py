"""The C-ABI library without a GPU: it loads, exports every symbol that
include/grkan.h declares, and rejects bad arguments with the documented codes
before touching CUDA."""
import ctypes
import os
import re

import pytest

import group_rational_kan_b200 as grk

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "grkan.h")

OK, NULL, SHAPE, DEGREE, DTYPE, WORKSPACE, CUDA, ALIAS, FLAGS, DEVICE = range(10)


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"GRKAN_API\s+[\w\s\*]+?\b(grkan_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for need in ("grkan_forward", "grkan_backward", "grkan_backward_workspace_bytes",
                 "grkan_status_string"):
        assert need in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(grk.library_path if os.path.exists(grk.library_path) else grk.lib()._name)
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert grk.grkan_abi_version() == grk.ABI_VERSION == 3


def test_status_strings():
    for code in range(10):
        s = grk.grkan_status_string(code)
        assert s.startswith("GRKAN_")
    assert "UNKNOWN" in grk.grkan_status_string(99)


def test_workspace_bytes():
    # KAT-B: d_g = 384 bf16 -> backward boxes of 8 rows x 192 channels (3 KiB), 2 per
    # group row, 8 boxes per unit -> 32 rows per tile, 3152 tiles
    assert grk.grkan_backward_workspace_bytes(512, 197, 3072, 8, 5, 4, grk.BF16) == 3152 * 8 * 10 * 4
    # KAT-T: d_g = 96 f32 -> boxes of 4 rows x 96 channels (1.5 KiB) -> 32 rows per
    # tile, 6304 tiles
    assert grk.grkan_backward_workspace_bytes(1024, 197, 768, 8, 5, 4, grk.F32) == 6304 * 8 * 10 * 4
    assert grk.grkan_backward_workspace_bytes(0, 197, 768, 8, 5, 4, grk.F32) == 0
    assert grk.grkan_backward_workspace_bytes(2, 3, 10, 3, 5, 4, grk.F32) == 0  # d % n_g != 0
    assert grk.grkan_backward_workspace_bytes(2, 3, 12, 3, 9, 4, grk.F32) == 0  # degree


def test_path_selection():
    A = 1 << 20  # an aligned fake address, never dereferenced
    kat_b = (512, 197, 3072, 8, 5, 4, grk.BF16)
    assert grk.grkan_forward_path(A, A, *kat_b) == 1
    assert grk.grkan_backward_path(A, A, A, *kat_b) == 1
    assert grk.grkan_backward_path(A, A, A, *kat_b, flags=grk.FLAG_GENERIC) == 0
    assert grk.grkan_backward_path(A + 4, A, A, *kat_b) == 0  # unaligned -> generic
    assert grk.grkan_forward_path(A, A, 2, 3, 30, 3, 5, 4, grk.F32) == 0  # 40-byte groups
    assert grk.grkan_forward_path(A, A, 2, 3, 48, 4, 3, 2, grk.F32) == 0  # other degree
    assert grk.grkan_forward_path(A, A, 2, 16, 64, 8, 5, 4, grk.F32) == 1  # tiny
    assert grk.grkan_forward_path(A, A, 256, 197, 3072, 1, 5, 4, grk.F32) == 1  # n_g = 1
    assert grk.grkan_forward_path(A, A, 256, 197, 3072, 64, 5, 4, grk.F32) == 1  # n_g = 64
    assert grk.grkan_forward_path(A, A, 2, 3, 12, 5, 5, 4, grk.F32) == -SHAPE
    assert grk.grkan_forward_path(A, A, 2, 3, 12, 3, 5, 4, 7) == -DTYPE
    assert grk.grkan_forward_path(A, A, 2, 3, 12, 3, 5, 4, grk.F32, flags=8) == -FLAGS


def test_linear_forward_path():
    """The fused linear forward's kernel by shape (no device needed): the cluster
    kernel for n_out > 512 when d is a multiple of 64, the one-CTA kernel
    otherwise."""
    p = grk.grkan_linear_forward_path
    kat_b = (512, 197, 3072, 8, 5, 4)
    assert p(*kat_b, 768, grk.BF16) == 1    # one tile, pairs of 384
    assert p(*kat_b, 1024, grk.BF16) == 1   # one tile, pairs of 512
    assert p(*kat_b, 576, grk.BF16) == 1
    assert p(*kat_b, 512, grk.BF16) == 0    # one 512-column pass of the one-CTA kernel
    assert p(*kat_b, 384, grk.BF16) == 0
    assert p(*kat_b, 1536, grk.BF16) == 1   # two tiles with pairs of 384
    assert p(*kat_b, 520, grk.BF16) == 1    # just past one 512-column pass
    assert p(*kat_b, 2048, grk.BF16) == 1   # two tiles with pairs of 512
    assert p(512, 197, 768, 8, 5, 4, 3072, grk.BF16) == 1   # three tiles of 1024
    assert p(2, 3, 160, 20, 5, 4, 768, grk.BF16) == 0       # d not a multiple of 64
    assert p(0, 197, 3072, 8, 5, 4, 768, grk.BF16) == 1     # empty: the shape rule still holds
    assert p(*kat_b, 768, grk.F32) == -DTYPE
    assert p(512, 197, 3072, 8, 3, 3, 768, grk.BF16) == -DEGREE
    assert p(*kat_b, 770, grk.BF16) == -SHAPE              # n_out % 8
    assert p(512, 197, 48, 6, 5, 4, 768, grk.BF16) == -SHAPE  # d % 32
    assert p(1, 1, 0, 8, 5, 4, 64, grk.BF16) == -SHAPE     # d == 0


def test_argument_errors_need_no_gpu():
    A = 1 << 20
    f = grk.grkan_forward_ex
    shape = (2, 3, 12, 3, 5, 4, grk.F32)
    assert f(None, A, A, A, *shape, 0, 0) == NULL
    assert f(A, None, A, A, *shape, 0, 0) == NULL
    assert f(A, A, None, A, *shape, 0, 0) == NULL
    assert f(A, A, A, None, *shape, 0, 0) == NULL
    assert f(A, A, A, None, 2, 3, 12, 3, 5, 0, grk.F32, 0, 0) != NULL  # n = 0: b may be NULL
    assert f(A, A, A, A, 2, 3, 12, 5, 5, 4, grk.F32, 0, 0) == SHAPE
    assert f(A, A, A, A, -1, 3, 12, 3, 5, 4, grk.F32, 0, 0) == SHAPE
    assert f(A, A, A, A, 2, 3, 12, 0, 5, 4, grk.F32, 0, 0) == SHAPE
    assert f(A, A, A, A, 2, 3, 12, 3, 9, 4, grk.F32, 0, 0) == DEGREE
    assert f(A, A, A, A, 2, 3, 12, 3, 5, -1, grk.F32, 0, 0) == DEGREE
    assert f(A, A, A, A, 2, 3, 12, 3, 5, 4, 3, 0, 0) == DTYPE
    assert f(A, A, A, A, *shape, 2, 0) == FLAGS
    assert f(A, A + 4, A, A, *shape, 0, 0) == ALIAS  # partial overlap
    assert f(A, A, A, A, 1 << 40, 1 << 40, 12, 3, 5, 4, grk.F32, 0, 0) == SHAPE  # overflow
    assert f(None, None, None, None, 0, 3, 12, 3, 5, 4, grk.F32, 0, 0) == OK  # empty: no-op
    # everything valid but no sm_100 device here
    if not _has_gpu():
        assert f(A, A, A, A, *shape, 0, 0) == DEVICE


def test_backward_argument_errors_need_no_gpu():
    X = 1 << 20   # x and dy (inputs may share memory)
    D = 1 << 24   # dx
    W = 1 << 30   # workspace
    shape = (2, 3, 12, 3, 5, 4, grk.F32)
    nbytes = 2 * 3 * 12 * 4
    need = grk.grkan_backward_workspace_bytes(*shape)
    assert need > 0
    b = grk.grkan_backward_ex
    assert b(X, X, X, X, D, None, X, *shape, W, need, 0, 0) == NULL
    assert b(X, X, X, X, D, X, None, *shape, W, need, 0, 0) == NULL
    assert b(X, X, X, X, D, X, X, *shape, None, need, 0, 0) == WORKSPACE
    assert b(X, X, X, X, D, X, X, *shape, W, need - 4, 0, 0) == WORKSPACE
    assert b(X, X, X, X, D, X, X, *shape, W + 4, need, 0, 0) == WORKSPACE  # unaligned
    assert b(X, X, X, X, X + 8, X, X, *shape, W, need, 0, 0) == ALIAS  # dx overlaps x
    assert b(X, X, X, X, X, X, X, *shape, W, need, 0, 0) == ALIAS  # dx == x: x must stay
    assert b(X, D + 16, X, X, D, X, X, *shape, W, need, 0, 0) == ALIAS  # dx overlaps dy
    assert b(X, X, X, X, D, X, X, *shape, X + 16, need, 0, 0) == ALIAS  # workspace inside x
    assert b(X, X, X, X, D, X, X, *shape, D + nbytes - 16, need, 0, 0) == ALIAS  # ... inside dx
    assert b(X, X, X, X, D, X, X, *shape, W, need, 4, 0) == FLAGS
    fb = grk.grkan_forward_backward
    Y = 1 << 28
    assert fb(X, D, X, X, Y, X, X, X, *shape, W, need, 0, 0) == ALIAS  # dx == x
    assert fb(X, D, X, X, X, D, X, X, *shape, W, need, 0, 0) == ALIAS  # y == x
    at = grk.grkan_backward_atomic
    assert at(X, X, X, X, X, X, X, *shape, 1, 0, 0) == ALIAS  # dx == x
    if not _has_gpu():
        assert b(X, X, X, X, D, X, X, *shape, W, need, 0, 0) == DEVICE
        assert b(X, D, X, X, D, X, X, *shape, W, need, 0, 0) == DEVICE  # dx == dy is allowed
        assert fb(X, D, X, X, Y, D, X, X, *shape, W, need, 0, 0) == DEVICE


def test_huge_rows_of_narrow_groups_take_the_generic_path():
    """The pipelined kernels keep a lane's offsets inside a TMA box in 32-bit
    integers; shapes whose box would span 2^31 bytes or more go to the generic
    kernels (bf16, d_g = 8: 192-row backward boxes)."""
    A = 1 << 20
    assert grk.grkan_forward_path(A, A, 1, 1, 8 << 10, 1 << 10, 5, 4, grk.BF16) == 1
    assert grk.grkan_backward_path(A, A, A, 1, 1, 8 << 10, 1 << 10, 5, 4, grk.BF16) == 1
    assert grk.grkan_forward_path(A, A, 1, 1, 8 << 20, 1 << 20, 5, 4, grk.BF16) == 0
    assert grk.grkan_backward_path(A, A, A, 1, 1, 8 << 20, 1 << 20, 5, 4, grk.BF16) == 0


def _has_gpu():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    """The binding has no CPU fallback: a missing library is an ImportError."""
    import importlib
    import group_rational_kan_b200.build as b
    monkeypatch.setattr(grk, "_lib", None)
    monkeypatch.setattr(grk, "library_path", str(tmp_path / "nope.so"))
    monkeypatch.setattr(b, "needs_build", lambda: False)
    with pytest.raises(ImportError):
        grk.lib()
    importlib.reload(grk)


def test_linear_backward_argument_errors_need_no_gpu():
    A = 1 << 20        # x
    DO = 1 << 28       # dout
    WT = 1 << 29       # W
    DX = 1 << 30       # dx
    WS = 1 << 31       # workspace
    K = (1 << 32)      # dA, dB, coefficients
    rows, d, n_g, nout = 300, 768, 4, 576
    need = grk.grkan_linear_backward_workspace_bytes(1, rows, d, n_g, 5, 4, nout, grk.BF16)
    # one float32 partial per (128-row tile, 64-channel block of a group, row quarter)
    assert need == 3 * (192 // 64) * 4 * n_g * 10 * 4
    assert grk.grkan_linear_backward_workspace_bytes(1, rows, d, n_g, 5, 4, nout, grk.F32) == 0
    assert grk.grkan_linear_backward_workspace_bytes(1, rows, d, 8, 5, 4, nout, grk.BF16) == 0
    assert grk.grkan_linear_backward_workspace_bytes(1, rows, d, n_g, 5, 4, 0, grk.BF16) == 0

    def call(x=A, dout=DO, W=WT, a=K, b=K + 64, dx=DX, dA=K + 256, dB=K + 512, rows=rows, d=d,
             n_g=n_g, m=5, n=4, nout=nout, dtype=grk.BF16, ws=WS, wsb=need):
        return grk.grkan_linear_backward(x, dout, W, a, b, dx, dA, dB, 1, rows, d, n_g, m, n,
                                         nout, dtype, ws, wsb, 0)

    assert call(dtype=grk.F32) == DTYPE
    assert call(m=4) == DEGREE
    assert call(n_g=8) == SHAPE            # d_g = 96: not a multiple of 64
    assert call(nout=100) == SHAPE         # nout % 8
    assert call(nout=-8) == SHAPE
    assert call(dA=None) == NULL
    assert call(x=None) == NULL
    assert call(dout=None) == NULL
    assert call(W=None) == NULL
    assert call(a=None) == NULL
    assert call(x=A + 8) == SHAPE          # 16-byte alignment
    assert call(ws=None) == WORKSPACE
    assert call(wsb=need - 4) == WORKSPACE
    assert call(ws=WS + 4) == WORKSPACE
    assert call(dx=A + 4096) == ALIAS      # dx overlaps x
    assert call(dx=DO) == ALIAS            # dx overlaps dout
    assert call(ws=DX + 4096) == ALIAS     # workspace inside dx
    assert call(nout=0, dx=None) == NULL   # dx = 0 is written
    if not _has_gpu():
        assert call() == DEVICE
        assert call(nout=0) == DEVICE      # zeroing needs the device too


def test_linear_forward_argument_errors_need_no_gpu():
    A, WT, O = 1 << 20, 1 << 29, 1 << 30
    K = 1 << 32

    def call(x=A, a=K, b=K + 64, W=WT, bias=None, out=O, d=768, n_g=8, m=5, n=4, nout=576,
             dtype=grk.BF16):
        return grk.grkan_linear_forward(x, a, b, W, bias, out, 1, 300, d, n_g, m, n, nout, dtype,
                                        0)

    assert call(dtype=grk.F32) == DTYPE
    assert call(n=3) == DEGREE
    assert call(d=760, n_g=8) == SHAPE     # d % 32
    assert call(nout=100) == SHAPE         # nout % 8
    assert call(x=None) == NULL
    assert call(W=WT + 8) == SHAPE         # alignment
    assert call(out=A + 64) == ALIAS       # out overlaps x
    if not _has_gpu():
        assert call() == DEVICE


def test_selftest_arguments_need_no_gpu():
    assert grk.grkan_selftest_wait_timeout(0, 0) == SHAPE
    assert grk.grkan_selftest_wait_timeout(2000001, 0) == SHAPE
    if not _has_gpu():
        assert grk.grkan_selftest_wait_timeout(1000, 0) == DEVICE

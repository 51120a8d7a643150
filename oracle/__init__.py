"""fp64 CPU oracle for the GR-KAN group-rational activation (ctypes binding).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package. The CUDA path never
calls it, and the two share no code. See ``grkan_oracle.h`` for the formulas
and their sources.

Pins (checked by ``tests/test_oracle_*.py`` against things other than the
oracle itself): identity initialisation, the b = 0 polynomial special case,
exact rational brute force on dyadic inputs, central finite differences for dx,
dA and dB, x = 0, linearity in dy, group relabelling, and an fp64 autograd
witness. The error scales that set the y / dx tolerances are pinned too:
kappa_q by brute force over the sign patterns of b, kappa_y as the largest
first-order sensitivity of y to relative coefficient perturbations (exact dual
numbers over every sign pattern) and by a closed form at nonnegative inputs,
kappa_dx by a closed form at nonnegative inputs, sign invariances and the
perturbation bound it gives, and the c2 noise scales by closed forms. Every
function here is pinned; ``tests/test_oracle_mutants.py`` plants 36 mistakes
and each one trips a pin.
"""
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "grkan_oracle.c")
LIB = os.path.join(_HERE, "libgrkan_oracle.so")

F32, BF16 = 0, 1

# Relative threshold below which the sign of Q(x) is treated as undecidable in
# float32 arithmetic: |Q| < AMB_REL * sum_j |b_j||x|^j. float32 evaluation of Q
# with n <= 8 terms carries an error of at most about 2 n u sum_j |b_j||x|^j,
# u = 2^-24; 2^-17 leaves a margin of 4 above that for n = 8.
AMB_REL = 2.0 ** -17


def build(src: str = SRC, out: str = LIB, force: bool = False) -> str:
    """Compile the oracle with gcc (C11, OpenMP)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < max(
            os.path.getmtime(src), os.path.getmtime(os.path.join(_HERE, "grkan_oracle.h"))):
        tmp = out + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c11",
                               "-ffp-contract=off", "-I", _HERE, "-o", tmp, src, "-lm"])
        os.replace(tmp, out)
    return out


def _ptr(a):
    return None if a is None else a.ctypes.data


class Oracle:
    """One loaded oracle library (the committed one, or a test's planted variant)."""

    def __init__(self, lib_path: str = None):
        if lib_path is None:
            lib_path = build()
        lib = ctypes.CDLL(lib_path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I = ctypes.c_int
        lib.gro_forward.argtypes = [P, I, I64, I64, I, I, I, P, P, P, I64, P, P]
        lib.gro_forward.restype = I
        lib.gro_backward_elem.argtypes = [P, P, I, I64, I64, I, I, I, P, P, P, I64, P, P, P, P, P]
        lib.gro_backward_elem.restype = I
        lib.gro_coef_grads.argtypes = [P, P, I, I64, I64, I, I, I, P, P, ctypes.c_double, P, P, P,
                                       P, P, P, P, P, I]
        lib.gro_coef_grads.restype = I
        lib.gro_max_threads.restype = I
        self.lib = lib

    @staticmethod
    def _prep(x, a, b, n_g):
        if x.dtype == np.float32:
            dtype = F32
        elif x.dtype == np.uint16:
            dtype = BF16
        else:
            raise TypeError("x must be float32 or uint16 (bf16 bits), got %s" % x.dtype)
        x = np.ascontiguousarray(x)
        rows, d = x.shape
        a = np.ascontiguousarray(np.asarray(a, dtype=np.float32), dtype=np.float64).reshape(n_g, -1)
        b = np.ascontiguousarray(np.asarray(b, dtype=np.float32), dtype=np.float64).reshape(n_g, -1)
        return x, dtype, rows, d, a, b, a.shape[1] - 1, b.shape[1]

    def forward(self, x, a, b, n_g, idx=None, kappa=False):
        """y (float64, same shape as x, or per idx) and optionally its error scale."""
        x, dtype, rows, d, a, b, m, n = self._prep(x, a, b, n_g)
        if idx is not None:
            idx = np.ascontiguousarray(idx, dtype=np.int64)
            cnt = idx.size
            shape = idx.shape
        else:
            cnt = rows * d
            shape = (rows, d)
        y = np.empty(cnt, np.float64)
        ky = np.empty(cnt, np.float64) if kappa else None
        rc = self.lib.gro_forward(x.ctypes.data, dtype, rows, d, n_g, m, n, a.ctypes.data,
                                  b.ctypes.data, _ptr(idx), cnt, y.ctypes.data, _ptr(ky))
        if rc:
            raise ValueError("gro_forward returned %d" % rc)
        return (y.reshape(shape), ky.reshape(shape)) if kappa else y.reshape(shape)

    def backward_elem(self, x, dy, a, b, n_g, idx=None, extras=False):
        """dx (float64). With extras=True also returns a dict of kappa_dx,
        dx_sign (..., 3) for s = -1, 0, +1, q and kappa_q."""
        x, dtype, rows, d, a, b, m, n = self._prep(x, a, b, n_g)
        dy = np.ascontiguousarray(dy)
        assert dy.dtype == x.dtype and dy.shape == x.shape
        if idx is not None:
            idx = np.ascontiguousarray(idx, dtype=np.int64)
            cnt = idx.size
            shape = idx.shape
        else:
            cnt = rows * d
            shape = (rows, d)
        dx = np.empty(cnt, np.float64)
        kdx = dxs = q = kq = None
        if extras:
            kdx = np.empty(cnt, np.float64)
            dxs = np.empty((cnt, 3), np.float64)
            q = np.empty(cnt, np.float64)
            kq = np.empty(cnt, np.float64)
        rc = self.lib.gro_backward_elem(x.ctypes.data, dy.ctypes.data, dtype, rows, d, n_g, m, n,
                                        a.ctypes.data, b.ctypes.data, _ptr(idx), cnt,
                                        dx.ctypes.data, _ptr(kdx), _ptr(dxs), _ptr(q), _ptr(kq))
        if rc:
            raise ValueError("gro_backward_elem returned %d" % rc)
        if not extras:
            return dx.reshape(shape)
        return dx.reshape(shape), {
            "kappa_dx": kdx.reshape(shape), "dx_sign": dxs.reshape(shape + (3,)),
            "q": q.reshape(shape), "kappa_q": kq.reshape(shape)}

    def coef_grads(self, x, dy, a, b, n_g, amb_rel=AMB_REL, nthreads=0):
        """dict with dA (n_g, m+1), dB (n_g, n), sabs_a, sabs_b (sums of |term|),
        c2_a, c2_b (conditioned sums of squares), amb_b (float64) and amb_count."""
        x, dtype, rows, d, a, b, m, n = self._prep(x, a, b, n_g)
        dy = np.ascontiguousarray(dy)
        assert dy.dtype == x.dtype and dy.shape == x.shape
        dA = np.empty((n_g, m + 1), np.float64)
        dB = np.empty((n_g, n), np.float64)
        sa = np.empty_like(dA)
        sb = np.empty_like(dB)
        ca = np.empty_like(dA)
        cb = np.empty_like(dB)
        ab = np.empty_like(dB)
        cnt = ctypes.c_int64(0)
        rc = self.lib.gro_coef_grads(x.ctypes.data, dy.ctypes.data, dtype, rows, d, n_g, m, n,
                                     a.ctypes.data, b.ctypes.data, float(amb_rel), dA.ctypes.data,
                                     dB.ctypes.data, sa.ctypes.data, sb.ctypes.data,
                                     ca.ctypes.data, cb.ctypes.data, ab.ctypes.data,
                                     ctypes.addressof(cnt), int(nthreads))
        if rc:
            raise ValueError("gro_coef_grads returned %d" % rc)
        return {"dA": dA, "dB": dB, "sabs_a": sa, "sabs_b": sb, "c2_a": ca, "c2_b": cb,
                "amb_b": ab, "amb_count": int(cnt.value)}

    def max_threads(self) -> int:
        return int(self.lib.gro_max_threads())


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def forward(*args, **kw):
    return default().forward(*args, **kw)


def backward_elem(*args, **kw):
    return default().backward_elem(*args, **kw)


def coef_grads(*args, **kw):
    return default().coef_grads(*args, **kw)

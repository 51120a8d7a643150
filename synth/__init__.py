"""Seeded synthetic inputs for GR-KAN workloads (x, dy, a, b).

Both the oracle and the CUDA path read what this module writes; it holds none
of the activation's arithmetic. The generator (``synth.c``) is counter-based:
element i of a tensor depends only on (seed, stream, i).

Streams: x = 1, dy = 2, a = 3, b = 4. Coefficients are float32, shape
a: (n_g, m+1) holding a_0..a_m, b: (n_g, n) holding b_1..b_n.
bf16 tensors are returned as numpy uint16 arrays of bf16 bit patterns.

Workload recipes follow the KAT model sizes (ViT-style, 224x224 images, 16x16
patches plus a class token: N = 197 tokens; MLP hidden width 4*embed) named in
the FlashKAT notes (sections "Main experiment" and "Loss / training strategy":
8 groups, 6 numerator and 4 denominator coefficients; first layer identity,
second layer Swish).
"""
import ctypes
import json
import os
import subprocess
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libgrkan_synth.so")
_lib = None

F32, BF16 = 0, 1
X_STREAM, DY_STREAM, A_STREAM, B_STREAM = 1, 2, 3, 4
KIND_NORMAL, KIND_STUDENT3, KIND_UNIFORM = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile synth.c into libgrkan_synth.so (gcc, OpenMP)."""
    src = os.path.join(_HERE, "synth.c")
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c11",
                               "-o", tmp, src, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        lib.synth_fill.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int, ctypes.c_int64,
                                   ctypes.c_int64, ctypes.c_double, ctypes.c_double, ctypes.c_int,
                                   ctypes.c_void_p, ctypes.c_int]
        lib.synth_fill.restype = ctypes.c_int
        lib.synth_fill_at.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int, ctypes.c_void_p,
                                      ctypes.c_int64, ctypes.c_double, ctypes.c_double, ctypes.c_int,
                                      ctypes.c_void_p]
        lib.synth_fill_at.restype = ctypes.c_int
        lib.synth_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def np_dtype(dtype: int):
    return np.float32 if dtype == F32 else np.uint16


def fill(out: np.ndarray, seed: int, stream: int, kind: int, scale: float, clip: float = 0.0,
         offset: int = 0, nthreads: int = 0) -> np.ndarray:
    """Write elements [offset, offset+out.size) of a seeded tensor into ``out``
    (float32, or uint16 holding bf16 bits). ``out`` must be C-contiguous."""
    lib = _load()
    assert out.flags["C_CONTIGUOUS"]
    dtype = F32 if out.dtype == np.float32 else BF16
    assert out.dtype in (np.float32, np.uint16)
    rc = lib.synth_fill(seed, stream, kind, offset, out.size, scale, clip, dtype,
                        out.ctypes.data, nthreads)
    if rc != 0:
        raise ValueError("synth_fill rejected its arguments")
    return out


def fill_ptr(ptr: int, count: int, dtype: int, seed: int, stream: int, kind: int, scale: float,
             clip: float = 0.0, offset: int = 0, nthreads: int = 0) -> None:
    """Same as :func:`fill` but into raw host memory (e.g. a pinned torch buffer)."""
    lib = _load()
    rc = lib.synth_fill(seed, stream, kind, offset, count, scale, clip, dtype, ptr, nthreads)
    if rc != 0:
        raise ValueError("synth_fill rejected its arguments")


def gather(idx: np.ndarray, dtype: int, seed: int, stream: int, kind: int, scale: float,
           clip: float = 0.0) -> np.ndarray:
    """Regenerate only the elements with flat indices ``idx``."""
    lib = _load()
    idx = np.ascontiguousarray(idx, dtype=np.int64)
    out = np.empty(idx.size, dtype=np_dtype(dtype))
    rc = lib.synth_fill_at(seed, stream, kind, idx.ctypes.data, idx.size, scale, clip, dtype,
                           out.ctypes.data)
    if rc != 0:
        raise ValueError("synth_fill_at rejected its arguments")
    return out


def bf16_bits_to_f32(u: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (u.astype(np.uint32) << 16).view(np.float32)


def max_threads() -> int:
    return int(_load().synth_max_threads())


def swish_fit():
    with open(os.path.join(_HERE, "swish_fit.json")) as f:
        j = json.load(f)
    return np.array(j["a"], dtype=np.float64), np.array(j["b"], dtype=np.float64)


@dataclass
class Workload:
    """One GR-KAN workload: shapes, dtypes and the recipe of every input."""
    name: str
    B: int
    N: int
    d: int
    n_g: int
    m: int
    n: int
    dtype: int
    x_kind: int
    x_scale: float
    x_clip: float
    dy_scale: float
    coef_base: str  # "zero", "identity" or "swish"
    coef_lo: float
    coef_hi: float
    seed: int = 0
    note: str = ""
    rows_override: Optional[int] = None
    extra: dict = field(default_factory=dict)

    @property
    def rows(self) -> int:
        return self.B * self.N if self.rows_override is None else self.rows_override

    @property
    def elems(self) -> int:
        return self.rows * self.d

    @property
    def es(self) -> int:
        return 4 if self.dtype == F32 else 2

    def with_rows(self, rows: int) -> "Workload":
        """The first ``rows`` rows of this workload (same values, element by element)."""
        w = Workload(**{k: getattr(self, k) for k in self.__dataclass_fields__})
        w.rows_override = rows
        return w

    def describe(self) -> dict:
        return {
            "workload": self.name, "B": self.B, "N": self.N, "d": self.d, "rows": self.rows,
            "n_g": self.n_g, "d_g": self.d // self.n_g, "m": self.m, "n": self.n,
            "dtype": "f32" if self.dtype == F32 else "bf16",
            "x": ("N(0,%g)" % self.x_scale) if self.x_kind == KIND_NORMAL
            else "Student-t(3) clipped at +-%g" % self.x_clip,
            "dy": "N(0,%g)" % self.dy_scale,
            "coefficients": "%s + U(%g,%g)" % (self.coef_base, self.coef_lo, self.coef_hi),
            "seed": self.seed,
        }

    # --- generation -------------------------------------------------------
    def coefficients(self):
        ua = np.empty(self.n_g * (self.m + 1), np.float32)
        ub = np.empty(self.n_g * self.n, np.float32)
        fill(ua, self.seed, A_STREAM, KIND_UNIFORM, self.coef_lo, self.coef_hi)
        fill(ub, self.seed, B_STREAM, KIND_UNIFORM, self.coef_lo, self.coef_hi)
        base_a = np.zeros(self.m + 1)
        base_b = np.zeros(self.n)
        if self.coef_base == "identity":
            if self.m >= 1:
                base_a[1] = 1.0
        elif self.coef_base == "swish":
            sa, sb = swish_fit()
            base_a[: min(self.m + 1, sa.size)] = sa[: self.m + 1]
            base_b[: min(self.n, sb.size)] = sb[: self.n]
        a = (np.tile(base_a, self.n_g) + ua.astype(np.float64)).astype(np.float32)
        b = (np.tile(base_b, self.n_g) + ub.astype(np.float64)).astype(np.float32)
        return a.reshape(self.n_g, self.m + 1), b.reshape(self.n_g, self.n)

    def x_into(self, out: np.ndarray, row0: int = 0, nthreads: int = 0) -> np.ndarray:
        kind = self.x_kind
        return fill(out, self.seed, X_STREAM, kind, self.x_scale, self.x_clip,
                    offset=row0 * self.d, nthreads=nthreads)

    def dy_into(self, out: np.ndarray, row0: int = 0, nthreads: int = 0) -> np.ndarray:
        return fill(out, self.seed, DY_STREAM, KIND_NORMAL, self.dy_scale, 0.0,
                    offset=row0 * self.d, nthreads=nthreads)

    def x(self, nthreads: int = 0) -> np.ndarray:
        return self.x_into(np.empty((self.rows, self.d), np_dtype(self.dtype)), nthreads=nthreads)

    def dy(self, nthreads: int = 0) -> np.ndarray:
        return self.dy_into(np.empty((self.rows, self.d), np_dtype(self.dtype)), nthreads=nthreads)

    def x_at(self, flat_idx: np.ndarray) -> np.ndarray:
        return gather(flat_idx, self.dtype, self.seed, X_STREAM, self.x_kind, self.x_scale,
                      self.x_clip)

    def dy_at(self, flat_idx: np.ndarray) -> np.ndarray:
        return gather(flat_idx, self.dtype, self.seed, DY_STREAM, KIND_NORMAL, self.dy_scale)


def _mk(name, B, N, d, dtype, x_kind, dy_scale, base, lo, hi, n_g=8, x_clip=0.0, note=""):
    return Workload(name=name, B=B, N=N, d=d, n_g=n_g, m=5, n=4, dtype=dtype, x_kind=x_kind,
                    x_scale=1.0, x_clip=x_clip, dy_scale=dy_scale, coef_base=base, coef_lo=lo,
                    coef_hi=hi, note=note)


def workload(name: str, n_g: Optional[int] = None, seed: int = 0) -> Workload:
    """The named workloads. ``stress`` takes n_g in {1, 8, 64} (default 8)."""
    if name == "tiny":
        w = _mk("tiny", 2, 16, 64, F32, KIND_NORMAL, 1.0, "zero", -0.5, 0.5)
    elif name == "kat_t":
        w = _mk("kat_t", 1024, 197, 768, F32, KIND_NORMAL, 1e-2, "identity", -0.1, 0.1,
                note="KAT-T MLP hidden activation, first GR-KAN layer (identity start)")
    elif name == "kat_s":
        w = _mk("kat_s", 1024, 197, 1536, BF16, KIND_NORMAL, 1e-2, "swish", -0.1, 0.1,
                note="KAT-S MLP hidden activation, Swish-start coefficients")
    elif name == "kat_b":
        w = _mk("kat_b", 512, 197, 3072, BF16, KIND_NORMAL, 1e-2, "zero", -0.5, 0.5,
                note="KAT-B MLP hidden activation")
    elif name == "stress":
        g = 8 if n_g is None else n_g
        w = _mk("stress", 256, 197, 3072, F32, KIND_STUDENT3, 1.0, "zero", -1.0, 1.0, n_g=g,
                x_clip=8.0, note="accumulation / group stress")
        w.name = "stress_ng%d" % g
    else:
        raise KeyError(name)
    if n_g is not None and name != "stress":
        w.n_g = n_g
    w.seed = seed
    return w


WORKLOADS = ("tiny", "kat_t", "kat_s", "kat_b", "stress")

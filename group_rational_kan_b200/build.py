"""Build the in-tree CUDA library libgrkan_b200.so for sm_100a with nvcc.

    python -m group_rational_kan_b200.build [--force] [--verbose]

The library is the C ABI of include/grkan.h; it links the CUDA runtime
statically and finds the driver's tensor-map encoder at run time, so it needs
no GPU to build.
"""
import argparse
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libgrkan_b200.so")
SOURCES = [os.path.join(CSRC, "grkan_api.cu")]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc():
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps():
    deps = list(SOURCES) + [os.path.join(INCLUDE, "grkan.h")]
    deps += [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    return deps


def needs_build():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in _deps())


def command(out=LIB, verbose=False, defines=()):
    """nvcc command line; ``defines`` are extra -D settings of the launch-shape
    knobs (GRK_BF16_BWD_WARPS, GRK_BF16_BWD_STAGES, GRK_FWD_WARPS, the store
    paths GRK_F32_FWD_STORE / GRK_BF16_FWD_STORE / GRK_F32_BWD_STORE /
    GRK_BF16_BWD_STORE, ... in csrc/grkan_tma.cuh; GRK_LIN_XFORM_WARPS in
    csrc/grkan_linear.cuh; GRK_DG_STAGES in csrc/grkan_linear_bwd.cuh;
    GRK_LIN_QUAD, GRK_QD_RAW_STAGES, GRK_QD_A_STAGES, GRK_QD_EPI_BUFS in
    csrc/grkan_linear_quad.cuh)."""
    cmd = [_nvcc(), "-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
           "-Xcompiler", "-fvisibility=hidden", "-I", INCLUDE, "-I", CSRC,
           *["-D" + d for d in defines], "-o", out, *SOURCES]
    if verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    return cmd


def build(force=False, verbose=False):
    """Compile the library if a source is newer than it (or force)."""
    if not force and not needs_build():
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    r = subprocess.run(command(tmp, verbose), capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed building libgrkan_b200.so")
    if verbose:
        sys.stderr.write(r.stdout + r.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))

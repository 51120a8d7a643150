"""B200 (sm_100a) GR-KAN group-rational activation: forward, backward dx and
the per-group coefficient gradients dA, dB.

Thin binding over the C ABI of ``include/grkan.h`` (libgrkan_b200.so): the
functions named ``grkan_*`` take the ABI's arguments (torch tensors or raw
integer pointers) and return its status code; ``forward`` / ``backward`` are
conveniences that allocate outputs with torch and raise on error. Every step
of the computation runs in the library's CUDA kernels; there is no CPU path.
PyTorch is used only for device memory and streams.
"""
import ctypes
import os
import threading

__all__ = [
    "GrkanError", "F32", "BF16", "FLAG_GENERIC", "lib", "library_path",
    "grkan_forward", "grkan_forward_ex", "grkan_backward", "grkan_backward_ex",
    "grkan_backward_partials", "grkan_backward_merge", "grkan_backward_workspace_bytes",
    "grkan_merge_ranks", "grkan_backward_noalloc", "NOALLOC_WORKSPACE_BYTES",
    "grkan_step_host", "grkan_step_host_scratch_bytes", "grkan_forward_backward",
    "grkan_backward_atomic", "ATOMIC_PER_ELEMENT", "ATOMIC_PER_BLOCK",
    "grkan_linear_forward", "grkan_linear_forward_path", "linear_forward",
    "grkan_linear_backward", "grkan_linear_backward_workspace_bytes", "linear_backward",
    "forward_backward",
    "grkan_forward_path", "grkan_backward_path", "grkan_device_error", "grkan_clear_device_error",
    "grkan_status_string", "grkan_abi_version", "grkan_last_error", "grkan_selftest_wait_timeout",
    "DEVICE_ERROR_SELFTEST", "forward", "backward", "workspace_bytes",
]

F32, BF16 = 0, 1
FLAG_GENERIC = 1
NOALLOC_WORKSPACE_BYTES = 4 << 20  # GRKAN_NOALLOC_WORKSPACE_BYTES
DEVICE_ERROR_SELFTEST = 16  # GRKAN_DEVICE_ERROR_SELFTEST
ABI_VERSION = 3

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libgrkan_b200.so")
_lib = None
_lock = threading.Lock()


class GrkanError(RuntimeError):
    def __init__(self, status, what=""):
        self.status = status
        msg = grkan_status_string(status)
        if status == 6:  # GRKAN_ERR_CUDA: add the failing CUDA call
            msg += " [%s]" % grkan_last_error()
        super().__init__("%s%s" % (what + ": " if what else "", msg))


def _load():
    from . import build as _build
    if _build.needs_build():
        _build.build()
    if not os.path.exists(library_path):
        raise ImportError("libgrkan_b200.so is missing and could not be built")
    L = ctypes.CDLL(library_path)
    P, I64, I32, U32, SZ = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_uint32,
                            ctypes.c_size_t)
    S = ctypes.c_int  # status enum
    sig = {
        "grkan_forward": (S, [P, P, P, P, I64, I64, I64, I32, I32, I32, ctypes.c_int, P]),
        "grkan_forward_ex": (S, [P, P, P, P, I64, I64, I64, I32, I32, I32, ctypes.c_int, U32, P]),
        "grkan_backward_workspace_bytes": (SZ, [I64, I64, I64, I32, I32, I32, ctypes.c_int]),
        "grkan_backward": (S, [P, P, P, P, P, P, P, I64, I64, I64, I32, I32, I32, ctypes.c_int,
                               P, SZ, P]),
        "grkan_backward_ex": (S, [P, P, P, P, P, P, P, I64, I64, I64, I32, I32, I32,
                                  ctypes.c_int, P, SZ, U32, P]),
        "grkan_backward_partials": (S, [P, P, P, P, P, I64, I64, I64, I32, I32, I32, ctypes.c_int,
                                        P, SZ, U32, P]),
        "grkan_backward_merge": (S, [P, SZ, P, P, P, I64, I64, I64, I32, I32, I32, ctypes.c_int,
                                     P]),
        "grkan_merge_ranks": (S, [P, I32, P, P, I32, I32, I32, P]),
        "grkan_linear_forward": (S, [P, P, P, P, P, P, I64, I64, I64, I32, I32, I32, I64,
                                     ctypes.c_int, P]),
        "grkan_linear_forward_path": (I32, [I64, I64, I64, I32, I32, I32, I64, ctypes.c_int]),
        "grkan_linear_backward_workspace_bytes": (SZ, [I64, I64, I64, I32, I32, I32, I64,
                                                       ctypes.c_int]),
        "grkan_linear_backward": (S, [P, P, P, P, P, P, P, P, I64, I64, I64, I32, I32, I32, I64,
                                      ctypes.c_int, P, SZ, P]),
        "grkan_backward_atomic": (S, [P, P, P, P, P, P, P, I64, I64, I64, I32, I32, I32,
                                      ctypes.c_int, I32, I32, P]),
        "grkan_forward_backward": (S, [P, P, P, P, P, P, P, P, I64, I64, I64, I32, I32, I32,
                                       ctypes.c_int, P, SZ, U32, P]),
        "grkan_step_host_scratch_bytes": (SZ, [I64, I64, I64, I32, I32, I32, ctypes.c_int, I64]),
        "grkan_step_host": (S, [P, P, P, P, P, P, P, P, P, I64, I64, I64, I32, I32, I32,
                                ctypes.c_int, P, SZ, I64, P]),
        "grkan_backward_noalloc": (S, [P, P, P, P, P, P, P, I64, I64, I64, I32, I32, I32,
                                       ctypes.c_int, P]),
        "grkan_forward_path": (I32, [P, P, I64, I64, I64, I32, I32, I32, ctypes.c_int, U32]),
        "grkan_backward_path": (I32, [P, P, P, I64, I64, I64, I32, I32, I32, ctypes.c_int, U32]),
        "grkan_device_error": (S, [P, P]),
        "grkan_clear_device_error": (S, [P]),
        "grkan_selftest_wait_timeout": (S, [U32, P]),
        "grkan_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "grkan_abi_version": (I32, []),
        "grkan_last_error": (ctypes.c_char_p, []),
    }
    L.grkan_abi_version.restype = I32
    L.grkan_abi_version.argtypes = []
    if L.grkan_abi_version() != ABI_VERSION:
        raise ImportError("libgrkan_b200.so ABI %d, binding expects %d" %
                          (L.grkan_abi_version(), ABI_VERSION))
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    return L


def lib():
    """The loaded CUDA library (built in-tree on first use if missing or stale)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                _lib = _load()
    return _lib


# --- argument marshalling ----------------------------------------------------

def _ptr(v):
    if v is None:
        return None
    if isinstance(v, int):
        return v
    return v.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def grkan_forward(x, y, a, b, B, N, d, n_g, m, n, dtype, stream=None):
    return lib().grkan_forward(_ptr(x), _ptr(y), _ptr(a), _ptr(b), B, N, d, n_g, m, n, dtype,
                               _stream(stream))


def grkan_forward_ex(x, y, a, b, B, N, d, n_g, m, n, dtype, flags, stream=None):
    return lib().grkan_forward_ex(_ptr(x), _ptr(y), _ptr(a), _ptr(b), B, N, d, n_g, m, n, dtype,
                                  flags, _stream(stream))


def grkan_backward_workspace_bytes(B, N, d, n_g, m, n, dtype):
    return lib().grkan_backward_workspace_bytes(B, N, d, n_g, m, n, dtype)


def grkan_backward(x, dy, a, b, dx, dA, dB, B, N, d, n_g, m, n, dtype, workspace,
                   workspace_bytes, stream=None):
    return lib().grkan_backward(_ptr(x), _ptr(dy), _ptr(a), _ptr(b), _ptr(dx), _ptr(dA), _ptr(dB),
                                B, N, d, n_g, m, n, dtype, _ptr(workspace), workspace_bytes,
                                _stream(stream))


def grkan_backward_ex(x, dy, a, b, dx, dA, dB, B, N, d, n_g, m, n, dtype, workspace,
                      workspace_bytes, flags, stream=None):
    return lib().grkan_backward_ex(_ptr(x), _ptr(dy), _ptr(a), _ptr(b), _ptr(dx), _ptr(dA),
                                   _ptr(dB), B, N, d, n_g, m, n, dtype, _ptr(workspace),
                                   workspace_bytes, flags, _stream(stream))


def grkan_backward_partials(x, dy, a, b, dx, B, N, d, n_g, m, n, dtype, workspace,
                            workspace_bytes, flags=0, stream=None):
    return lib().grkan_backward_partials(_ptr(x), _ptr(dy), _ptr(a), _ptr(b), _ptr(dx), B, N, d,
                                         n_g, m, n, dtype, _ptr(workspace), workspace_bytes, flags,
                                         _stream(stream))


def grkan_backward_merge(workspace, workspace_bytes, dA, dB, sums64, B, N, d, n_g, m, n, dtype,
                         stream=None):
    return lib().grkan_backward_merge(_ptr(workspace), workspace_bytes, _ptr(dA), _ptr(dB),
                                      _ptr(sums64), B, N, d, n_g, m, n, dtype, _stream(stream))


def grkan_merge_ranks(gathered, world, dA, dB, n_g, m, n, stream=None):
    return lib().grkan_merge_ranks(_ptr(gathered), world, _ptr(dA), _ptr(dB), n_g, m, n,
                                   _stream(stream))


def grkan_backward_noalloc(x, dy, a, b, dx, dA, dB, B, N, d, n_g, m, n, dtype, stream=None):
    """grkan_backward with the library's static scratch array as workspace (for
    callers that cannot allocate device memory per call)."""
    return lib().grkan_backward_noalloc(_ptr(x), _ptr(dy), _ptr(a), _ptr(b), _ptr(dx), _ptr(dA),
                                        _ptr(dB), B, N, d, n_g, m, n, dtype, _stream(stream))


ATOMIC_PER_ELEMENT = 1
ATOMIC_PER_BLOCK = 2


def grkan_linear_forward(x, a, b, W, bias, out, B, N, d, n_g, m, n, nout, dtype, stream=None):
    return lib().grkan_linear_forward(_ptr(x), _ptr(a), _ptr(b), _ptr(W), _ptr(bias), _ptr(out),
                                      B, N, d, n_g, m, n, nout, dtype, _stream(stream))


def grkan_linear_forward_path(B, N, d, n_g, m, n, nout, dtype):
    return lib().grkan_linear_forward_path(B, N, d, n_g, m, n, nout, dtype)


def linear_forward(x, a, b, n_g, W, bias=None, stream=None):
    """GR-KAN followed by a linear layer: (B, N, d) bf16 -> (B, N, nout) bf16."""
    import torch
    B, N, d, dt = _dims(x, n_g)
    m, n = _coef(a, b, n_g)
    nout = W.shape[0]
    out = torch.empty(x.shape[:-1] + (nout,), dtype=x.dtype, device=x.device)
    _check(grkan_linear_forward(x, a, b, W, bias, out, B, N, d, n_g, m, n, nout, dt, stream),
           "grkan_linear_forward")
    return out


def grkan_linear_backward_workspace_bytes(B, N, d, n_g, m, n, nout, dtype):
    return lib().grkan_linear_backward_workspace_bytes(B, N, d, n_g, m, n, nout, dtype)


def grkan_linear_backward(x, dout, W, a, b, dx, dA, dB, B, N, d, n_g, m, n, nout, dtype,
                          workspace, workspace_bytes, stream=None):
    return lib().grkan_linear_backward(_ptr(x), _ptr(dout), _ptr(W), _ptr(a), _ptr(b), _ptr(dx),
                                       _ptr(dA), _ptr(dB), B, N, d, n_g, m, n, nout, dtype,
                                       _ptr(workspace), workspace_bytes, _stream(stream))


def linear_backward(x, dout, W, a, b, n_g, dx=None, dA=None, dB=None, workspace=None,
                    stream=None):
    """(dx, dA, dB) of GR-KAN followed by a linear layer, from the layer output's
    gradient dout (B, N, nout) bf16 and the weight W (nout, d) bf16."""
    import torch
    B, N, d, dt = _dims(x, n_g)
    m, n = _coef(a, b, n_g)
    nout = W.shape[0]
    if dx is None:
        dx = torch.empty_like(x)
    if dA is None:
        dA = torch.empty((n_g, m + 1), dtype=torch.float32, device=x.device)
    if dB is None:
        dB = torch.empty((n_g, n), dtype=torch.float32, device=x.device)
    wsb = grkan_linear_backward_workspace_bytes(B, N, d, n_g, m, n, nout, dt)
    if workspace is None:
        workspace = torch.empty(max(wsb, 16), dtype=torch.uint8, device=x.device)
    _check(grkan_linear_backward(x, dout, W, a, b, dx, dA, dB, B, N, d, n_g, m, n, nout, dt,
                                 workspace, workspace.numel() * workspace.element_size(), stream),
           "grkan_linear_backward")
    return dx, dA, dB


def grkan_backward_atomic(x, dy, a, b, dx, dA, dB, B, N, d, n_g, m, n, dtype, mode, block_rows=0,
                          stream=None):
    return lib().grkan_backward_atomic(_ptr(x), _ptr(dy), _ptr(a), _ptr(b), _ptr(dx), _ptr(dA),
                                       _ptr(dB), B, N, d, n_g, m, n, dtype, mode, block_rows,
                                       _stream(stream))


def grkan_forward_backward(x, dy, a, b, y, dx, dA, dB, B, N, d, n_g, m, n, dtype, workspace,
                           workspace_bytes, flags=0, stream=None):
    return lib().grkan_forward_backward(_ptr(x), _ptr(dy), _ptr(a), _ptr(b), _ptr(y), _ptr(dx),
                                        _ptr(dA), _ptr(dB), B, N, d, n_g, m, n, dtype,
                                        _ptr(workspace), workspace_bytes, flags, _stream(stream))


def grkan_step_host_scratch_bytes(B, N, d, n_g, m, n, dtype, chunk_rows=0):
    return lib().grkan_step_host_scratch_bytes(B, N, d, n_g, m, n, dtype, chunk_rows)


def grkan_step_host(x_host, dy_host, a, b, y_host, dx_host, dA_host, dB_host, sums64, B, N, d,
                    n_g, m, n, dtype, scratch, scratch_bytes, chunk_rows=0, stream=None):
    """Forward + backward of host tensors (pinned torch CPU tensors or raw host
    pointers) streamed through device scratch; dA_host / dB_host are host,
    sums64 (float64 sums for a data-parallel merge) is a device tensor or None."""
    return lib().grkan_step_host(_ptr(x_host), _ptr(dy_host), _ptr(a), _ptr(b), _ptr(y_host),
                                 _ptr(dx_host), _ptr(dA_host), _ptr(dB_host), _ptr(sums64), B, N,
                                 d, n_g, m, n, dtype, _ptr(scratch), scratch_bytes, chunk_rows,
                                 _stream(stream))


def grkan_forward_path(x, y, B, N, d, n_g, m, n, dtype, flags=0):
    return lib().grkan_forward_path(_ptr(x), _ptr(y), B, N, d, n_g, m, n, dtype, flags)


def grkan_backward_path(x, dy, dx, B, N, d, n_g, m, n, dtype, flags=0):
    return lib().grkan_backward_path(_ptr(x), _ptr(dy), _ptr(dx), B, N, d, n_g, m, n, dtype, flags)


def grkan_device_error(stream=None):
    """(status, code): code != 0 means a bounded wait in a kernel ran out."""
    code = ctypes.c_uint32(0)
    st = lib().grkan_device_error(ctypes.addressof(code), _stream(stream))
    return st, int(code.value)


def grkan_selftest_wait_timeout(limit_us, stream=None):
    return lib().grkan_selftest_wait_timeout(limit_us, _stream(stream))


def grkan_clear_device_error(stream=None):
    return lib().grkan_clear_device_error(_stream(stream))


def grkan_status_string(status):
    try:
        return lib().grkan_status_string(int(status)).decode()
    except Exception:  # library not loadable: still describe the code
        return "status %d" % int(status)


def grkan_abi_version():
    return lib().grkan_abi_version()


def grkan_last_error():
    return lib().grkan_last_error().decode()


# --- conveniences (torch tensors in, torch tensors out) ------------------------

def _check(st, what):
    if st != 0:
        raise GrkanError(st, what)


def _dims(x, n_g):
    import torch
    if x.dtype == torch.float32:
        dt = F32
    elif x.dtype == torch.bfloat16:
        dt = BF16
    else:
        raise TypeError("x must be float32 or bfloat16, got %s" % x.dtype)
    if not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous CUDA tensor")
    if x.dim() == 3:
        B, N, d = x.shape
    elif x.dim() == 2:
        (B, d), N = x.shape, 1
    else:
        raise ValueError("x must be (B, N, d) or (rows, d)")
    return int(B), int(N), int(d), dt


def _coef(a, b, n_g):
    m = a.shape[-1] - 1
    n = b.shape[-1] if b is not None else 0
    return m, n


def workspace_bytes(x, a, b, n_g):
    B, N, d, dt = _dims(x, n_g)
    m, n = _coef(a, b, n_g)
    return grkan_backward_workspace_bytes(B, N, d, n_g, m, n, dt)


def forward(x, a, b, n_g, out=None, flags=0, stream=None):
    """y = P(x) / (1 + |Q(x)|) with per-group coefficients a (n_g, m+1), b (n_g, n)."""
    import torch
    B, N, d, dt = _dims(x, n_g)
    m, n = _coef(a, b, n_g)
    y = torch.empty_like(x) if out is None else out
    _check(grkan_forward_ex(x, y, a, b, B, N, d, n_g, m, n, dt, flags, stream), "grkan_forward")
    return y


def backward(x, dy, a, b, n_g, dx=None, dA=None, dB=None, workspace=None, flags=0, stream=None):
    """(dx, dA, dB) for upstream gradient dy. dA, dB are float32 (n_g, m+1), (n_g, n)."""
    import torch
    B, N, d, dt = _dims(x, n_g)
    m, n = _coef(a, b, n_g)
    if dx is None:
        dx = torch.empty_like(x)
    if dA is None:
        dA = torch.empty((n_g, m + 1), dtype=torch.float32, device=x.device)
    if dB is None:
        dB = torch.empty((n_g, n), dtype=torch.float32, device=x.device)
    wsb = grkan_backward_workspace_bytes(B, N, d, n_g, m, n, dt)
    if workspace is None:
        workspace = torch.empty(max(wsb, 16), dtype=torch.uint8, device=x.device)
    _check(grkan_backward_ex(x, dy, a, b, dx, dA, dB, B, N, d, n_g, m, n, dt, workspace,
                             workspace.numel() * workspace.element_size(), flags, stream),
           "grkan_backward")
    return dx, dA, dB


def forward_backward(x, dy, a, b, n_g, flags=0, stream=None):
    """(y, dx, dA, dB) in one pass (recompute mode)."""
    import torch
    B, N, d, dt = _dims(x, n_g)
    m, n = _coef(a, b, n_g)
    y = torch.empty_like(x)
    dx = torch.empty_like(x)
    dA = torch.empty((n_g, m + 1), dtype=torch.float32, device=x.device)
    dB = torch.empty((n_g, n), dtype=torch.float32, device=x.device)
    wsb = grkan_backward_workspace_bytes(B, N, d, n_g, m, n, dt)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=x.device)
    _check(grkan_forward_backward(x, dy, a, b, y, dx, dA, dB, B, N, d, n_g, m, n, dt, ws,
                                  ws.numel(), flags, stream), "grkan_forward_backward")
    return y, dx, dA, dB

"""BitLinear W1.58·A8 matmul (BitNet b1.58) for NVIDIA B200.

Thin binding over ``libbitlinear.so`` (C ABI in ``include/bitlinear.h``).  The
functions here only marshal arguments: torch tensors supply device pointers
and the current CUDA stream, every step of the path runs in the library's
kernels, and a missing library raises instead of falling back to anything.

Names match the C ABI: :func:`bitlinear_quantize_weights`,
:func:`bitlinear_quantize_act`, :func:`bitlinear_forward` and the grouped
variants.  ``lib()`` returns the raw ctypes handle for pointer-level callers.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbitlinear.so")
LIB_PATH = os.environ.get("BITLINEAR_LIB", LIB_PATH)  # a build elsewhere (same ABI)
MAX_GROUP = 16
MAX_K = 1 << 20

BL_F32, BL_BF16 = 0, 1
STATUS = {
    0: "BL_OK", 1: "BL_ERR_NULL", 2: "BL_ERR_SHAPE", 3: "BL_ERR_ALIGN", 4: "BL_ERR_DTYPE",
    5: "BL_ERR_WORKSPACE", 6: "BL_ERR_ARCH", 7: "BL_ERR_CUDA", 8: "BL_ERR_COUNT", 9: "BL_ERR_TIMEOUT",
    10: "BL_ERR_FLAGS",
}
BL_LINEAR_WEIGHTS_STATIC = 1

_lock = threading.Lock()
_lib = None


class BitLinearError(RuntimeError):
    def __init__(self, status: int, call: str, msg: str):
        super().__init__(f"{call}: {STATUS.get(status, status)} ({msg})")
        self.status = status


class ActProblem(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("x_q", ctypes.c_void_p), ("beta", ctypes.c_void_p),
                ("M", ctypes.c_int64), ("K", ctypes.c_int64)]


class ForwardProblem(ctypes.Structure):
    _fields_ = [("x_q", ctypes.c_void_p), ("beta", ctypes.c_void_p), ("W_packed", ctypes.c_void_p),
                ("alpha", ctypes.c_void_p), ("bias", ctypes.c_void_p), ("y", ctypes.c_void_p),
                ("acc_out", ctypes.c_void_p), ("M", ctypes.c_int64), ("N", ctypes.c_int64),
                ("K", ctypes.c_int64)]


class LinearProblem(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("x_q", ctypes.c_void_p), ("beta", ctypes.c_void_p),
                ("W_packed", ctypes.c_void_p), ("alpha", ctypes.c_void_p), ("bias", ctypes.c_void_p),
                ("y", ctypes.c_void_p), ("acc_out", ctypes.c_void_p), ("M", ctypes.c_int64),
                ("N", ctypes.c_int64), ("K", ctypes.c_int64)]


class ActSumProblem(ctypes.Structure):
    _fields_ = [("a", ctypes.c_void_p), ("b", ctypes.c_void_p), ("x_sum", ctypes.c_void_p), ("x_q", ctypes.c_void_p),
                ("beta", ctypes.c_void_p), ("M", ctypes.c_int64), ("K", ctypes.c_int64)]


def lib():
    """The loaded ctypes library; raises if the CUDA library was not built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"{LIB_PATH} is missing: build it with "
                                  "`python -m bitlinear_w1_a8_03_b200.build` (there is no CPU fallback)")
            L = ctypes.CDLL(LIB_PATH)
            p, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
            L.bitlinear_packed_row_bytes.argtypes = [i64]
            L.bitlinear_packed_row_bytes.restype = sz
            L.bitlinear_quantize_weights_workspace_bytes.argtypes = [i64, i64]
            L.bitlinear_quantize_weights_workspace_bytes.restype = sz
            L.bitlinear_quantize_weights.argtypes = [p, i32, i64, i64, p, p, p, sz, p]
            L.bitlinear_quantize_weights_static.argtypes = [p, i32, i64, i64, p, p, p]
            L.bitlinear_quantize_act.argtypes = [p, i32, i64, i64, p, p, p]
            L.bitlinear_forward.argtypes = [p, p, i64, i64, p, p, i64, p, p, p, p]
            L.bitlinear_quantize_act_grouped.argtypes = [ctypes.POINTER(ActProblem), i32, i32, p]
            L.bitlinear_forward_grouped.argtypes = [ctypes.POINTER(ForwardProblem), i32, p]
            L.bitlinear_linear.argtypes = [p, i32, i64, i64, p, p, i64, p, p, p, p, p, p]
            L.bitlinear_linear_grouped.argtypes = [ctypes.POINTER(LinearProblem), i32, i32, ctypes.c_uint32, p]
            L.bitlinear_linear_block.argtypes = [ctypes.POINTER(ActSumProblem), i32, ctypes.POINTER(ForwardProblem), i32,
                                                 ctypes.c_uint32, p]
            L.bitlinear_device_error.argtypes = [ctypes.POINTER(ctypes.c_int)]
            L.bitlinear_selftest_timeout.argtypes = [ctypes.c_uint32, p]
            L.bitlinear_status_string.argtypes = [i32]
            L.bitlinear_status_string.restype = ctypes.c_char_p
            L.bitlinear_version.argtypes = []
            for name in ("bitlinear_quantize_weights", "bitlinear_quantize_weights_static",
                         "bitlinear_quantize_act", "bitlinear_forward",
                         "bitlinear_quantize_act_grouped", "bitlinear_forward_grouped", "bitlinear_linear",
                         "bitlinear_linear_grouped", "bitlinear_linear_block", "bitlinear_device_error",
                         "bitlinear_selftest_timeout",
                         "bitlinear_version"):
                getattr(L, name).restype = i32
            _lib = L
    return _lib


def check(status: int, call: str) -> None:
    if status != 0:
        raise BitLinearError(status, call, lib().bitlinear_status_string(status).decode())


# ------------------------------------------------------------------ torch helpers
def _torch():
    import torch
    return torch


def _stream(stream=None) -> int:
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float32:
        return BL_F32
    if t.dtype == torch.bfloat16:
        return BL_BF16
    raise TypeError(f"expected float32 or bfloat16, got {t.dtype}")


def _need(t, name):
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")


def packed_row_bytes(K: int) -> int:
    return int(lib().bitlinear_packed_row_bytes(K))


def bitlinear_quantize_weights(W, W_packed=None, alpha=None, workspace=None, stream=None):
    """W [N][K] (fp32/bf16, CUDA) -> (W_packed uint8 [N][16·ceil(K/64)], alpha float32 [1])."""
    torch = _torch()
    _need(W, "W")
    N, K = W.shape
    if W_packed is None:
        W_packed = torch.empty((N, packed_row_bytes(K)), dtype=torch.uint8, device=W.device)
    if alpha is None:
        alpha = torch.empty(1, dtype=torch.float32, device=W.device)
    ws = int(lib().bitlinear_quantize_weights_workspace_bytes(N, K))
    if workspace is None:
        workspace = torch.empty(max(ws, 8), dtype=torch.uint8, device=W.device)
    check(lib().bitlinear_quantize_weights(_ptr(W), _dtype_code(W), N, K, _ptr(W_packed), _ptr(alpha),
                                           _ptr(workspace), workspace.numel() * workspace.element_size(),
                                           _stream(stream)), "bitlinear_quantize_weights")
    return W_packed, alpha


def bitlinear_quantize_act(x, x_q=None, beta=None, stream=None):
    """x [M][K] (fp32/bf16, CUDA) -> (x_q int8 [M][K], beta float32 [M])."""
    torch = _torch()
    _need(x, "x")
    M, K = x.shape
    if x_q is None:
        x_q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if beta is None:
        beta = torch.empty(M, dtype=torch.float32, device=x.device)
    check(lib().bitlinear_quantize_act(_ptr(x), _dtype_code(x), M, K, _ptr(x_q), _ptr(beta), _stream(stream)),
          "bitlinear_quantize_act")
    return x_q, beta


def bitlinear_forward(x_q, beta, W_packed, alpha, N: int, bias=None, y=None, acc_out=None, stream=None):
    """y [M][N] float32 = (x̃·Ŵᵀ)·(α·β/127) (+ bias); optional int32 accumulators."""
    torch = _torch()
    M, K = x_q.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=x_q.device)
    check(lib().bitlinear_forward(_ptr(x_q), _ptr(beta), M, K, _ptr(W_packed), _ptr(alpha), N, _ptr(bias),
                                  _ptr(y), _ptr(acc_out), _stream(stream)), "bitlinear_forward")
    return y


def bitlinear_quantize_act_grouped(xs, outs, stream=None):
    """Quantise several activation tensors of one dtype in one launch.
    ``outs`` is a list of (x_q, beta) pairs matching ``xs``."""
    arr = (ActProblem * len(xs))()
    for i, (x, (xq, b)) in enumerate(zip(xs, outs)):
        arr[i] = ActProblem(_ptr(x), _ptr(xq), _ptr(b), x.shape[0], x.shape[1])
    check(lib().bitlinear_quantize_act_grouped(arr, len(xs), _dtype_code(xs[0]), _stream(stream)),
          "bitlinear_quantize_act_grouped")


def make_forward_problems(problems):
    """ctypes array for bitlinear_forward_grouped from dicts with keys
    x_q, beta, W_packed, alpha, N, y and optional bias, acc_out."""
    arr = (ForwardProblem * len(problems))()
    for i, p in enumerate(problems):
        M, K = p["x_q"].shape
        arr[i] = ForwardProblem(_ptr(p["x_q"]), _ptr(p["beta"]), _ptr(p["W_packed"]), _ptr(p["alpha"]),
                                _ptr(p.get("bias")), _ptr(p["y"]), _ptr(p.get("acc_out")), M, p["N"], K)
    return arr


def bitlinear_forward_grouped(problems, stream=None):
    """Several independent forwards in one launch (see make_forward_problems)."""
    arr = problems if isinstance(problems, ctypes.Array) else make_forward_problems(problems)
    check(lib().bitlinear_forward_grouped(arr, len(arr), _stream(stream)), "bitlinear_forward_grouped")


def bitlinear_linear(x, W_packed, alpha, N: int, bias=None, x_q=None, beta=None, y=None, acc_out=None, stream=None):
    """Quantise x and multiply in one call (two overlapped kernels); returns y."""
    torch = _torch()
    _need(x, "x")
    M, K = x.shape
    if x_q is None:
        x_q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if beta is None:
        beta = torch.empty(M, dtype=torch.float32, device=x.device)
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=x.device)
    check(lib().bitlinear_linear(_ptr(x), _dtype_code(x), M, K, _ptr(W_packed), _ptr(alpha), N, _ptr(bias),
                                 _ptr(x_q), _ptr(beta), _ptr(y), _ptr(acc_out), _stream(stream)), "bitlinear_linear")
    return y


def make_linear_problems(problems):
    """ctypes array for bitlinear_linear_grouped from dicts with keys
    x, x_q, beta, W_packed, alpha, N, y and optional bias, acc_out."""
    arr = (LinearProblem * len(problems))()
    for i, p in enumerate(problems):
        M, K = p["x"].shape
        arr[i] = LinearProblem(_ptr(p["x"]), _ptr(p["x_q"]), _ptr(p["beta"]), _ptr(p["W_packed"]), _ptr(p["alpha"]),
                               _ptr(p.get("bias")), _ptr(p["y"]), _ptr(p.get("acc_out")), M, p["N"], K)
    return arr


def bitlinear_linear_grouped(problems, dtype_code: int | None = None, flags: int = 0, stream=None):
    """Several independent linears in one grouped quantisation + one grouped
    product.  flags=BL_LINEAR_WEIGHTS_STATIC: no work in flight writes the weights."""
    if isinstance(problems, ctypes.Array):
        arr = problems
        assert dtype_code is not None
    else:
        arr = make_linear_problems(problems)
        dtype_code = _dtype_code(problems[0]["x"]) if dtype_code is None else dtype_code
    check(lib().bitlinear_linear_grouped(arr, len(arr), dtype_code, flags, _stream(stream)),
          "bitlinear_linear_grouped")


def make_act_sum_problems(acts):
    """ctypes array for bitlinear_linear_block from dicts with keys a, x_q, beta
    and optional b (second float32 addend) and x_sum (stores a + b)."""
    arr = (ActSumProblem * len(acts))()
    for i, p in enumerate(acts):
        M, K = p["a"].shape
        arr[i] = ActSumProblem(_ptr(p["a"]), _ptr(p.get("b")), _ptr(p.get("x_sum")), _ptr(p["x_q"]), _ptr(p["beta"]),
                               M, K)
    return arr


def bitlinear_linear_block(acts, fwds, flags: int = 0, stream=None):
    """Quantise the inputs `acts` (each a, or a + b, float32) in one launch, then
    run the products `fwds` (dicts as for make_forward_problems) in one launch.
    Either may be empty; ctypes arrays from make_act_sum_problems /
    make_forward_problems are passed through as they are."""
    a_arr = acts if isinstance(acts, ctypes.Array) else (make_act_sum_problems(acts) if acts else None)
    f_arr = fwds if isinstance(fwds, ctypes.Array) else (make_forward_problems(fwds) if fwds else None)
    check(lib().bitlinear_linear_block(a_arr, len(acts), f_arr, len(fwds), flags, _stream(stream)),
          "bitlinear_linear_block")


def bitlinear_device_error() -> int:
    """Read and clear the device error word (0 = none)."""
    code = ctypes.c_int(0)
    check(lib().bitlinear_device_error(ctypes.byref(code)), "bitlinear_device_error")
    return code.value

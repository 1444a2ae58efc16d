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
BL_LINEAR_HADAMARD = 2

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


class HostIO(ctypes.Structure):
    _fields_ = [("x_host", ctypes.c_void_p), ("y_host", ctypes.c_void_p)]


class LinearProblem(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("x_q", ctypes.c_void_p), ("beta", ctypes.c_void_p),
                ("W_packed", ctypes.c_void_p), ("alpha", ctypes.c_void_p), ("bias", ctypes.c_void_p),
                ("y", ctypes.c_void_p), ("acc_out", ctypes.c_void_p), ("M", ctypes.c_int64),
                ("N", ctypes.c_int64), ("K", ctypes.c_int64)]


class ScaledProblem(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("x_q", ctypes.c_void_p), ("beta", ctypes.c_void_p),
                ("W_packed", ctypes.c_void_p), ("alpha", ctypes.c_void_p), ("bias", ctypes.c_void_p),
                ("y", ctypes.c_void_p), ("acc_out", ctypes.c_void_p), ("M", ctypes.c_int64), ("N", ctypes.c_int64),
                ("K", ctypes.c_int64), ("group", ctypes.c_int64)]


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
            L.bitlinear_linear_grouped_host.argtypes = [ctypes.POINTER(LinearProblem), ctypes.POINTER(HostIO), i32,
                                                        i32, ctypes.c_uint32, p]
            L.bitlinear_linear_block.argtypes = [ctypes.POINTER(ActSumProblem), i32, ctypes.POINTER(ForwardProblem), i32,
                                                 ctypes.c_uint32, p]
            L.bitlinear_hadamard_block.argtypes = [i64]
            L.bitlinear_hadamard_block.restype = i64
            L.bitlinear_hadamard.argtypes = [p, i32, i64, i64, i64, ctypes.c_float, p, p]
            L.bitlinear_quantize_act_hadamard.argtypes = [p, i32, i64, i64, i64, p, p, p]
            L.bitlinear_quantize_weights_scaled.argtypes = [p, i32, i64, i64, i64, p, p, p]
            L.bitlinear_linear_scaled.argtypes = [ctypes.POINTER(ScaledProblem), i32, i32, ctypes.c_uint32, p]
            L.bitlinear_quantize_act_a4.argtypes = [p, i32, i64, i64, p, p, p]
            L.bitlinear_forward_a4.argtypes = [p, p, i64, i64, p, p, i64, p, p, p, p]
            L.bitlinear_linear_a4.argtypes = [ctypes.POINTER(LinearProblem), i32, i32, ctypes.c_uint32, p]
            L.bitlinear_train_forward.argtypes = [p, i32, i64, i64, p, i32, i64, p, p, p, p, p, p, sz, p]
            L.bitlinear_ste_backward.argtypes = [p, i64, i64, i64, p, p, p, p, p, i32, p, p, p]
            L.bitlinear_device_error.argtypes = [ctypes.POINTER(ctypes.c_int)]
            L.bitlinear_selftest_timeout.argtypes = [ctypes.c_uint32, p]
            L.bitlinear_status_string.argtypes = [i32]
            L.bitlinear_status_string.restype = ctypes.c_char_p
            L.bitlinear_version.argtypes = []
            for name in ("bitlinear_quantize_weights", "bitlinear_quantize_weights_static",
                         "bitlinear_quantize_act", "bitlinear_forward",
                         "bitlinear_quantize_act_grouped", "bitlinear_forward_grouped", "bitlinear_linear",
                         "bitlinear_linear_grouped", "bitlinear_linear_block", "bitlinear_device_error",
                         "bitlinear_selftest_timeout", "bitlinear_hadamard", "bitlinear_quantize_act_hadamard",
                         "bitlinear_quantize_weights_scaled", "bitlinear_linear_scaled",
                         "bitlinear_quantize_act_a4", "bitlinear_forward_a4", "bitlinear_linear_a4",
                         "bitlinear_train_forward", "bitlinear_ste_backward",
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


def make_host_io(pairs):
    """ctypes array for bitlinear_linear_grouped_host from (x_host, y_host)
    pairs of CPU tensors (pinned for asynchronous copies)."""
    arr = (HostIO * len(pairs))()
    for i, (xh, yh) in enumerate(pairs):
        arr[i] = HostIO(xh.data_ptr(), yh.data_ptr())
    return arr


def bitlinear_linear_grouped_host(problems, io, dtype_code: int, flags: int = 0, stream=None):
    """bitlinear_linear_grouped with x copied from and y copied to host memory
    on the stream (ctypes arrays from make_linear_problems and make_host_io)."""
    check(lib().bitlinear_linear_grouped_host(problems, io, len(problems), dtype_code, flags, _stream(stream)),
          "bitlinear_linear_grouped_host")


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


# ------------------------------------------------------------------ rotation
def hadamard_block(K: int) -> int:
    """The block a BL_LINEAR_HADAMARD linear uses for K input features."""
    return int(lib().bitlinear_hadamard_block(K))


def bitlinear_hadamard(x, block: int, scale: float = 1.0, out=None, stream=None):
    """(x·H)·scale per row in float32 (H block-diagonal Sylvester Hadamard)."""
    torch = _torch()
    _need(x, "x")
    M, K = x.shape
    if out is None:
        out = torch.empty((M, K), dtype=torch.float32, device=x.device)
    check(lib().bitlinear_hadamard(_ptr(x), _dtype_code(x), M, K, block, scale, _ptr(out), _stream(stream)),
          "bitlinear_hadamard")
    return out


def bitlinear_quantize_act_hadamard(x, block: int, x_q=None, beta=None, stream=None):
    """Per-token int8 quantisation of x·H: (x_q int8 [M][K], beta float32 [M])."""
    torch = _torch()
    _need(x, "x")
    M, K = x.shape
    if x_q is None:
        x_q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if beta is None:
        beta = torch.empty(M, dtype=torch.float32, device=x.device)
    check(lib().bitlinear_quantize_act_hadamard(_ptr(x), _dtype_code(x), M, K, block, _ptr(x_q), _ptr(beta),
                                                _stream(stream)), "bitlinear_quantize_act_hadamard")
    return x_q, beta


def bitlinear_quantize_weights_rotated(W, block: int | None = None, stream=None):
    """Weights of a rotated layer: W' = W·H/block (float32, on the device), then
    the absmean quantisation of W'.  Returns (W_packed, alpha)."""
    K = W.shape[1]
    block = hadamard_block(K) if block is None else block
    Wr = bitlinear_hadamard(W, block, 1.0 / block, stream=stream)
    out = bitlinear_quantize_weights(Wr, stream=stream)
    del Wr
    return out


# ------------------------------------------------------------------ scale granularity
def bitlinear_quantize_weights_scaled(W, group: int, W_packed=None, alpha=None, stream=None):
    """One α per group of `group` input features of each row (group >= K: per
    row).  Returns (W_packed uint8 [N][16·ceil(K/64)], alpha float32 [N][G])."""
    torch = _torch()
    _need(W, "W")
    N, K = W.shape
    G = 1 if group >= K else -(-K // group)
    if W_packed is None:
        W_packed = torch.empty((N, packed_row_bytes(K)), dtype=torch.uint8, device=W.device)
    if alpha is None:
        alpha = torch.empty((N, G), dtype=torch.float32, device=W.device)
    check(lib().bitlinear_quantize_weights_scaled(_ptr(W), _dtype_code(W), N, K, group, _ptr(W_packed), _ptr(alpha),
                                                  _stream(stream)), "bitlinear_quantize_weights_scaled")
    return W_packed, alpha


def make_scaled_problems(problems):
    """ctypes array for bitlinear_linear_scaled from dicts with keys x_q, beta,
    W_packed, alpha, group, N, y and optional x, bias, acc_out."""
    arr = (ScaledProblem * len(problems))()
    for i, p in enumerate(problems):
        M, K = p["x_q"].shape
        arr[i] = ScaledProblem(_ptr(p.get("x")), _ptr(p["x_q"]), _ptr(p["beta"]), _ptr(p["W_packed"]),
                               _ptr(p["alpha"]), _ptr(p.get("bias")), _ptr(p["y"]), _ptr(p.get("acc_out")), M, p["N"],
                               K, p["group"])
    return arr


def bitlinear_linear_scaled(problems, dtype_code: int = BL_BF16, flags: int = 0, stream=None):
    """Linears with one α per group (see make_scaled_problems)."""
    arr = problems if isinstance(problems, ctypes.Array) else make_scaled_problems(problems)
    check(lib().bitlinear_linear_scaled(arr, len(arr), dtype_code, flags, _stream(stream)), "bitlinear_linear_scaled")


# ------------------------------------------------------------------ 4-bit activations
def bitlinear_quantize_act_a4(x, x_q4=None, beta=None, stream=None):
    """x [M][K] -> (x_q4 uint8 [M][ceil(K/2)] packed 4-bit, beta float32 [M])."""
    torch = _torch()
    _need(x, "x")
    M, K = x.shape
    if x_q4 is None:
        x_q4 = torch.empty((M, (K + 1) // 2), dtype=torch.uint8, device=x.device)
    if beta is None:
        beta = torch.empty(M, dtype=torch.float32, device=x.device)
    check(lib().bitlinear_quantize_act_a4(_ptr(x), _dtype_code(x), M, K, _ptr(x_q4), _ptr(beta), _stream(stream)),
          "bitlinear_quantize_act_a4")
    return x_q4, beta


def bitlinear_forward_a4(x_q4, beta, K: int, W_packed, alpha, N: int, bias=None, y=None, acc_out=None, stream=None):
    """y [M][N] = fp32(x̃·Ŵᵀ)·(α·β/7) (+ bias) on packed 4-bit activations."""
    torch = _torch()
    M = x_q4.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=x_q4.device)
    check(lib().bitlinear_forward_a4(_ptr(x_q4), _ptr(beta), M, K, _ptr(W_packed), _ptr(alpha), N, _ptr(bias), _ptr(y),
                                     _ptr(acc_out), _stream(stream)), "bitlinear_forward_a4")
    return y


def make_linear_a4_problems(problems):
    """ctypes array for bitlinear_linear_a4: dicts as for make_linear_problems,
    with x_q a packed uint8 [M][ceil(K/2)] buffer."""
    arr = (LinearProblem * len(problems))()
    for i, p in enumerate(problems):
        M, K = p["x"].shape
        arr[i] = LinearProblem(_ptr(p["x"]), _ptr(p["x_q"]), _ptr(p["beta"]), _ptr(p["W_packed"]), _ptr(p["alpha"]),
                               _ptr(p.get("bias")), _ptr(p["y"]), _ptr(p.get("acc_out")), M, p["N"], K)
    return arr


def bitlinear_linear_a4(problems, dtype_code: int = BL_BF16, flags: int = 0, stream=None):
    arr = problems if isinstance(problems, ctypes.Array) else make_linear_a4_problems(problems)
    check(lib().bitlinear_linear_a4(arr, len(arr), dtype_code, flags, _stream(stream)), "bitlinear_linear_a4")


# ------------------------------------------------------------------ training (straight-through estimator)
def bitlinear_train_forward(W, x, W_packed=None, alpha=None, x_q=None, beta=None, y=None, workspace=None, stream=None):
    """Forward of a training step on latent weights W [N][K]: quantise W, then
    the linear on x [M][K].  Returns (y, W_packed, alpha, x_q, beta)."""
    torch = _torch()
    _need(W, "W")
    _need(x, "x")
    N, K = W.shape
    M = x.shape[0]
    dev = W.device
    W_packed = torch.empty((N, packed_row_bytes(K)), dtype=torch.uint8, device=dev) if W_packed is None else W_packed
    alpha = torch.empty(1, dtype=torch.float32, device=dev) if alpha is None else alpha
    x_q = torch.empty((M, K), dtype=torch.int8, device=dev) if x_q is None else x_q
    beta = torch.empty(M, dtype=torch.float32, device=dev) if beta is None else beta
    y = torch.empty((M, N), dtype=torch.float32, device=dev) if y is None else y
    ws = int(lib().bitlinear_quantize_weights_workspace_bytes(N, K))
    if workspace is None:
        workspace = torch.empty(max(ws, 8), dtype=torch.uint8, device=dev)
    check(lib().bitlinear_train_forward(_ptr(W), _dtype_code(W), N, K, _ptr(x), _dtype_code(x), M, _ptr(W_packed),
                                        _ptr(alpha), _ptr(x_q), _ptr(beta), _ptr(y), _ptr(workspace),
                                        workspace.numel(), _stream(stream)), "bitlinear_train_forward")
    return y, W_packed, alpha, x_q, beta


def bitlinear_ste_backward(g, W_packed, alpha, x_q, beta, W, grad_x=True, grad_W=True, stream=None):
    """Straight-through backward for g = ∂L/∂y [M][N]: returns (grad_x [M][K] or
    None, grad_W [N][K] or None)."""
    torch = _torch()
    M, N = g.shape
    K = W.shape[1]
    gx = torch.empty((M, K), dtype=torch.float32, device=g.device) if grad_x is True else (grad_x or None)
    gw = torch.empty((N, K), dtype=torch.float32, device=g.device) if grad_W is True else (grad_W or None)
    check(lib().bitlinear_ste_backward(_ptr(g), M, N, K, _ptr(W_packed), _ptr(alpha), _ptr(x_q), _ptr(beta), _ptr(W),
                                       _dtype_code(W), _ptr(gx), _ptr(gw), _stream(stream)), "bitlinear_ste_backward")
    return gx, gw

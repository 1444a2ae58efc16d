"""CPU oracle for the BitLinear W1.58·A8 matmul (ctypes + numpy over plain C).

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``, the smoke check in
``__graft_entry__`` and the benchmark's CPU-baseline / reference arm may import
this package.  It shares no code with the CUDA library and never imports it.

Pinned functions (the pins live in ``tests/test_oracle_pins.py``, for the
layer stack ``tests/test_oracle_stack.py``, and for the rotation, the finer
scale granularities and the 4-bit activations ``tests/test_oracle_variants.py``):
``absmean``, ``ternarize``, ``pack``, ``quantize_act``, ``ternary_matmul``,
``dequant``, ``forward``, ``stack_layer``, ``stack_forward``, ``hadamard``,
``hadamard_block``, ``quantize_weights_rotated``, ``quantize_act_rotated``,
``absmean_groups``, ``ternarize_groups``, ``forward_groups``,
``quantize_act_a4``, ``unpack_a4``, ``dequant_a4``, ``forward_a4``,
``ste_grad_x``, ``ste_grad_w`` (pins in ``tests/test_oracle_train.py``).  No
function here is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bitlinear_oracle.c")
_HDR = os.path.join(_HERE, "bitlinear_oracle.h")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

F32, BF16 = 0, 1
CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no GPU involved); returns the library path."""
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def configure(lib):
    """Declare the C signatures on a loaded oracle library."""
    p, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
    lib.orc_abs_exponent_bins.argtypes = [p, i32, i64, p]
    lib.orc_ternarize.argtypes = [p, i32, i64, f32, p]
    lib.orc_packed_row_bytes.argtypes = [i64]
    lib.orc_packed_row_bytes.restype = i64
    lib.orc_pack.argtypes = [p, i64, i64, p]
    lib.orc_pack.restype = None
    lib.orc_quantize_act.argtypes = [p, i32, i64, i64, p, p]
    lib.orc_ternary_matmul.argtypes = [p, p, i64, i64, i64, p, i32]
    lib.orc_dequant.argtypes = [p, p, f32, p, i64, i64, p]
    lib.orc_dequant.restype = None
    lib.orc_forward.argtypes = [p, i32, i64, i64, p, f32, p, i64, p, p, p, p, i32]
    lib.orc_hadamard.argtypes = [p, i32, i64, i64, i64, f32, p]
    lib.orc_absmean_groups.argtypes = [p, i32, i64, i64, i64, p]
    lib.orc_ternarize_groups.argtypes = [p, i32, i64, i64, i64, p, p]
    lib.orc_forward_groups.argtypes = [p, p, i64, i64, p, p, i64, p, i64, p, i32]
    lib.orc_quantize_act_a4.argtypes = [p, i32, i64, i64, p, p]
    lib.orc_unpack_a4.argtypes = [p, i64, i64, p]
    lib.orc_unpack_a4.restype = None
    lib.orc_dequant_a4.argtypes = [p, p, f32, p, i64, i64, p]
    lib.orc_dequant_a4.restype = None
    lib.orc_ste_grad_x.argtypes = [p, i64, i64, p, i64, f32, p, i32]
    lib.orc_ste_grad_w.argtypes = [p, i64, i64, p, p, i64, p, i32, f32, p, i32]
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = configure(ctypes.CDLL(build()))
    return _lib


def _ptr(a: np.ndarray | None):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _as_input(a: np.ndarray):
    """float32 array, or bfloat16 given as its uint16 bit pattern."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.float32:
        return a, F32
    if a.dtype == np.uint16:
        return a, BF16
    raise TypeError(f"oracle inputs are float32 or bf16 bits (uint16), got {a.dtype}")


def packed_row_bytes(K: int) -> int:
    return int(_load().orc_packed_row_bytes(K))


def absmean(W: np.ndarray) -> np.float32:
    """α = mean(|W|) of the whole tensor ([BitNet 三值权重实战] §2.3).

    The sum of |W| is exact (integer bins per binary32 exponent); the mean is
    rounded once to binary64 (Python's int/int true division is correctly
    rounded) and then to binary32: α = RN32(RN64(Σ|W| / count)).
    """
    W, dt = _as_input(W)
    if W.size == 0:
        raise ValueError("empty weight tensor")
    bins = np.zeros(256, dtype=np.int64)
    if _load().orc_abs_exponent_bins(_ptr(W), dt, W.size, _ptr(bins)) != 0:
        raise ValueError("non-finite weight")
    # |w| = sig * 2^(max(E,1) - 150), so 2^149 * Σ|w| = Σ bins[E] << (max(E,1) - 1)
    scaled = sum(int(b) << (max(e, 1) - 1) for e, b in enumerate(bins.tolist()) if b)
    return np.float32(scaled / (W.size << 149))


def ternarize(W: np.ndarray, alpha) -> np.ndarray:
    """Codes ŵ = clip(round(W/α), -1, 1) as int8, same shape as W (§2.3, §4.1)."""
    W, dt = _as_input(W)
    out = np.empty(W.shape, dtype=np.int8)
    _load().orc_ternarize(_ptr(W), dt, W.size, ctypes.c_float(float(np.float32(alpha))), _ptr(out))
    return out


def pack(codes: np.ndarray) -> np.ndarray:
    """2-bit packed rows [N][16·ceil(K/64)] uint8 of int8 codes [N][K]."""
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    N, K = codes.shape
    out = np.empty((N, packed_row_bytes(K)), dtype=np.uint8)
    _load().orc_pack(_ptr(codes), N, K, _ptr(out))
    return out


def quantize_weights(W: np.ndarray):
    """(packed, α, codes) for a weight matrix [N][K]."""
    alpha = absmean(W)
    codes = ternarize(W, alpha)
    return pack(codes), alpha, codes


def quantize_act(x: np.ndarray):
    """(x̃ int8 [M][K], β float32 [M]) per token (§2.4, §4.1)."""
    x, dt = _as_input(x)
    M, K = x.shape
    xq = np.empty((M, K), dtype=np.int8)
    beta = np.empty(M, dtype=np.float32)
    _load().orc_quantize_act(_ptr(x), dt, M, K, _ptr(xq), _ptr(beta))
    return xq, beta


def ternary_matmul(xq: np.ndarray, codes: np.ndarray, threads: int = 1) -> np.ndarray:
    """int32 acc[M][N] = x̃·Ŵᵀ by add / subtract / skip ([1.58 位大模型] §3.3)."""
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    M, K = xq.shape
    N = codes.shape[0]
    assert codes.shape[1] == K
    acc = np.empty((M, N), dtype=np.int32)
    if _load().orc_ternary_matmul(_ptr(xq), _ptr(codes), M, N, K, _ptr(acc), threads) != 0:
        raise OverflowError("accumulator outside int32")
    return acc


def dequant(acc: np.ndarray, beta: np.ndarray, alpha, bias: np.ndarray | None = None) -> np.ndarray:
    """y = fp32(acc)·fp32(α·β/127) (+ bias) (§2.4–§2.5, §4.2)."""
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    beta = np.ascontiguousarray(beta, dtype=np.float32)
    M, N = acc.shape
    if bias is not None:
        bias = np.ascontiguousarray(bias, dtype=np.float32)
    y = np.empty((M, N), dtype=np.float32)
    _load().orc_dequant(_ptr(acc), _ptr(beta), ctypes.c_float(float(np.float32(alpha))), _ptr(bias), M, N, _ptr(y))
    return y


def forward(x: np.ndarray, codes: np.ndarray, alpha, bias: np.ndarray | None = None, threads: int = 1):
    """Inference forward on cached codes: returns (x̃, β, acc, y)."""
    x, dt = _as_input(x)
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    M, K = x.shape
    N = codes.shape[0]
    xq = np.empty((M, K), dtype=np.int8)
    beta = np.empty(M, dtype=np.float32)
    acc = np.empty((M, N), dtype=np.int32)
    y = np.empty((M, N), dtype=np.float32)
    if bias is not None:
        bias = np.ascontiguousarray(bias, dtype=np.float32)
    rc = _load().orc_forward(_ptr(x), dt, M, K, _ptr(codes), ctypes.c_float(float(np.float32(alpha))),
                             _ptr(bias), N, _ptr(xq), _ptr(beta), _ptr(acc), _ptr(y), threads)
    if rc != 0:
        raise OverflowError("accumulator outside int32")
    return xq, beta, acc, y


# ----------------------------------------------------------------------------- layer stack
STACK_MATRICES = ("q", "k", "v", "o", "gate", "up", "down")


def stack_layer(h: np.ndarray, layer: dict, threads: int = 1) -> dict:
    """One layer of the linear stack: every BitLinear input is quantised on
    entry and the residual addition stays in float ("1.58-bit 大模型极限量化实战"
    §6.1).  The pages give no wiring between the seven linears, so the reading
    is: q, k, v, gate and up consume quant(h); o consumes quant(y_v); down
    consumes quant(y_up); the next layer's input is y_o + y_down, added in
    binary32.  `layer` maps each name in STACK_MATRICES to (codes, alpha);
    h is float32 [M][hidden].  Returns every product's output and h_next."""
    h = np.ascontiguousarray(h, dtype=np.float32)
    out = {}
    for name in ("q", "k", "v", "gate", "up"):
        codes, alpha = layer[name]
        out[name] = forward(h, codes, alpha, threads=threads)[3]
    codes, alpha = layer["o"]
    out["o"] = forward(out["v"], codes, alpha, threads=threads)[3]
    codes, alpha = layer["down"]
    out["down"] = forward(out["up"], codes, alpha, threads=threads)[3]
    out["h_next"] = np.add(out["o"], out["down"], dtype=np.float32)
    return out


def stack_forward(h0: np.ndarray, layers: list, threads: int = 1) -> list:
    """stack_layer applied layer after layer from h0; returns each layer's outputs."""
    outs, h = [], h0
    for layer in layers:
        o = stack_layer(h, layer, threads=threads)
        outs.append(o)
        h = o["h_next"]
    return outs


# ----------------------------------------------------------------------------- rotation
def hadamard_block(K: int, cap: int = 8192) -> int:
    """Block order used when a rotation is asked for without one: the largest
    power of two dividing K, at most `cap` (4096 for K = 4096, 256 for 11008)."""
    b = 1
    while K % (2 * b) == 0 and 2 * b <= cap:
        b *= 2
    return b


def hadamard(x: np.ndarray, block: int, scale: float = 1.0) -> np.ndarray:
    """x·H per row, H block-diagonal Sylvester Hadamard of order `block`, by the
    binary32 butterfly (stages h = 1, 2, 4, …), outputs times `scale`
    ([BitNet 三值权重实战] §6.2)."""
    x, dt = _as_input(x)
    M, K = x.shape
    out = np.empty((M, K), dtype=np.float32)
    if _load().orc_hadamard(_ptr(x), dt, M, K, block, ctypes.c_float(float(np.float32(scale))), _ptr(out)) != 0:
        raise ValueError("block must be a power of two dividing K")
    return out


def quantize_weights_rotated(W: np.ndarray, block: int):
    """(packed, α, codes, W') of W' = W·H/block: the weight side of the rotation,
    so that (x·H)·W'ᵀ = x·Wᵀ in exact arithmetic."""
    Wr = hadamard(W, block, 1.0 / block)
    packed, alpha, codes = quantize_weights(Wr)
    return packed, alpha, codes, Wr


def quantize_act_rotated(x: np.ndarray, block: int):
    """(x̃, β, x·H): the absmax int8 quantisation of the rotated activations."""
    xr = hadamard(x, block)
    xq, beta = quantize_act(xr)
    return xq, beta, xr


# ----------------------------------------------------------------------------- scale granularity
def absmean_groups(W: np.ndarray, group: int) -> np.ndarray:
    """α [N][ceil(K/group)]: exact mean of |W| over each group of `group`
    consecutive elements of a row, RN32(RN64(·)) (per row: group >= K)."""
    W, dt = _as_input(W)
    N, K = W.shape
    G = -(-K // group)
    out = np.empty((N, G), dtype=np.float32)
    if _load().orc_absmean_groups(_ptr(W), dt, N, K, group, _ptr(out)) != 0:
        raise ValueError("non-finite weight or bad group")
    return out


def ternarize_groups(W: np.ndarray, alpha: np.ndarray, group: int) -> np.ndarray:
    """Codes ŵ = clip(round(W/α_group), -1, 1)."""
    W, dt = _as_input(W)
    N, K = W.shape
    alpha = np.ascontiguousarray(alpha, dtype=np.float32)
    out = np.empty((N, K), dtype=np.int8)
    _load().orc_ternarize_groups(_ptr(W), dt, N, K, group, _ptr(alpha), _ptr(out))
    return out


def quantize_weights_groups(W: np.ndarray, group: int):
    """(packed, α [N][G], codes) with one α per group of each row."""
    alpha = absmean_groups(W, group)
    codes = ternarize_groups(W, alpha, group)
    return pack(codes), alpha, codes


def forward_groups(xq: np.ndarray, beta: np.ndarray, codes: np.ndarray, alpha: np.ndarray, group: int,
                   bias: np.ndarray | None = None, threads: int = 1) -> np.ndarray:
    """y with one α per group: S = Σ_b α_b·acc_b (binary64, groups in order),
    y = RN32(RN32(S)·RN32(RN64(β/127))) (+ bias)."""
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    beta = np.ascontiguousarray(beta, dtype=np.float32)
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    alpha = np.ascontiguousarray(alpha, dtype=np.float32)
    M, K = xq.shape
    N = codes.shape[0]
    if bias is not None:
        bias = np.ascontiguousarray(bias, dtype=np.float32)
    y = np.empty((M, N), dtype=np.float32)
    _load().orc_forward_groups(_ptr(xq), _ptr(beta), M, K, _ptr(codes), _ptr(alpha), group, _ptr(bias), N, _ptr(y),
                               threads)
    return y


# ----------------------------------------------------------------------------- 4-bit activations
def quantize_act_a4(x: np.ndarray):
    """(x̃ packed 4-bit [M][ceil(K/2)] uint8, β [M]): clip(round(7x/β), -7, 7)."""
    x, dt = _as_input(x)
    M, K = x.shape
    xq4 = np.empty((M, (K + 1) // 2), dtype=np.uint8)
    beta = np.empty(M, dtype=np.float32)
    _load().orc_quantize_act_a4(_ptr(x), dt, M, K, _ptr(xq4), _ptr(beta))
    return xq4, beta


def unpack_a4(xq4: np.ndarray, K: int) -> np.ndarray:
    xq4 = np.ascontiguousarray(xq4, dtype=np.uint8)
    M = xq4.shape[0]
    out = np.empty((M, K), dtype=np.int8)
    _load().orc_unpack_a4(_ptr(xq4), M, K, _ptr(out))
    return out


def dequant_a4(acc: np.ndarray, beta: np.ndarray, alpha, bias: np.ndarray | None = None) -> np.ndarray:
    """y = fp32(acc)·fp32(α·β/7) (+ bias)."""
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    beta = np.ascontiguousarray(beta, dtype=np.float32)
    M, N = acc.shape
    if bias is not None:
        bias = np.ascontiguousarray(bias, dtype=np.float32)
    y = np.empty((M, N), dtype=np.float32)
    _load().orc_dequant_a4(_ptr(acc), _ptr(beta), ctypes.c_float(float(np.float32(alpha))), _ptr(bias), M, N, _ptr(y))
    return y


def forward_a4(x: np.ndarray, codes: np.ndarray, alpha, bias: np.ndarray | None = None, threads: int = 1):
    """4-bit-activation forward on cached codes: returns (x̃ packed, β, acc, y)."""
    xq4, beta = quantize_act_a4(x)
    K = codes.shape[1]
    acc = ternary_matmul(unpack_a4(xq4, K), codes, threads=threads)
    return xq4, beta, acc, dequant_a4(acc, beta, alpha, bias)


# ----------------------------------------------------------------------------- training (STE)
def ste_grad_x(g: np.ndarray, codes: np.ndarray, alpha, threads: int = 1) -> np.ndarray:
    """∂L/∂x [M][K] = α·Σ_n g[m][n]·ŵ[n][k] (binary64 sum, one binary32 rounding)
    ([BitNet 三值权重实战] §3.3: the quantisers pass the gradient straight through)."""
    g = np.ascontiguousarray(g, dtype=np.float32)
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    M, N = g.shape
    K = codes.shape[1]
    out = np.empty((M, K), dtype=np.float32)
    _load().orc_ste_grad_x(_ptr(g), M, N, _ptr(codes), K, ctypes.c_float(float(np.float32(alpha))), _ptr(out), threads)
    return out


def ste_grad_w(g: np.ndarray, xq: np.ndarray, beta: np.ndarray, W: np.ndarray, alpha, threads: int = 1) -> np.ndarray:
    """∂L/∂W [N][K] = [|W/α| <= 1]·Σ_m RN32(g[m][n]·s_m)·x̃[m][k] (§3.3, §6.3:
    no gradient outside the clip range), s_m = RN32(RN64(β_m/127))."""
    g = np.ascontiguousarray(g, dtype=np.float32)
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    beta = np.ascontiguousarray(beta, dtype=np.float32)
    W, dt = _as_input(W)
    M, N = g.shape
    K = xq.shape[1]
    out = np.empty((N, K), dtype=np.float32)
    _load().orc_ste_grad_w(_ptr(g), M, N, _ptr(xq), _ptr(beta), K, _ptr(W), dt,
                           ctypes.c_float(float(np.float32(alpha))), _ptr(out), threads)
    return out


def train_step(W: np.ndarray, x: np.ndarray, g: np.ndarray, threads: int = 1):
    """One training step of the layer on latent weights W: the forward with
    the weights quantised afresh (§4.2, training branch) and the STE backward
    for the upstream gradient g.  Returns (y, grad_x, grad_W, α, codes, x̃, β)."""
    alpha = absmean(W)
    codes = ternarize(W, alpha)
    xq, beta, acc, y = forward(x, codes, alpha, threads=threads)
    return (y, ste_grad_x(g, codes, alpha, threads), ste_grad_w(g, xq, beta, W, alpha, threads), alpha, codes,
            xq, beta)

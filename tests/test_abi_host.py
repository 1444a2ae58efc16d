"""Host-side checks of the C ABI: the library loads without a GPU, exports every
function include/bitlinear.h declares, and rejects bad arguments on the host
(before any CUDA call) with the documented status.  Fake, never-dereferenced
pointer values stand in for device buffers; no call here reaches a kernel."""
import ctypes
import os
import re

import pytest
import torch

import bitlinear_w1_a8_03_b200 as bl
from bitlinear_w1_a8_03_b200 import build as blbuild

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "bitlinear.h")
OK, NULL, SHAPE, ALIGN, DTYPE, WORKSPACE, ARCH, CUDA, COUNT, TIMEOUT, FLAGS = range(11)
P = 0x7F0000000000  # 16-byte aligned fake device address (never dereferenced)


@pytest.fixture(scope="module")
def L():
    blbuild.build()
    return bl.lib()


def declared_functions():
    text = open(HDR, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bitlinear_\w+)\s*\(", text)))


def test_header_symbols_exported(L):
    names = declared_functions()
    assert {"bitlinear_quantize_weights", "bitlinear_quantize_act", "bitlinear_forward"} <= set(names)
    for n in names:
        assert hasattr(L, n), f"{n} declared in bitlinear.h but not exported"
    assert L.bitlinear_version() == 102  # 1.02: bitlinear_linear_grouped_host added


def test_struct_layout_matches_header():
    assert ctypes.sizeof(bl.ActProblem) == 5 * 8
    assert ctypes.sizeof(bl.ForwardProblem) == 10 * 8


def test_packed_row_bytes(L):
    for K, want in [(0, 0), (-3, 0), (1, 16), (4, 16), (64, 16), (65, 32), (256, 64), (4096, 1024),
                    (11008, 2752), (28672, 7168)]:
        assert L.bitlinear_packed_row_bytes(K) == want


def test_status_strings(L):
    for s in range(11):
        assert L.bitlinear_status_string(s)
    assert b"unknown" in L.bitlinear_status_string(99)


def test_quantize_weights_argument_errors(L):
    q = L.bitlinear_quantize_weights
    ws = L.bitlinear_quantize_weights_workspace_bytes(4, 64)
    assert ws >= 80
    assert q(None, 0, 4, 64, P, P, P, ws, None) == NULL
    assert q(P, 0, 4, 64, None, P, P, ws, None) == NULL
    assert q(P, 7, 4, 64, P, P, P, ws, None) == DTYPE
    assert q(P, 0, 0, 64, P, P, P, ws, None) == SHAPE
    assert q(P, 0, 4, 0, P, P, P, ws, None) == SHAPE
    assert q(P, 0, 4, (1 << 20) + 1, P, P, P, ws, None) == SHAPE
    assert q(P, 0, 1 << 30, 1 << 20, P, P, P, ws, None) == SHAPE  # N·K above 2^40
    assert q(P, 0, 4, 64, P + 8, P, P, ws, None) == ALIGN  # W_packed must be 16-byte aligned
    assert q(P + 2, 0, 4, 64, P, P, P, ws, None) == ALIGN  # fp32 W must be 4-byte aligned
    assert q(P, 0, 4, 64, P, P, None, ws, None) == WORKSPACE
    assert q(P, 0, 4, 64, P, P, P, ws - 1, None) == WORKSPACE


def test_quantize_act_argument_errors(L):
    q = L.bitlinear_quantize_act
    assert q(None, 0, 1, 64, P, P, None) == NULL
    assert q(P, 0, 1, 64, None, P, None) == NULL
    assert q(P, 0, 1, 64, P, None, None) == NULL
    assert q(P, 2, 1, 64, P, P, None) == DTYPE
    assert q(P, 0, 0, 64, P, P, None) == SHAPE
    assert q(P, 0, 1, 0, P, P, None) == SHAPE
    assert q(P + 1, 1, 1, 64, P, P, None) == ALIGN  # bf16 must be 2-byte aligned
    arr = (bl.ActProblem * 17)()
    assert L.bitlinear_quantize_act_grouped(arr, 0, 0, None) == COUNT
    assert L.bitlinear_quantize_act_grouped(arr, 17, 0, None) == COUNT


def test_forward_argument_errors(L):
    f = L.bitlinear_forward
    assert f(None, P, 1, 64, P, P, 8, None, P, None, None) == NULL
    assert f(P, P, 1, 64, P, P, 8, None, None, None, None) == NULL
    assert f(P, P, 0, 64, P, P, 8, None, P, None, None) == SHAPE
    assert f(P, P, 1, 64, P, P, 0, None, P, None, None) == SHAPE
    assert f(P, P, 1, 0, P, P, 8, None, P, None, None) == SHAPE
    assert f(P, P, 1, 64, P + 4, P, 8, None, P, None, None) == ALIGN
    assert f(P, P, 1, 64, P, P, 8, P + 2, P, None, None) == ALIGN  # bias
    arr = (bl.ForwardProblem * 1)()
    assert L.bitlinear_forward_grouped(arr, 0, None) == COUNT
    lin = (bl.LinearProblem * 1)()
    assert L.bitlinear_linear_grouped(lin, 1, 0, 4, None) == 10  # BL_ERR_FLAGS (2 is BL_LINEAR_HADAMARD)
    assert L.bitlinear_linear_grouped(lin, 1, 0, 0, None) == NULL
    assert L.bitlinear_forward_grouped(None, 1, None) == NULL


@pytest.mark.skipif(torch.cuda.is_available(), reason="on a GPU these fake pointers would reach a kernel")
def test_valid_arguments_without_device_report_cuda_error(L):
    ws = L.bitlinear_quantize_weights_workspace_bytes(4, 64)
    assert L.bitlinear_quantize_weights(P, 0, 4, 64, P, P, P, ws, None) == CUDA
    assert L.bitlinear_quantize_act(P, 0, 1, 64, P, P, None) == CUDA
    assert L.bitlinear_forward(P, P, 1, 64, P, P, 8, None, P, None, None) == CUDA


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(bl, "_lib", None)
    monkeypatch.setattr(bl, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        bl.lib()


def test_linear_block_argument_errors(L):
    assert ctypes.sizeof(bl.ActSumProblem) == 7 * 8
    acts = (bl.ActSumProblem * 2)()
    fwd = (bl.ForwardProblem * 1)()
    blk = L.bitlinear_linear_block
    assert blk(None, 1, None, 0, 0, None) == NULL
    assert blk(acts, 0, None, 0, 0, None) == COUNT          # nothing to do
    assert blk(acts, 17, None, 0, 0, None) == COUNT
    assert blk(acts, -1, None, 0, 0, None) == COUNT
    acts[0] = bl.ActSumProblem(P, P, None, P, P, 1, 64)
    assert blk(acts, 1, None, 0, 2, None) == FLAGS
    acts[0] = bl.ActSumProblem(None, P, None, P, P, 1, 64)
    assert blk(acts, 1, None, 0, 0, None) == NULL
    acts[0] = bl.ActSumProblem(P, P, None, None, P, 1, 64)
    assert blk(acts, 1, None, 0, 0, None) == NULL
    acts[0] = bl.ActSumProblem(P, P, None, P, P, 0, 64)
    assert blk(acts, 1, None, 0, 0, None) == SHAPE
    acts[0] = bl.ActSumProblem(P + 2, P, None, P, P, 1, 64)
    assert blk(acts, 1, None, 0, 0, None) == ALIGN
    acts[0] = bl.ActSumProblem(P, P + 2, None, P, P, 1, 64)
    assert blk(acts, 1, None, 0, 0, None) == ALIGN
    acts[0] = bl.ActSumProblem(P, None, P + 1, P, P, 1, 64)
    assert blk(acts, 1, None, 0, 0, None) == ALIGN
    acts[0] = bl.ActSumProblem(P, None, None, P, P, 1, 64)
    assert blk(acts, 1, fwd, 1, 0, None) == NULL             # forward problem left empty
    assert blk(None, 0, fwd, 1, 0, None) == NULL


def test_hadamard_argument_errors(L):
    assert L.bitlinear_hadamard_block(4096) == 4096
    assert L.bitlinear_hadamard_block(11008) == 256
    assert L.bitlinear_hadamard_block(3 * 16384) == 8192
    assert L.bitlinear_hadamard_block(7) == 1 and L.bitlinear_hadamard_block(0) == 0
    h, qh = L.bitlinear_hadamard, L.bitlinear_quantize_act_hadamard
    assert h(None, 0, 1, 64, 64, 1.0, P, None) == NULL
    assert h(P, 0, 1, 64, 64, 1.0, None, None) == NULL
    assert h(P, 5, 1, 64, 64, 1.0, P, None) == DTYPE
    assert h(P, 0, 1, 64, 48, 1.0, P, None) == SHAPE      # not a power of two
    assert h(P, 0, 1, 96, 64, 1.0, P, None) == SHAPE      # does not divide K
    assert h(P, 0, 1, 16384, 16384, 1.0, P, None) == SHAPE  # above the largest block
    assert h(P, 0, 0, 64, 64, 1.0, P, None) == SHAPE
    assert h(P + 2, 0, 1, 64, 64, 1.0, P, None) == ALIGN
    assert qh(P, 0, 1, 64, 64, None, P, None) == NULL
    assert qh(P, 1, 1, 64, 64, P, P + 2, None) == ALIGN
    arr = (bl.LinearProblem * 1)()
    arr[0] = bl.LinearProblem(P, P, P, P, P, None, P, None, 1, 64, 63)
    assert L.bitlinear_linear_grouped(arr, 1, 0, bl.BL_LINEAR_HADAMARD, None) == SHAPE  # block 1: nothing to rotate
    assert L.bitlinear_linear_grouped(arr, 1, 0, 4, None) == FLAGS


def test_scaled_argument_errors(L):
    q = L.bitlinear_quantize_weights_scaled
    assert q(None, 0, 4, 1000, 128, P, P, None) == NULL
    assert q(P, 0, 4, 1000, 100, P, P, None) == SHAPE   # below K and not a multiple of 64
    assert q(P, 0, 4, 1000, 0, P, P, None) == SHAPE
    assert q(P, 0, 4, 1000, 128, P + 8, P, None) == ALIGN
    assert q(P, 7, 4, 1000, 128, P, P, None) == DTYPE
    arr = (bl.ScaledProblem * 1)()
    arr[0] = bl.ScaledProblem(None, P, P, P, P, None, P, P, 1, 64, 1000, 128)  # acc_out with several α per row
    assert L.bitlinear_linear_scaled(arr, 1, 0, 0, None) == SHAPE
    arr[0] = bl.ScaledProblem(None, P, P, P, P, None, P, None, 1, 64, 1000, 96)
    assert L.bitlinear_linear_scaled(arr, 1, 0, 0, None) == SHAPE
    assert L.bitlinear_linear_scaled(arr, 0, 0, 0, None) == COUNT
    assert L.bitlinear_linear_scaled(arr, 1, 0, 2, None) == FLAGS
    assert ctypes.sizeof(bl.ScaledProblem) == 12 * 8


def test_a4_argument_errors(L):
    assert L.bitlinear_quantize_act_a4(None, 0, 1, 64, P, P, None) == NULL
    assert L.bitlinear_quantize_act_a4(P, 3, 1, 64, P, P, None) == DTYPE
    assert L.bitlinear_quantize_act_a4(P, 0, 0, 64, P, P, None) == SHAPE
    assert L.bitlinear_quantize_act_a4(P + 2, 0, 1, 64, P, P, None) == ALIGN
    assert L.bitlinear_forward_a4(P, P, 1, 64, P + 4, P, 8, None, P, None, None) == ALIGN
    assert L.bitlinear_forward_a4(P, P, 1, 64, P, P, 0, None, P, None, None) == SHAPE
    arr = (bl.LinearProblem * 1)()
    assert L.bitlinear_linear_a4(arr, 1, 0, 0, None) == NULL
    assert L.bitlinear_linear_a4(arr, 1, 0, 2, None) == FLAGS
    assert L.bitlinear_linear_a4(arr, 17, 0, 0, None) == COUNT


def test_train_argument_errors(L):
    b = L.bitlinear_ste_backward
    assert b(None, 1, 8, 64, P, P, P, P, P, 0, P, P, None) == NULL
    assert b(P, 1, 8, 64, None, P, P, P, P, 0, P, None, None) == NULL   # grad_x needs the codes
    assert b(P, 1, 8, 64, P, P, None, P, P, 0, None, P, None) == NULL   # grad_W needs x_q
    assert b(P, 0, 8, 64, P, P, P, P, P, 0, P, P, None) == SHAPE
    assert b(P, 1, 8, 64, P, P, P, P, P, 9, None, P, None) == DTYPE
    assert b(P + 2, 1, 8, 64, P, P, P, P, P, 0, P, P, None) == ALIGN
    ws = L.bitlinear_quantize_weights_workspace_bytes(8, 64)
    t = L.bitlinear_train_forward
    assert t(P, 0, 8, 64, None, 0, 1, P, P, P, P, P, P, ws, None) == NULL
    assert t(P, 0, 8, 64, P, 0, 0, P, P, P, P, P, P, ws, None) == SHAPE
    assert t(P, 0, 8, 64, P, 0, 1, P, P, P, P, P, P, 0, None) == WORKSPACE


def test_linear_grouped_host_argument_errors(L):
    """bitlinear_linear_grouped_host checks every argument before its first
    copy: nothing is enqueued for a bad call."""
    assert ctypes.sizeof(bl.HostIO) == 2 * 8
    lin = (bl.LinearProblem * 1)()
    io = (bl.HostIO * 1)()
    h = L.bitlinear_linear_grouped_host
    lin[0] = bl.LinearProblem(P, P, P, P, P, None, P, None, 1, 8, 64)
    assert h(None, io, 1, 0, 0, None) == NULL
    assert h(lin, None, 1, 0, 0, None) == NULL
    assert h(lin, io, 1, 0, 0, None) == NULL            # host pointers left empty
    io[0] = bl.HostIO(0x1000, 0x2000)
    assert h(lin, io, 0, 0, 0, None) == COUNT
    assert h(lin, io, 17, 0, 0, None) == COUNT
    assert h(lin, io, 1, 7, 0, None) == DTYPE
    assert h(lin, io, 1, 0, 4, None) == FLAGS
    lin[0] = bl.LinearProblem(P, P, P, P, P, None, P, None, 0, 8, 64)
    assert h(lin, io, 1, 0, 0, None) == SHAPE
    lin[0] = bl.LinearProblem(P + 2, P, P, P, P, None, P, None, 1, 8, 64)
    assert h(lin, io, 1, 0, 0, None) == ALIGN
    lin[0] = bl.LinearProblem(P, P, P, P, P, None, None, None, 1, 8, 64)
    assert h(lin, io, 1, 0, 0, None) == NULL            # device y missing

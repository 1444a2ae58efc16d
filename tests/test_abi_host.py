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
    assert L.bitlinear_version() == 100


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
    assert L.bitlinear_linear_grouped(lin, 1, 0, 2, None) == 10  # BL_ERR_FLAGS
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

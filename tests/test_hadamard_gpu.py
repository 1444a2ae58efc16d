"""GPU parity of the Hadamard rotation before the absmax quantisation
("1.58-bit 大模型极限量化实战", chenxutan.com/d/5049.html §6.2) against the
oracle: the rotated values, the rotated activations' x̃ and β, and the weights
quantised from W·H/b are bit-exact (both sides run the same binary32 butterfly
in the same stage order); a rotated linear's int32 accumulators are exact and
its outputs within 1e-5 relative."""
import numpy as np
import pytest
import torch

import bitlinear_w1_a8_03_b200 as bl
import oracle
from bitlinear_w1_a8_03_b200 import synth, workloads
from tests.gpu_util import as_input, np_

pytestmark = pytest.mark.gpu

# (M, K, block): register path (one tile), shared-memory stages (block > 512),
# small blocks, a block equal to K, and rows longer than one tile (K > 16384)
CASES = [(1, 64, 64), (3, 256, 256), (2, 4096, 4096), (1, 11008, 256), (4, 8192, 8192), (1, 28672, 4096),
         (2, 4096, 16), (5, 1024, 1024), (1, 16384, 8192), (2, 2112, 64)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("M,K,block", CASES)
def test_rotation_bit_exact(M, K, block, dtype):
    x = synth.activations(K + M, M, K, outliers=True)
    xd, xo = as_input(x, dtype)
    for scale in (1.0, 1.0 / block):
        got = bl.bitlinear_hadamard(xd, block, scale)
        torch.cuda.synchronize()
        assert np.array_equal(np_(got), oracle.hadamard(xo, block, scale)), (M, K, block, scale)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("M,K,block", CASES)
def test_rotated_act_quant_bit_exact(M, K, block, dtype):
    x = synth.activations(2 * K + M, M, K, outliers=True)
    x[0, :7] = 0.0  # zeros and a spike keep the edge cases in play
    xd, xo = as_input(x, dtype)
    xq, beta = bl.bitlinear_quantize_act_hadamard(xd, block)
    torch.cuda.synchronize()
    xq_r, beta_r, _ = oracle.quantize_act_rotated(xo, block)
    assert np.array_equal(np_(beta), beta_r)
    assert np.array_equal(np_(xq), xq_r)


def test_rotated_zero_token():
    x = np.zeros((2, 512), dtype=np.float32)
    x[1, 3] = -2.0
    xq, beta = bl.bitlinear_quantize_act_hadamard(torch.from_numpy(x).cuda(), 512)
    torch.cuda.synchronize()
    xq_r, beta_r, _ = oracle.quantize_act_rotated(x, 512)
    assert np.array_equal(np_(xq), xq_r) and np.array_equal(np_(beta), beta_r)
    assert not np.any(np_(xq)[0]) and np_(beta)[0] == np.float32(1e-8)


def test_rotated_linear_7b_decode_set():
    """The seven 7B-shaped linears at one token with BL_LINEAR_HADAMARD: the
    weights quantised from W·H/b on the device match the oracle's (α and every
    packed byte), and the rotated linear matches the oracle's rotated forward."""
    specs = workloads.decode_7b_layer_set(M=1)
    probs, refs = [], []
    for s in specs:
        W = synth.weights(s.seed, s.N, s.K, s.w_std)
        b = bl.hadamard_block(s.K)
        packed, alpha = bl.bitlinear_quantize_weights_rotated(torch.from_numpy(W).cuda(), b)
        p_ref, a_ref, codes, _ = oracle.quantize_weights_rotated(W, b)
        torch.cuda.synchronize()
        assert np_(alpha)[0] == a_ref
        assert np.array_equal(np_(packed), p_ref)
        x = synth.activations(s.x_seed, 1, s.K, outliers=True)
        xd, xo = as_input(x, "bf16")
        probs.append(dict(x=xd, x_q=torch.empty((1, s.K), dtype=torch.int8, device="cuda"),
                          beta=torch.empty(1, dtype=torch.float32, device="cuda"), W_packed=packed, alpha=alpha,
                          N=s.N, y=torch.empty((1, s.N), dtype=torch.float32, device="cuda"),
                          acc_out=torch.empty((1, s.N), dtype=torch.int32, device="cuda")))
        refs.append((xo, codes, a_ref, b))
    bl.bitlinear_linear_grouped(probs, flags=bl.BL_LINEAR_HADAMARD | bl.BL_LINEAR_WEIGHTS_STATIC)
    torch.cuda.synchronize()
    assert bl.bitlinear_device_error() == 0
    for p, (xo, codes, a_ref, b) in zip(probs, refs):
        xq_r, beta_r, _ = oracle.quantize_act_rotated(xo, b)
        acc_r = oracle.ternary_matmul(xq_r, codes, threads=8)
        y_r = oracle.dequant(acc_r, beta_r, a_ref).astype(np.float64)
        assert np.array_equal(np_(p["x_q"]), xq_r)
        assert np.array_equal(np_(p["beta"]), beta_r)
        assert np.array_equal(np_(p["acc_out"]), acc_r)
        y = np_(p["y"]).astype(np.float64)
        assert np.all(np.abs(y - y_r) <= 1e-5 * np.abs(y_r) + 1e-37)


def test_rotated_prefill_grouped():
    """Many tokens: the rotation kernel, then the tensor-core GEMM."""
    specs = [workloads.prefill(4096, 4096, M=256), workloads.prefill(11008, 4096, M=256)]
    probs, refs = [], []
    for s in specs:
        W = synth.weights(s.seed, s.N, s.K, s.w_std)
        b = bl.hadamard_block(s.K)
        packed, alpha = bl.bitlinear_quantize_weights_rotated(torch.from_numpy(W).cuda(), b)
        _, a_ref, codes, _ = oracle.quantize_weights_rotated(W, b)
        x = synth.activations(s.x_seed, s.M, s.K, outliers=True)
        xd, xo = as_input(x, "bf16")
        probs.append(dict(x=xd, x_q=torch.empty((s.M, s.K), dtype=torch.int8, device="cuda"),
                          beta=torch.empty(s.M, dtype=torch.float32, device="cuda"), W_packed=packed, alpha=alpha,
                          N=s.N, y=torch.empty((s.M, s.N), dtype=torch.float32, device="cuda"),
                          acc_out=torch.empty((s.M, s.N), dtype=torch.int32, device="cuda")))
        refs.append((xo, codes, a_ref, b))
    bl.bitlinear_linear_grouped(probs, flags=bl.BL_LINEAR_HADAMARD)
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    for p, (xo, codes, a_ref, b), s in zip(probs, refs, specs):
        xq_r, beta_r, _ = oracle.quantize_act_rotated(xo, b)
        assert np.array_equal(np_(p["x_q"]), xq_r) and np.array_equal(np_(p["beta"]), beta_r)
        rows = np.unique(np.concatenate([np.arange(128), rng.choice(s.N, 32, replace=False)]))
        acc_r = oracle.ternary_matmul(xq_r, codes[rows], threads=8)
        y_r = oracle.dequant(acc_r, beta_r, a_ref).astype(np.float64)
        assert np.array_equal(np_(p["acc_out"])[:, rows], acc_r)
        y = np_(p["y"])[:, rows].astype(np.float64)
        assert np.all(np.abs(y - y_r) <= 1e-5 * np.abs(y_r) + 1e-37)


# (N, K): rotation blocks of 64 (K = 64, and a row ending in a partial
# 64-element chunk), 16, 256, the largest row the one-token kernel rotates
# in its prologue, and one longer (28672: the separate rotation launch)
ONE_TOKEN = [(40, 64), (136, 2112), (72, 1040), (1000, 11008), (264, 16384), (24, 24576), (16, 28672)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_rotated_linear_one_token(dtype, fusion):
    """One token with BL_LINEAR_HADAMARD, with the rotation inside the product
    kernel's prologue (forced on), in its own launch (off) or as the library
    picks: x̃, β and the int32 accumulators bit-exact, y within 1e-5."""
    probs, refs = [], []
    for j, (N, K) in enumerate(ONE_TOKEN):
        b = bl.hadamard_block(K)
        W = synth.weights(100 + j, N, K, 0.02)
        packed, alpha = bl.bitlinear_quantize_weights_rotated(torch.from_numpy(W).cuda(), b)
        _, a_ref, codes, _ = oracle.quantize_weights_rotated(W, b)
        x = synth.activations(200 + j, 1, K, outliers=True)
        if j == 2:
            x[:] = 0.0  # a zero token: β = 1e-8 and every code 0
        xd, xo = as_input(x, dtype)
        probs.append(dict(x=xd, x_q=torch.empty((1, K), dtype=torch.int8, device="cuda"),
                          beta=torch.empty(1, dtype=torch.float32, device="cuda"), W_packed=packed, alpha=alpha,
                          N=N, y=torch.empty((1, N), dtype=torch.float32, device="cuda"),
                          acc_out=torch.empty((1, N), dtype=torch.int32, device="cuda")))
        refs.append((xo, codes, a_ref, b))
    # one call per problem: forced on, every row that fits the prologue is fused
    for p in probs:
        bl.bitlinear_linear_grouped([p], flags=bl.BL_LINEAR_HADAMARD)
    torch.cuda.synchronize()
    assert bl.bitlinear_device_error() == 0
    for p, (xo, codes, a_ref, b) in zip(probs, refs):
        xq_r, beta_r, _ = oracle.quantize_act_rotated(xo, b)
        acc_r = oracle.ternary_matmul(xq_r, codes, threads=8)
        y_r = oracle.dequant(acc_r, beta_r, a_ref).astype(np.float64)
        assert np.array_equal(np_(p["beta"]), beta_r)
        assert np.array_equal(np_(p["x_q"]), xq_r)
        assert np.array_equal(np_(p["acc_out"]), acc_r)
        y = np_(p["y"]).astype(np.float64)
        assert np.all(np.abs(y - y_r) <= 1e-5 * np.abs(y_r) + 1e-37)

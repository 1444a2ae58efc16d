"""GPU parity of the 4-bit activation variant ("BitNet CPU 实测",
cf-1.com/news/5800143 §2.1) against the oracle: the packed 4-bit x̃ (every
byte), β, the int32 accumulators and y = fp32(acc)·RN32(RN64(α·β/7)) are
bit-exact (the same binary32 steps on both sides)."""
import numpy as np
import pytest
import torch

import bitlinear_w1_a8_03_b200 as bl
import oracle
from bitlinear_w1_a8_03_b200 import synth, workloads
from tests.gpu_util import as_input, np_

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("M,K", [(1, 256), (3, 4096), (2, 301), (5, 11008), (1, 7), (4, 1000)])
def test_act_a4_bit_exact(M, K, dtype):
    x = synth.activations(M * 31 + K, M, K, outliers=True)
    if M > 1:
        x[1] = 0.0
    xd, xo = as_input(x, dtype)
    xq4, beta = bl.bitlinear_quantize_act_a4(xd)
    torch.cuda.synchronize()
    q_r, b_r = oracle.quantize_act_a4(xo)
    assert np.array_equal(np_(beta), b_r)
    assert np.array_equal(np_(xq4), q_r)


def test_act_a4_ties(golden):
    g = golden("act_int4_ties.txt")
    x = torch.tensor([g["x"]], dtype=torch.float32, device="cuda")
    xq4, beta = bl.bitlinear_quantize_act_a4(x)
    torch.cuda.synchronize()
    assert np_(beta)[0] == np.float32(g["beta"][0])
    assert np.array_equal(np_(xq4)[0], np.uint8(g["packed"]))


@pytest.mark.parametrize("M", [1, 2, 4, 7])
@pytest.mark.parametrize("N,K", [(64, 4096), (40, 300), (24, 11008), (9, 64)])
def test_forward_a4_bit_exact(M, N, K):
    W = synth.weights(N + K, N, K, 0.02)
    packed, alpha = bl.bitlinear_quantize_weights(torch.from_numpy(W).cuda())
    _, a_ref, codes = oracle.quantize_weights(W)
    x = synth.activations(M + 5 * K, M, K, outliers=True)
    xd, xo = as_input(x, "bf16")
    xq4, beta = bl.bitlinear_quantize_act_a4(xd)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    bias = torch.from_numpy(synth.activations(9, 1, N)[0]).cuda() if M == 2 else None
    y = bl.bitlinear_forward_a4(xq4, beta, K, packed, alpha, N, bias=bias, acc_out=acc)
    torch.cuda.synchronize()
    q_r, b_r, acc_r, y_r = oracle.forward_a4(xo, codes, a_ref, bias=None if bias is None else np_(bias), threads=8)
    assert np.array_equal(np_(xq4), q_r) and np.array_equal(np_(beta), b_r)
    assert np.array_equal(np_(acc), acc_r)
    assert np.array_equal(np_(y), y_r)


def test_linear_a4_7b_decode_set():
    specs = workloads.decode_7b_layer_set(M=1)
    probs, refs = [], []
    for s in specs:
        W = synth.weights(s.seed, s.N, s.K, s.w_std)
        packed, alpha = bl.bitlinear_quantize_weights(torch.from_numpy(W).cuda())
        _, a_ref, codes = oracle.quantize_weights(W)
        x = synth.activations(s.x_seed, 1, s.K, outliers=True)
        xd, xo = as_input(x, "bf16")
        probs.append(dict(x=xd, x_q=torch.empty((1, (s.K + 1) // 2), dtype=torch.uint8, device="cuda"),
                          beta=torch.empty(1, dtype=torch.float32, device="cuda"), W_packed=packed, alpha=alpha,
                          N=s.N, y=torch.empty((1, s.N), dtype=torch.float32, device="cuda"),
                          acc_out=torch.empty((1, s.N), dtype=torch.int32, device="cuda")))
        refs.append((xo, codes, a_ref))
    bl.bitlinear_linear_a4(probs, flags=bl.BL_LINEAR_WEIGHTS_STATIC)
    torch.cuda.synchronize()
    assert bl.bitlinear_device_error() == 0
    for p, (xo, codes, a_ref) in zip(probs, refs):
        q_r, b_r, acc_r, y_r = oracle.forward_a4(xo, codes, a_ref, threads=8)
        assert np.array_equal(np_(p["x_q"]), q_r) and np.array_equal(np_(p["beta"]), b_r)
        assert np.array_equal(np_(p["acc_out"]), acc_r)
        assert np.array_equal(np_(p["y"]), y_r)

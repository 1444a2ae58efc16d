"""Tensor-core (tcgen05) GEMM path: more than four tokens go through the int8
tensor cores.  Bit-exact int32 accumulators and x̃ against the oracle, fp32
outputs within 1e-5 relative, over token counts that cover every tile width
(16 .. 256 tokens) with ragged edges in tokens, rows and K."""
import numpy as np
import pytest
import torch

import bitlinear_w1_a8_03_b200 as bl
import oracle
from bitlinear_w1_a8_03_b200 import synth
from tests.gpu_util import as_input, dev_f32, np_

pytestmark = pytest.mark.gpu


def run_case(M, K, N, seed, bias=False, dtype="bf16"):
    W = synth.weights(seed, N, K, 0.02)
    x = synth.activations(seed, M, K, outliers=True)
    Wd, Wo = as_input(W, "f32")
    packed, alpha = bl.bitlinear_quantize_weights(Wd)
    p_ref, a_ref, codes = oracle.quantize_weights(Wo)
    assert np_(alpha)[0] == a_ref and np.array_equal(np_(packed), p_ref)
    xd, xo = as_input(x, dtype)
    b = synth.activations(seed + 1, 1, N)[0] if bias else None
    xq, beta = bl.bitlinear_quantize_act(xd)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    y = bl.bitlinear_forward(xq, beta, packed, alpha, N, bias=None if b is None else dev_f32(b), acc_out=acc)
    xq_r, beta_r, acc_r, y_r = oracle.forward(xo, codes, a_ref, bias=b, threads=8)
    assert np.array_equal(np_(xq), xq_r)
    assert np.array_equal(np_(acc), acc_r)
    err = np.abs(np_(y).astype(np.float64) - y_r)
    assert np.all(err <= 1e-5 * np.abs(y_r) + 1e-37)
    assert bl.bitlinear_device_error() == 0


@pytest.mark.parametrize("M", [5, 8, 16, 17, 32, 33, 64, 65, 128, 129, 256, 300])
def test_gemm_token_counts(M):
    run_case(M, 256, 200, seed=600 + M, bias=(M % 2 == 1))


@pytest.mark.parametrize("K,N", [(16, 130), (48, 128), (128, 127), (192, 257), (1024, 384), (4096 + 64, 256),
                                 (512, 254), (1536, 381)])
def test_gemm_ragged_k_and_rows(K, N):
    run_case(37, K, N, seed=700 + K + N)


@pytest.mark.parametrize("M", [8, 16, 24, 48])
def test_gemm_few_tokens_many_stages_and_tiles(M):
    """The few-token tensor-core path (tiles of 127 rows, K stages of 512)
    over several stages, a ragged last stage and a one-row last tile."""
    run_case(M, 2560 + 64, 127 * 4 + 1, seed=650 + M, bias=(M == 24))


@pytest.mark.parametrize("M,K,N", [(16, 512 * 6 + 64, 300), (64, 512 * 6 + 64, 300), (16, 4096, 127 * 150),
                                   (40, 512 * 5 + 64, 127 * 4 + 1)])
def test_gemm_few_tokens_split_k_pairs(M, K, N):
    """Few tiles with long K: the two CTAs of a cluster each take half of
    every tile's K stages (an odd stage count; three tiles per cluster with
    150 tiles) and the first adds the second's partial accumulators."""
    run_case(M, K, N, seed=660 + M + K % 97)


@pytest.mark.parametrize("M", [3, 4])
def test_gemm_three_four_tokens_large_weights(M):
    """Three or four tokens on 8 MB of weights go to the tensor-core GEMM
    rather than the streaming GEMV (checked: the same results)."""
    run_case(M, 4096, 8192, seed=690 + M)


@pytest.mark.parametrize("M", [3, 4])
def test_linear_grouped_three_four_tokens_large_weights(M, fusion):
    """bitlinear_linear_grouped at three or four tokens over 8 MB of weights:
    act quant + GEMM by default, the fused GEMV when fusion is forced on."""
    K, N = 4096, 8192
    W = synth.weights(710 + M, N, K, 0.02)
    x = synth.activations(720 + M, M, K, outliers=True)
    Wd, Wo = as_input(W, "f32")
    packed, alpha = bl.bitlinear_quantize_weights(Wd)
    _, a_ref, codes = oracle.quantize_weights(Wo)
    xd, xo = as_input(x, "bf16")
    p = dict(x=xd, x_q=torch.empty((M, K), dtype=torch.int8, device="cuda"),
             beta=torch.empty(M, dtype=torch.float32, device="cuda"), W_packed=packed, alpha=alpha, N=N,
             y=torch.empty((M, N), dtype=torch.float32, device="cuda"),
             acc_out=torch.empty((M, N), dtype=torch.int32, device="cuda"))
    bl.bitlinear_linear_grouped([p])
    torch.cuda.synchronize()
    assert bl.bitlinear_device_error() == 0
    xq_r, beta_r, acc_r, y_r = oracle.forward(xo, codes, a_ref, threads=8)
    assert np.array_equal(np_(p["x_q"]), xq_r) and np.array_equal(np_(p["beta"]), beta_r)
    assert np.array_equal(np_(p["acc_out"]), acc_r)
    err = np.abs(np_(p["y"]).astype(np.float64) - y_r)
    assert np.all(err <= 1e-5 * np.abs(y_r) + 1e-37)


def test_gemm_prefill_shape_small_rows():
    """2048 tokens (the prefill token count) on a few hundred rows."""
    run_case(2048, 1024, 256, seed=800, dtype="f32")


@pytest.mark.parametrize("M", [16, 37, 300])
def test_gemm_grouped_problems(M):
    """Several problems of different K and N in one tensor-core launch."""
    shapes = [(256, 200), (1024, 384), (4096 + 64, 130), (128, 16)]
    probs, refs = [], []
    for i, (K, N) in enumerate(shapes):
        W = synth.weights(7000 + 13 * i + M, N, K, 0.02)
        x = synth.activations(7100 + 13 * i + M, M, K, outliers=True)
        Wd, Wo = as_input(W, "f32")
        packed, alpha = bl.bitlinear_quantize_weights(Wd)
        p_ref, a_ref, codes = oracle.quantize_weights(Wo)
        xd, xo = as_input(x, "bf16")
        xq, beta = bl.bitlinear_quantize_act(xd)
        pr = dict(x_q=xq, beta=beta, W_packed=packed, alpha=alpha, N=N,
                  y=torch.empty((M, N), dtype=torch.float32, device="cuda"),
                  acc_out=torch.empty((M, N), dtype=torch.int32, device="cuda"))
        probs.append(pr)
        refs.append(oracle.forward(xo, codes, a_ref, threads=8))
    bl.bitlinear_forward_grouped(probs)
    torch.cuda.synchronize()
    assert bl.bitlinear_device_error() == 0
    for pr, (xq_r, beta_r, acc_r, y_r) in zip(probs, refs):
        assert np.array_equal(np_(pr["acc_out"]), acc_r)
        err = np.abs(np_(pr["y"]).astype(np.float64) - y_r)
        assert np.all(err <= 1e-5 * np.abs(y_r) + 1e-37)


def test_gemm_more_tiles_than_the_host_deal_lists():
    """More than 2048 tiles (here 32 token tiles × 66 row tiles): the kernel
    deals them round-robin instead of from the host's per-CTA lists.  Checked
    on every token of 96 sampled rows (and the last row)."""
    M, K, N = 8192, 64, 256 * 65 + 7
    W = synth.weights(910, N, K, 0.02)
    x = synth.activations(911, M, K, outliers=True)
    Wd, Wo = as_input(W, "f32")
    packed, alpha = bl.bitlinear_quantize_weights(Wd)
    _, a_ref, codes = oracle.quantize_weights(Wo)
    xd, xo = as_input(x, "bf16")
    xq, beta = bl.bitlinear_quantize_act(xd)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    y = bl.bitlinear_forward(xq, beta, packed, alpha, N, acc_out=acc)
    torch.cuda.synchronize()
    assert bl.bitlinear_device_error() == 0
    xq_r, beta_r = oracle.quantize_act(xo)
    assert np.array_equal(np_(xq), xq_r)
    rows = np.unique(np.concatenate([np.random.default_rng(912).choice(N, 96, replace=False), [N - 1]]))
    acc_r = oracle.ternary_matmul(xq_r, codes[rows], threads=8)
    y_r = oracle.dequant(acc_r, beta_r, a_ref).astype(np.float64)
    assert np.array_equal(acc[:, torch.from_numpy(rows).cuda()].cpu().numpy(), acc_r)
    err = np.abs(y[:, torch.from_numpy(rows).cuda()].cpu().numpy().astype(np.float64) - y_r)
    assert np.all(err <= 1e-5 * np.abs(y_r) + 1e-37)

"""GPU parity of the finer scale granularities against the oracle: one α per
output row ("1.58 位大模型", nxmr.cn/news/148658 §3.1, §4.2) and one α per
block of 128 input features of a row (2kiu.com/news/4928193 §2.3, §4.2).

α (exact mean of each group, RN32(RN64(·))) and every packed byte are
bit-exact.  With one α per row y = RN32(RN32(α_n·acc)·RN32(RN64(β/127))) is
exact on both sides, so y is bit-exact too (and the int32 accumulators).  With
several α per row S = Σ_b α_b·acc_b is a binary64 sum whose order differs
between the oracle (sequential) and the GPU (per lane, then a tree): the bar is
1e-5 relative plus 2^-40·Σ_b|α_b·acc_b|·s, which bounds the binary64 rounding
of either order (each term is exact, at most 2^14 terms) after the one binary32
rounding of S."""
import numpy as np
import pytest
import torch

import bitlinear_w1_a8_03_b200 as bl
import oracle
from bitlinear_w1_a8_03_b200 import synth, workloads
from tests.gpu_util import as_input, np_

pytestmark = pytest.mark.gpu


def _weights(N, K, group, seed, dtype="f32"):
    W = synth.weights(seed, N, K, 0.02)
    Wd, Wo = as_input(W, dtype)
    packed, alpha = bl.bitlinear_quantize_weights_scaled(Wd, group)
    p_ref, a_ref, codes = oracle.quantize_weights_groups(Wo, group if group < K else K)
    torch.cuda.synchronize()
    assert np.array_equal(np_(alpha), a_ref)
    assert np.array_equal(np_(packed), p_ref)
    return packed, alpha, codes, a_ref


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N,K,group", [(5, 300, 300), (64, 4096, 128), (33, 11008, 128), (7, 1000, 10 ** 6),
                                       (3, 200, 64), (16, 4096, 4096), (9, 704, 192)])
def test_group_weights_bit_exact(N, K, group, dtype):
    _weights(N, K, group, N + K, dtype)


def _block_bound(xq, codes, alpha, group, beta):
    """Σ_b |α_b·acc_b| · s_m for every (m, n): the scale of the binary64 sum."""
    M, K = xq.shape
    N = codes.shape[0]
    T = np.zeros((M, N))
    for b in range(alpha.shape[1]):
        sl = slice(b * group, min(K, (b + 1) * group))
        acc_b = oracle.ternary_matmul(xq[:, sl], codes[:, sl], threads=8).astype(np.float64)
        T += np.abs(acc_b * alpha[:, b].astype(np.float64)[None, :])
    s = np.float32(beta.astype(np.float64) / 127.0).astype(np.float64)
    return T * s[:, None]


@pytest.mark.parametrize("M", [1, 2, 4, 5, 17])
@pytest.mark.parametrize("N,K,group", [(40, 4096, 4096), (24, 11008, 11008), (40, 4096, 128), (24, 11008, 128),
                                       (13, 320, 64), (10, 300, 300)])
def test_scaled_forward(M, N, K, group):
    packed, alpha, codes, a_ref = _weights(N, K, group, 7 * M + K)
    x = synth.activations(M + K, M, K, outliers=True)
    xd, xo = as_input(x, "bf16")
    xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    beta = torch.empty(M, dtype=torch.float32, device="cuda")
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    per_row = group >= K
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda") if per_row else None
    bias = torch.from_numpy(synth.activations(3, 1, N)[0]).cuda() if M == 2 else None
    bl.bitlinear_linear_scaled([dict(x=xd, x_q=xq, beta=beta, W_packed=packed, alpha=alpha, group=group, N=N, y=y,
                                     acc_out=acc, bias=bias)])
    torch.cuda.synchronize()
    assert bl.bitlinear_device_error() == 0
    xq_r, beta_r = oracle.quantize_act(xo)
    assert np.array_equal(np_(xq), xq_r) and np.array_equal(np_(beta), beta_r)
    g = K if per_row else group
    y_r = oracle.forward_groups(xq_r, beta_r, codes, a_ref, g, bias=None if bias is None else np_(bias), threads=8)
    if per_row:
        assert np.array_equal(np_(acc), oracle.ternary_matmul(xq_r, codes, threads=8))
        assert np.array_equal(np_(y), y_r)
    else:
        bound = _block_bound(xq_r, codes, a_ref, group, beta_r)
        d = np.abs(np_(y).astype(np.float64) - y_r.astype(np.float64))
        assert np.all(d <= 1e-5 * np.abs(y_r.astype(np.float64)) + 2.0 ** -40 * bound + 1e-37)


@pytest.mark.parametrize("group", [128, 10 ** 6])
def test_scaled_7b_decode_set(group):
    """The seven 7B-shaped linears at one token, per row and per 128-block, in
    one grouped call with weights flagged static."""
    specs = workloads.decode_7b_layer_set(M=1)
    probs, refs = [], []
    for s in specs:
        packed, alpha, codes, a_ref = _weights(s.N, s.K, group, s.seed)
        x = synth.activations(s.x_seed, 1, s.K, outliers=True)
        xd, xo = as_input(x, "bf16")
        probs.append(dict(x=xd, x_q=torch.empty((1, s.K), dtype=torch.int8, device="cuda"),
                          beta=torch.empty(1, dtype=torch.float32, device="cuda"), W_packed=packed, alpha=alpha,
                          group=group, N=s.N, y=torch.empty((1, s.N), dtype=torch.float32, device="cuda")))
        refs.append((xo, codes, a_ref))
    bl.bitlinear_linear_scaled(probs, flags=bl.BL_LINEAR_WEIGHTS_STATIC)
    torch.cuda.synchronize()
    for p, (xo, codes, a_ref), s in zip(probs, refs, specs):
        xq_r, beta_r = oracle.quantize_act(xo)
        g = min(group, s.K)
        y_r = oracle.forward_groups(xq_r, beta_r, codes, a_ref, g, threads=8)
        if group >= s.K:
            assert np.array_equal(np_(p["y"]), y_r)
        else:
            bound = _block_bound(xq_r, codes, a_ref, group, beta_r)
            d = np.abs(np_(p["y"]).astype(np.float64) - y_r.astype(np.float64))
            assert np.all(d <= 1e-5 * np.abs(y_r.astype(np.float64)) + 2.0 ** -40 * bound + 1e-37)

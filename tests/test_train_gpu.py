"""GPU parity of the training step with the straight-through estimator
("1.58-bit 大模型极限量化实战" §3.3, §4.2 training branch, §6.3) against the
oracle.  Forward: α, every packed byte, x̃, β bit-exact, y within 1e-5
relative.  Backward: float32 sums (each output by one thread, in index order)
against the oracle's binary64 sums; the bar is 1e-5 relative plus the float32
summation bound (L + 2)·2^-24·Σ|terms| (L terms per output), and weights
outside the clip range get exactly zero."""
import numpy as np
import pytest
import torch

import bitlinear_w1_a8_03_b200 as bl
import oracle
from bitlinear_w1_a8_03_b200 import synth
from tests.gpu_util import as_input, np_

pytestmark = pytest.mark.gpu


def _close(got, ref, scale, L):
    d = np.abs(got.astype(np.float64) - ref.astype(np.float64))
    return np.all(d <= 1e-5 * np.abs(ref.astype(np.float64)) + (L + 2) * 2.0 ** -24 * scale + 1e-37)


@pytest.mark.parametrize("M,N,K", [(1, 256, 256), (5, 100, 300), (64, 256, 512), (257, 130, 70), (512, 1024, 1024)])
def test_train_step(M, N, K):
    W = synth.weights(M + N + K, N, K, 0.02)
    W[0, :3] = 0.2  # outside the clip range
    x = synth.activations(K + 1, M, K, outliers=True)
    g = synth.activations(N + 2, M, N)
    Wd = torch.from_numpy(W).cuda()
    xd, xo = as_input(x, "bf16")
    y, packed, alpha, xq, beta = bl.bitlinear_train_forward(Wd, xd)
    gd = torch.from_numpy(g).cuda()
    gx, gw = bl.bitlinear_ste_backward(gd, packed, alpha, xq, beta, Wd)
    torch.cuda.synchronize()
    assert bl.bitlinear_device_error() == 0
    y_r, gx_r, gw_r, a_r, codes, xq_r, beta_r = oracle.train_step(W, xo, g, threads=8)
    assert np_(alpha)[0] == a_r
    assert np.array_equal(np_(packed), oracle.pack(codes))
    assert np.array_equal(np_(xq), xq_r) and np.array_equal(np_(beta), beta_r)
    yy = np_(y).astype(np.float64)
    assert np.all(np.abs(yy - y_r) <= 1e-5 * np.abs(y_r) + 1e-37)
    sx = float(a_r) * (np.abs(g).astype(np.float64) @ np.abs(codes).astype(np.float64))
    assert _close(np_(gx), gx_r, sx, N)
    s = np.float32(beta_r.astype(np.float64) / 127.0).astype(np.float64)
    sw = (np.abs(g).astype(np.float64) * s[:, None]).T @ np.abs(xq_r).astype(np.float64)
    assert _close(np_(gw), gw_r, sw, M)
    mask = np.abs(W / np.float32(a_r)) <= 1
    assert not np.any(np_(gw)[~mask]) and not mask[0, 0]


def test_train_worked_example(golden):
    d = golden("ste_worked_example.txt")
    W = torch.tensor([d["W"]], dtype=torch.float32, device="cuda")
    x = torch.tensor([d["x"]], dtype=torch.float32, device="cuda")
    g = torch.tensor([d["g"]], dtype=torch.float32, device="cuda")
    y, packed, alpha, xq, beta = bl.bitlinear_train_forward(W, x)
    gx, gw = bl.bitlinear_ste_backward(g, packed, alpha, xq, beta, W)
    torch.cuda.synchronize()
    assert np.array_equal(np_(gx)[0], np.float32(d["grad_x"]))
    s = np.float32(1.0 / 127.0)
    assert np.array_equal(np_(gw)[0], np.float32([0.0, np.float32(2 * s) * 64, np.float32(2 * s) * -64, 0.0]))


def test_backward_one_output_only():
    M, N, K = 3, 40, 64
    W = torch.from_numpy(synth.weights(1, N, K, 0.02)).cuda()
    x = torch.from_numpy(synth.activations(1, M, K)).cuda()
    g = torch.from_numpy(synth.activations(2, M, N)).cuda()
    y, packed, alpha, xq, beta = bl.bitlinear_train_forward(W, x)
    gx, gw = bl.bitlinear_ste_backward(g, packed, alpha, xq, beta, W, grad_x=True, grad_W=False)
    assert gw is None and gx is not None
    gx2, gw2 = bl.bitlinear_ste_backward(g, packed, alpha, xq, beta, W, grad_x=False, grad_W=True)
    torch.cuda.synchronize()
    assert gx2 is None and gw2 is not None

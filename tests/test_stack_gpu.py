"""The decoder-layer linear stack on the GPU (bitlinear_linear_block layer after
layer) against the oracle's stack: every product's output, every layer's
input h and the final h bit-exact, on small stacks and on two full 7B-shaped
layers; the full 32-layer stack through properties that hold at any depth."""
import os

import numpy as np
import pytest
import torch

import bitlinear_w1_a8_03_b200 as bl
import oracle
from bitlinear_w1_a8_03_b200 import synth
from bitlinear_w1_a8_03_b200.stack import MATRICES, LinearStack, shapes
from tests.gpu_util import np_

pytestmark = pytest.mark.gpu
THREADS = os.cpu_count() or 1


def _layers(hidden, ffn, L, base_seed):
    """Device (packed, alpha) and oracle (codes, alpha) for every matrix;
    seed = base + 7·layer + matrix index."""
    sh = shapes(hidden, ffn)
    dev_layers, orc_layers = [], []
    for l in range(L):
        d, o = {}, {}
        for i, n in enumerate(MATRICES):
            N, K = sh[n]
            W = synth.weights(base_seed + 7 * l + i, N, K, 0.02)
            packed, alpha = bl.bitlinear_quantize_weights(torch.from_numpy(W).cuda())
            a_ref = oracle.absmean(W)
            codes = oracle.ternarize(W, a_ref)
            assert np_(alpha)[0] == a_ref
            assert np.array_equal(np_(packed), oracle.pack(codes))
            d[n] = (packed, alpha)
            o[n] = (codes, a_ref)
        dev_layers.append(d)
        orc_layers.append(o)
    return dev_layers, orc_layers


def _check(hidden, ffn, L, M, base_seed):
    dev_layers, orc_layers = _layers(hidden, ffn, L, base_seed)
    h0 = synth.activations(base_seed + 999, M, hidden, outliers=True)
    st = LinearStack(dev_layers, hidden, ffn, M, torch.device("cuda"), keep_all=True)
    st.h0.copy_(torch.from_numpy(h0))
    st.run()
    torch.cuda.synchronize()
    assert bl.bitlinear_device_error() == 0
    ref = oracle.stack_forward(h0, orc_layers, threads=THREADS)
    h = h0
    for l in range(L):
        assert np.array_equal(np_(st.h_in[l]), h), f"layer {l} input"
        for n in MATRICES:
            assert np.array_equal(np_(st.y[l][n]), ref[l][n]), f"layer {l} {n}"
        h = ref[l]["h_next"]
    assert np.array_equal(np_(st.h_final), h)


@pytest.mark.parametrize("M", [1, 3, 16])
def test_small_stack_bitexact(M, fusion):
    """Three layers at hidden 256 / FFN 512: GEMV path (1, 3 tokens, fused or
    not) and tensor-core path (16 tokens)."""
    _check(256, 512, 3, M, base_seed=5100 + M)


@pytest.mark.parametrize("M", [1, 16])
def test_two_full_7b_layers_bitexact(M):
    """Two layers at the 7B shapes (hidden 4096, FFN 11008)."""
    _check(4096, 11008, 2, M, base_seed=5000)


def _random_stack(L, hidden, ffn, seed):
    g = torch.Generator(device="cuda")
    sh = shapes(hidden, ffn)
    layers = []
    for l in range(L):
        d = {}
        for i, n in enumerate(MATRICES):
            g.manual_seed(seed + 7 * l + i)
            W = torch.randn(sh[n], generator=g, device="cuda") * 0.02
            d[n] = bl.bitlinear_quantize_weights(W)
            del W
        layers.append(d)
    return layers


def test_full_32_layer_stack_properties():
    """The full 7B-shaped stack, M = 1: two runs agree bit for bit, and scaling
    the input by 2^k scales every layer's input and the output exactly by 2^k
    (per-token absmax quantisation is scale-invariant while every max|x| is
    large enough for β's 1e-8 to vanish, checked below)."""
    layers = _random_stack(32, 4096, 11008, seed=5000)
    st = LinearStack(layers, 4096, 11008, 1, torch.device("cuda"), keep_all=True)
    h0 = torch.from_numpy(synth.activations(5999, 1, 4096, outliers=True)).cuda()
    st.h0.copy_(h0)
    st.run()
    torch.cuda.synchronize()
    base_in = [t.clone() for t in st.h_in]
    base_out = st.h_final.clone()
    assert torch.isfinite(base_out).all()
    for l in range(32):
        for t in (base_in[l], st.y[l]["v"], st.y[l]["up"]):
            assert t.abs().max().item() >= 2.0
    st.run()
    torch.cuda.synchronize()
    assert torch.equal(st.h_final, base_out)
    for k in (3, -1):
        st.h0.copy_(h0 * 2.0 ** k)
        st.run()
        torch.cuda.synchronize()
        assert torch.equal(st.h_final, base_out * 2.0 ** k)
        for l in range(32):
            assert torch.equal(st.h_in[l], base_in[l] * 2.0 ** k)
    assert bl.bitlinear_device_error() == 0

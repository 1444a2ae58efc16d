"""Full-size parity at the benchmark shapes, through the same C-ABI calls the
benchmark times.  Weight quantisation (α, every packed byte) and activation
quantisation (every x̃, β) are compared in full; the products are compared on
sampled output rows that the oracle computes one by one (bit-exact int32
accumulators, fp32 outputs within 1e-5 relative).

Workloads (seeded synthetic, W ~ N(0, σ²) float32, x bfloat16):
  7B decode layer set, M = 1: q,k,v,o 4096→4096; gate,up 4096→11008;
      down 11008→4096; σ = 0.02; 0.1% ×20 outlier channels in x.
  100B batched decode: (K, N) = (8192, 28672) and (28672, 8192), σ = 0.015,
      M ∈ {1, 2, 4, 8, 16, 32, 64}.
  Prefill: M = 2048, (K, N) ∈ {(4096, 4096), (4096, 11008), (11008, 4096)},
      σ = 0.02, outliers in x.
"""
import numpy as np
import pytest
import torch

import bitlinear_w1_a8_03_b200 as bl
import oracle
from bitlinear_w1_a8_03_b200 import synth
from bitlinear_w1_a8_03_b200 import workloads
from tests.gpu_util import as_input, np_

pytestmark = pytest.mark.gpu


def quantize_both(W):
    Wd = torch.from_numpy(W).cuda()
    packed, alpha = bl.bitlinear_quantize_weights(Wd)
    del Wd
    p_ref, a_ref, codes = oracle.quantize_weights(W)
    assert np_(alpha)[0] == a_ref
    assert np.array_equal(np_(packed), p_ref)
    return packed, alpha, codes, a_ref


def sample_rows(N, seed, n=160):
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([[0, N - 1], rng.choice(N, size=min(n, N), replace=False)]))
    return rows


def check_sampled(xq, beta, acc, y, xo, codes, a_ref, rows):
    xq_r, beta_r = oracle.quantize_act(xo)
    assert np.array_equal(np_(xq), xq_r)
    assert np.array_equal(np_(beta), beta_r)
    acc_r = oracle.ternary_matmul(xq_r, codes[rows], threads=8)
    y_r = oracle.dequant(acc_r, beta_r, a_ref)
    assert np.array_equal(np_(acc)[:, rows], acc_r)
    ys = np_(y)[:, rows].astype(np.float64)
    assert np.all(np.abs(ys - y_r) <= 1e-5 * np.abs(y_r) + 1e-37)


def test_7b_decode_layer_set_grouped():
    mats = workloads.decode_7b_layer_set()
    problems, inputs = [], []
    xs, outs = [], []
    for spec in mats:
        W = synth.weights(spec.seed, spec.N, spec.K, spec.w_std)
        packed, alpha, codes, a_ref = quantize_both(W)
        x = synth.activations(spec.seed, 1, spec.K, outliers=True)
        xd, xo = as_input(x, "bf16")
        xs.append(xd)
        outs.append((torch.empty((1, spec.K), dtype=torch.int8, device="cuda"),
                     torch.empty(1, dtype=torch.float32, device="cuda")))
        problems.append(dict(x_q=outs[-1][0], beta=outs[-1][1], W_packed=packed, alpha=alpha, N=spec.N,
                             y=torch.empty((1, spec.N), dtype=torch.float32, device="cuda"),
                             acc_out=torch.empty((1, spec.N), dtype=torch.int32, device="cuda")))
        inputs.append((xo, codes, a_ref))
    bl.bitlinear_quantize_act_grouped(xs, outs)
    bl.bitlinear_forward_grouped(problems)
    for p, (xo, codes, a_ref) in zip(problems, inputs):
        rows = np.arange(codes.shape[0])  # M = 1: every row is cheap for the oracle
        check_sampled(p["x_q"], p["beta"], p["acc_out"], p["y"], xo, codes, a_ref, rows)


@pytest.fixture(scope="module", params=[(8192, 28672), (28672, 8192)], ids=["K8192_N28672", "K28672_N8192"])
def weights_100b(request):
    K, N = request.param
    spec = workloads.batched_decode_100b(K, N, 1)
    W = synth.weights(spec.seed, N, K, spec.w_std)
    out = quantize_both(W)
    del W
    return (K, N) + out


@pytest.mark.parametrize("M", [1, 2, 4, 8, 16, 32, 64])
def test_100b_batched_decode(weights_100b, M):
    K, N, packed, alpha, codes, a_ref = weights_100b
    spec = workloads.batched_decode_100b(K, N, M)
    x = synth.activations(spec.x_seed, M, K)
    xd, xo = as_input(x, "bf16")
    xq, beta = bl.bitlinear_quantize_act(xd)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    y = bl.bitlinear_forward(xq, beta, packed, alpha, N, acc_out=acc)
    check_sampled(xq, beta, acc, y, xo, codes, a_ref, sample_rows(N, M))


@pytest.mark.parametrize("K,N", [(4096, 4096), (4096, 11008), (11008, 4096)])
def test_prefill_2048(K, N):
    spec = workloads.prefill(K, N)
    W = synth.weights(spec.seed, N, K, spec.w_std)
    packed, alpha, codes, a_ref = quantize_both(W)
    x = synth.activations(spec.x_seed, spec.M, K, outliers=True)
    xd, xo = as_input(x, "bf16")
    xq, beta = bl.bitlinear_quantize_act(xd)
    acc = torch.empty((spec.M, N), dtype=torch.int32, device="cuda")
    y = bl.bitlinear_forward(xq, beta, packed, alpha, N, acc_out=acc)
    check_sampled(xq, beta, acc, y, xo, codes, a_ref, sample_rows(N, K, n=48))


@pytest.mark.parametrize("M", [1, 2, 4, 8, 16, 32, 64])
def test_100b_bench_call_graph_rotating_replicas(weights_100b, M):
    """The call the benchmark times for the 100B sweep: one
    bitlinear_linear_grouped problem flagged BL_LINEAR_WEIGHTS_STATIC, two
    steps in one CUDA graph over two weight replicas, a new input per step."""
    K, N, packed, alpha, codes, a_ref = weights_100b
    spec = workloads.batched_decode_100b(K, N, M)
    replicas = [packed, packed.clone()]
    steps = []
    for st in range(2):
        xb = synth.f32_to_bf16_bits(synth.activations(spec.x_seed + 1000 * st, M, K))
        xd = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).cuda()
        p = dict(x=xd, x_q=torch.empty((M, K), dtype=torch.int8, device="cuda"),
                 beta=torch.empty(M, dtype=torch.float32, device="cuda"), W_packed=replicas[st], alpha=alpha, N=N,
                 y=torch.empty((M, N), dtype=torch.float32, device="cuda"),
                 acc_out=torch.empty((M, N), dtype=torch.int32, device="cuda"))
        steps.append((xb, p, bl.make_linear_problems([p])))
    L = bl.lib()
    stream = torch.cuda.Stream()

    def call(st):
        bl.check(L.bitlinear_linear_grouped(steps[st][2], 1, bl.BL_BF16, bl.BL_LINEAR_WEIGHTS_STATIC,
                                            stream.cuda_stream), "bitlinear_linear_grouped")

    with torch.cuda.stream(stream):
        call(0)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        call(0)
        call(1)
    with torch.cuda.stream(stream):
        g.replay()
    stream.synchronize()
    assert bl.bitlinear_device_error() == 0
    for st, (xb, p, _) in enumerate(steps):
        check_sampled(p["x_q"], p["beta"], p["acc_out"], p["y"], xb, codes, a_ref, sample_rows(N, 31 * M + st))
    del g

"""Parity of the exact calls bench.py times, at their full size and call shape.

Decode: one ``bitlinear_linear_grouped`` call over the seven linears of a
7B-shaped decoder layer at one token (bf16 inputs with 0.1 % ×20 outlier
channels), flagged ``BL_LINEAR_WEIGHTS_STATIC`` so that the product kernel
quantises its own inputs in its prologue and is chained to the previous step
by programmatic dependent launch; several steps are captured in one CUDA graph
over rotating weight replicas, with a different input in every step.  Every
x̃, β, int32 accumulator and output of every step is checked against the
oracle's forward ("1.58-bit 大模型极限量化实战", chenxutan.com/d/5049.html §4.2,
inference path): integers bit-exact, y within 1e-5 relative.

Prefill: one grouped ``bitlinear_linear_grouped`` call over the three M = 2048
shapes (the act-quant kernel, then one tensor-core GEMM launch over all three
matrices), two steps in one CUDA graph; every x̃ and β is checked, and the
products on every row of one full 128-row tile per shape plus sampled rows.
"""
import re

import numpy as np
import pytest
import torch

import bitlinear_w1_a8_03_b200 as bl
import oracle
from bitlinear_w1_a8_03_b200 import synth, workloads
from tests.gpu_util import np_

pytestmark = pytest.mark.gpu


def _bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _weights(spec):
    W = synth.weights(spec.seed, spec.N, spec.K, spec.w_std)
    packed, alpha = bl.bitlinear_quantize_weights(torch.from_numpy(W).cuda())
    p_ref, a_ref, codes = oracle.quantize_weights(W)
    assert np_(alpha)[0] == a_ref
    assert np.array_equal(np_(packed), p_ref)
    return packed, alpha, codes, a_ref


def _kernel_names(fn):
    """Names of the CUDA kernels one eager call of fn launches."""
    from torch.profiler import ProfilerActivity, profile
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        fn()
        torch.cuda.synchronize()
    return [e.name for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA]


def _check_y(y, y_ref):
    y = y.astype(np.float64)
    assert np.all(np.abs(y - y_ref) <= 1e-5 * np.abs(y_ref) + 1e-37)


def test_decode_7b_fused_static_graph_rotating_replicas():
    specs = workloads.decode_7b_layer_set(M=1)
    R, S = 2, 4  # weight replicas, graph steps
    base = [_weights(s) for s in specs]
    packed = [[b[0] for b in base]] + [[b[0].clone() for b in base] for _ in range(R - 1)]
    steps = []
    for st in range(S):
        xs = [synth.f32_to_bf16_bits(synth.activations(s.x_seed + 1000 * st, 1, s.K, outliers=True)) for s in specs]
        probs = []
        for i, s in enumerate(specs):
            probs.append(dict(x=_bf16_dev(xs[i]).view(1, s.K),
                              x_q=torch.empty((1, s.K), dtype=torch.int8, device="cuda"),
                              beta=torch.empty(1, dtype=torch.float32, device="cuda"),
                              W_packed=packed[st % R][i], alpha=base[i][1], N=s.N,
                              y=torch.empty((1, s.N), dtype=torch.float32, device="cuda"),
                              acc_out=torch.empty((1, s.N), dtype=torch.int32, device="cuda") if st < 2 else None))
        steps.append((xs, probs, bl.make_linear_problems(probs)))
    L = bl.lib()
    stream = torch.cuda.Stream()
    sh = stream.cuda_stream

    def call(st):
        bl.check(L.bitlinear_linear_grouped(steps[st][2], len(specs), bl.BL_BF16, bl.BL_LINEAR_WEIGHTS_STATIC, sh),
                 "bitlinear_linear_grouped")

    with torch.cuda.stream(stream):
        for st in range(S):  # eager warm-up, as the benchmark does
            call(st)
    stream.synchronize()
    # the auto rule must pick the single fused launch for this call
    with torch.cuda.stream(stream):
        names = _kernel_names(lambda: call(0))
    # the last template argument is the prologue mode: 1 = quantise x in the kernel
    assert len(names) == 1 and re.search(r"gemv_stream_kernel<1,[^>]*, 1>", names[0]), names
    for _, probs, _ in steps:  # outputs of the graph run must not be the warm-up's
        for p in probs:
            p["y"].fill_(float("nan"))
            p["x_q"].fill_(0)
            p["beta"].fill_(-1.0)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for st in range(S):
            call(st)
    with torch.cuda.stream(stream):
        g.replay()
    stream.synchronize()
    assert bl.bitlinear_device_error() == 0
    for st, (xs, probs, _) in enumerate(steps):
        for i, s in enumerate(specs):
            codes, a_ref = base[i][2], base[i][3]
            xq_r, beta_r, acc_r, y_r = oracle.forward(xs[i].reshape(1, s.K), codes, a_ref, threads=8)
            p = probs[i]
            assert np.array_equal(np_(p["x_q"]), xq_r), (st, s.name)
            assert np.array_equal(np_(p["beta"]), beta_r), (st, s.name)
            if p["acc_out"] is not None:
                assert np.array_equal(np_(p["acc_out"]), acc_r), (st, s.name)
            _check_y(np_(p["y"]), y_r)
    del g


def test_prefill_grouped_three_shapes_graph():
    specs = [workloads.prefill(4096, 4096), workloads.prefill(4096, 11008), workloads.prefill(11008, 4096)]
    base = [_weights(s) for s in specs]
    S = 2
    steps = []
    for st in range(S):
        xs = [synth.f32_to_bf16_bits(synth.activations(s.x_seed + 1000 * st, s.M, s.K, outliers=True)) for s in specs]
        probs = [dict(x=_bf16_dev(xs[i]), x_q=torch.empty((s.M, s.K), dtype=torch.int8, device="cuda"),
                      beta=torch.empty(s.M, dtype=torch.float32, device="cuda"), W_packed=base[i][0],
                      alpha=base[i][1], N=s.N, y=torch.empty((s.M, s.N), dtype=torch.float32, device="cuda"),
                      acc_out=torch.empty((s.M, s.N), dtype=torch.int32, device="cuda"))
                 for i, s in enumerate(specs)]
        steps.append((xs, probs, bl.make_linear_problems(probs)))
    L = bl.lib()
    stream = torch.cuda.Stream()
    sh = stream.cuda_stream

    def call(st):
        bl.check(L.bitlinear_linear_grouped(steps[st][2], len(specs), bl.BL_BF16, bl.BL_LINEAR_WEIGHTS_STATIC, sh),
                 "bitlinear_linear_grouped")

    with torch.cuda.stream(stream):
        call(0)
    stream.synchronize()
    with torch.cuda.stream(stream):
        names = _kernel_names(lambda: call(0))
    # the act quant runs as one launch per CTA size (here the 4096- and the
    # 11008-wide inputs), then one grouped tensor-core GEMM
    assert len(names) == 3 and all("act_quant_kernel" in n for n in names[:2]), names
    assert "gemm_tc_kernel<256>" in names[2], names
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for st in range(S):
            call(st)
    with torch.cuda.stream(stream):
        g.replay()
    stream.synchronize()
    assert bl.bitlinear_device_error() == 0
    rng = np.random.default_rng(7)
    for st, (xs, probs, _) in enumerate(steps):
        for i, s in enumerate(specs):
            codes, a_ref = base[i][2], base[i][3]
            p = probs[i]
            xq_r, beta_r = oracle.quantize_act(xs[i])
            assert np.array_equal(np_(p["x_q"]), xq_r), (st, s.name)
            assert np.array_equal(np_(p["beta"]), beta_r), (st, s.name)
            tiles = (s.N + 127) // 128
            t = (st + i) % tiles  # a different full tile per step and shape
            rows = np.unique(np.concatenate([np.arange(128 * t, min(s.N, 128 * t + 128)), [s.N - 1],
                                             rng.choice(s.N, size=48, replace=False)]))
            acc_r = oracle.ternary_matmul(xq_r, codes[rows], threads=8)
            y_r = oracle.dequant(acc_r, beta_r, a_ref)
            assert np.array_equal(np_(p["acc_out"])[:, rows], acc_r), (st, s.name)
            _check_y(np_(p["y"])[:, rows], y_r)
    del g


def test_linear_grouped_host_7b_decode_set_two_streams():
    """The end-to-end call the benchmark times: bitlinear_linear_grouped_host
    copies x from pinned host memory, runs the seven 7B linears and copies y
    back to pinned host memory.  Two steps on two streams with their own
    buffers; problem 1 reads problem 0's input (copied once), the others lie
    back to back (merged copies).  Every y equals the oracle's forward within
    1e-5, and x_q, β the oracle's quantisation."""
    specs = workloads.decode_7b_layer_set(M=1)
    assert specs[0].K == specs[1].K
    base = [_weights(s) for s in specs]
    L = bl.lib()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    own = [i for i in range(len(specs)) if i != 1]
    k_tot = sum(specs[i].K for i in own)
    n_tot = sum(s.N for s in specs)
    steps = []
    for st in range(2):
        bits = {i: synth.f32_to_bf16_bits(synth.activations(specs[i].x_seed + 500 * st, 1, specs[i].K, outliers=True))
                for i in own}
        x_host = torch.from_numpy(np.concatenate([bits[i].reshape(-1) for i in own]).view(np.int16)).view(
            torch.bfloat16).pin_memory()
        y_host = torch.full((n_tot,), float("nan"), dtype=torch.float32).pin_memory()
        x_dev = torch.empty(k_tot, dtype=torch.bfloat16, device="cuda")
        y_dev = torch.empty(n_tot, dtype=torch.float32, device="cuda")
        off, ox = {}, 0
        for i in own:
            off[i] = ox
            ox += specs[i].K
        off[1] = off[0]
        bits[1] = bits[0]
        probs, io, oy = [], [], 0
        for i, s in enumerate(specs):
            probs.append(dict(x=x_dev[off[i]:off[i] + s.K].view(1, s.K),
                              x_q=torch.empty((1, s.K), dtype=torch.int8, device="cuda"),
                              beta=torch.empty(1, dtype=torch.float32, device="cuda"), W_packed=base[i][0],
                              alpha=base[i][1], N=s.N, y=y_dev[oy:oy + s.N].view(1, s.N)))
            io.append((x_host[off[i]:off[i] + s.K], y_host[oy:oy + s.N]))
            oy += s.N
        arr, hio = bl.make_linear_problems(probs), bl.make_host_io(io)
        bl.bitlinear_linear_grouped_host(arr, hio, bl.BL_BF16, bl.BL_LINEAR_WEIGHTS_STATIC, streams[st])
        steps.append((bits, probs, y_host))
    torch.cuda.synchronize()
    assert bl.bitlinear_device_error() == 0
    for bits, probs, y_host in steps:
        oy = 0
        for i, s in enumerate(specs):
            xq_r, beta_r, _, y_r = oracle.forward(bits[i].reshape(1, s.K), base[i][2], base[i][3], threads=8)
            assert np.array_equal(np_(probs[i]["x_q"]), xq_r) and np.array_equal(np_(probs[i]["beta"]), beta_r)
            y = y_host[oy:oy + s.N].numpy().astype(np.float64).reshape(1, s.N)
            assert np.all(np.abs(y - y_r) <= 1e-5 * np.abs(y_r) + 1e-37), s.name
            oy += s.N

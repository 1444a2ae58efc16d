"""Pins for the CPU oracle: each check comes from the pages or from mathematics,
never from the oracle itself, and each is chosen so that a plausible slip in
the oracle (dropped term, wrong sign, wrong index, wrong rounding) fails it.

Pages: [BitNet 三值权重实战] = "1.58-bit 大模型极限量化实战：从 BitNet 三值权重
到单颗 CPU 跑起 100B 模型" (chenxutan.com/d/5049.html); [1.58 位大模型] =
nxmr.cn/news/148658.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from bitlinear_w1_a8_03_b200 import synth


def f32(v):
    return np.asarray(v, dtype=np.float32)


# ---------------------------------------------------------------- worked example
def test_worked_example_alpha_and_codes(golden):
    """[BitNet 三值权重实战] §2.6: α = 0.6125, codes [1, 0, 0, -1], 50% zeros."""
    g = golden("worked_example.txt")
    W = f32(g["W"]).reshape(1, 4)
    alpha = oracle.absmean(W)
    assert abs(float(alpha) - g["alpha"][0]) <= float(np.spacing(np.float32(0.6125)))
    q = W.astype(np.float64) / float(alpha)
    assert np.allclose(q.ravel(), g["W_over_alpha"], atol=0.006)  # page prints 2-3 digits
    codes = oracle.ternarize(W, alpha)
    assert codes.ravel().tolist() == [int(v) for v in g["codes"]]
    assert float(np.mean(codes == 0)) == g["zero_fraction"][0]


def test_worked_example_forward(golden):
    """Worked-example codes times the page's activation rule give acc = 254,
    and y = acc·α·β/127 within the two binary32 roundings of the dequant."""
    g = golden("worked_example.txt")
    t = golden("rounding_ties.txt")
    W = f32(g["W"]).reshape(1, 4)
    packed, alpha, codes = oracle.quantize_weights(W)
    x = f32(t["x2"]).reshape(1, 4)
    xq, beta, acc, y = oracle.forward(x, codes, alpha)
    assert xq.ravel().tolist() == [int(v) for v in t["x2_q"]]
    assert float(beta[0]) == 1.0
    assert int(acc[0, 0]) == int(t["acc_worked"][0])
    exact = 254.0 * float(alpha) * 1.0 / 127.0
    assert abs(float(y[0, 0]) - exact) <= 2 * float(np.spacing(np.float32(exact)))
    # the float path of the same example, x·Wᵀ = 0.9 + 0.15 - 0.025... sign check
    assert float(y[0, 0]) > 0 and float((x @ W.T)[0, 0]) > 0


# ---------------------------------------------------------------- rounding ties
def test_weight_ties_round_half_even(golden):
    t = golden("rounding_ties.txt")
    W = f32(t["W"]).reshape(1, 4)
    alpha = oracle.absmean(W)
    assert float(alpha) == t["W_alpha"][0]
    assert oracle.ternarize(W, alpha).ravel().tolist() == [int(v) for v in t["W_codes"]]


def test_activation_ties_round_half_even(golden):
    t = golden("rounding_ties.txt")
    x = f32(t["x"]).reshape(1, 4)
    xq, beta = oracle.quantize_act(x)
    assert float(beta[0]) == t["x_beta"][0]
    assert xq.ravel().tolist() == [int(v) for v in t["x_q"]]


# ---------------------------------------------------------------- absmean exactness
def _alpha_by_fractions(W):
    s = sum((Fraction(float(abs(v))) for v in np.asarray(W, dtype=np.float32).ravel()), Fraction(0))
    return np.float32(float(s / W.size))  # float(Fraction) is correctly rounded


@pytest.mark.parametrize("seed", range(6))
def test_absmean_equals_exact_rational_mean(seed):
    """α = RN32(RN64(mean|W|)) with the sum exact; checked against rational
    arithmetic on inputs that span many exponents, denormals and signed zeros."""
    rng = np.random.default_rng(seed)
    n = 997
    mag = rng.uniform(-149, 20, size=n)
    W = (np.sign(rng.standard_normal(n)) * np.exp2(mag)).astype(np.float32)
    W[::50] = 0.0
    W[1::50] = -0.0
    W[2::53] = np.float32(1e-45)  # smallest denormal
    assert oracle.absmean(W) == _alpha_by_fractions(W)


def test_absmean_bf16_and_f32_agree():
    x = synth.normal_f32(synth.stream_key(7, 1), 4096, 0.02)
    b = synth.f32_to_bf16_bits(x)
    assert oracle.absmean(b) == oracle.absmean(synth.bf16_bits_to_f32(b))
    assert oracle.absmean(b) == _alpha_by_fractions(synth.bf16_bits_to_f32(b))


def test_absmean_close_to_fp64_sum_large():
    W = synth.weights(11, 512, 1024, 0.02)
    ref = np.sum(np.abs(W.astype(np.float64))) / W.size
    assert abs(float(oracle.absmean(W)) - ref) <= 1e-7 * ref


def test_absmean_order_free():
    W = synth.weights(3, 64, 96, 0.02)
    perm = np.random.default_rng(0).permutation(W.size)
    assert oracle.absmean(W) == oracle.absmean(W.ravel()[perm].reshape(W.shape))


# ---------------------------------------------------------------- ternarize
def test_ternarize_constant_matrix():
    """W constant c: α = |c|, W/α = ±1 → every code is sign(c)."""
    for c in (0.37, -2.5):
        W = np.full((3, 17), c, dtype=np.float32)
        a = oracle.absmean(W)
        assert float(a) == abs(c) or abs(float(a) - abs(c)) <= np.spacing(np.float32(abs(c)))
        assert np.all(oracle.ternarize(W, a) == np.sign(c))


def test_ternarize_thresholds_match_definition():
    """Brute force: code = sign(w) if |w/α| > 0.5 (ties at exactly 0.5 go to
    0 and ties at 1.5 go to ±2 → ±1), checked in exact rational arithmetic."""
    rng = np.random.default_rng(5)
    W = (rng.standard_normal(4000) * 0.02).astype(np.float32)
    alpha = np.float32(0.015)
    codes = oracle.ternarize(W, alpha)
    for w, c in zip(W.tolist(), codes.tolist()):
        q = np.float32(w) / alpha  # one binary32 division
        fq = Fraction(float(q))
        want = 0 if abs(fq) <= Fraction(1, 2) else (1 if fq > 0 else -1)
        assert c == want


def test_zero_fraction_closed_form():
    """Gaussian W: α → σ·sqrt(2/π); P(code 0) = erf(0.5·sqrt(2/π)/sqrt(2)) ≈ 0.310,
    inside the pages' "30%-50% zeros" ([BitNet 三值权重实战] §4.3)."""
    W = synth.weights(0, 256, 256, 0.02)
    alpha = oracle.absmean(W)
    assert abs(float(alpha) / (0.02 * math.sqrt(2 / math.pi)) - 1) < 0.02
    p0 = math.erf(0.5 * math.sqrt(2 / math.pi) / math.sqrt(2))
    codes = oracle.ternarize(W, alpha)
    assert abs(float(np.mean(codes == 0)) - p0) < 0.01
    assert abs(float(np.mean(codes == 1)) - (1 - p0) / 2) < 0.01


# ---------------------------------------------------------------- packing
def decode_packed(packed, K):
    """Independent decoder of the stated layout: weight 16g+4s+b is byte b of
    32-bit word g, bits 2s..2s+1; codes 00/01/10 = -1/0/+1."""
    N, rb = packed.shape
    out = np.zeros((N, rb * 4), dtype=np.int16)
    for k in range(rb * 4):
        g, i = divmod(k, 16)
        s, b = divmod(i, 4)
        out[:, k] = (packed[:, 4 * g + b].astype(np.int16) >> (2 * s)) & 3
    return out[:, :K] - 1, out[:, K:]


def test_pack_worked_example_bytes(golden):
    g = golden("worked_example.txt")
    packed = oracle.pack(np.array([[int(v) for v in g["codes"]]], dtype=np.int8))
    assert packed.shape == (1, 16)
    # bytes 0..3 carry weights 0..3 in bits 0-1 (codes 10,01,01,00) under the
    # padding code 01 in bits 2-7; bytes 4..15 are pure padding.
    assert packed[0].tolist() == [0x56, 0x55, 0x55, 0x54] + [0x55] * 12


@pytest.mark.parametrize("K", [1, 3, 4, 5, 16, 17, 63, 64, 65, 100, 256, 260])
def test_pack_roundtrip_and_padding(K):
    rng = np.random.default_rng(K)
    codes = rng.integers(-1, 2, size=(5, K)).astype(np.int8)
    packed = oracle.pack(codes)
    assert packed.shape == (5, 16 * ((K + 63) // 64))
    dec, pad = decode_packed(packed, K)
    assert np.array_equal(dec, codes)
    assert np.all(pad == 1)  # padding is the zero code 01
    two_bit = np.stack([(packed >> (2 * s)) & 3 for s in range(4)])
    assert not np.any(two_bit == 3)  # code 11 is never written


# ---------------------------------------------------------------- activation quant
def test_act_quant_per_token_and_bounds():
    x = synth.activations(1, 9, 300, outliers=True)
    xq, beta = oracle.quantize_act(x)
    assert np.all(np.abs(xq.astype(np.int32)) <= 127)
    for m in range(9):
        assert beta[m] == np.float32(np.max(np.abs(x[m]))) + np.float32(1e-8)
        xr, br = oracle.quantize_act(x[m:m + 1])
        assert np.array_equal(xr[0], xq[m]) and br[0] == beta[m]
        assert 127 in np.abs(xq[m].astype(np.int32))  # the absmax element maps to ±127


def test_act_quant_against_torch_ops():
    """Same rounding as torch's float32 tensor ops: round(x·127/β), half to even."""
    x = synth.activations(2, 6, 515, outliers=True)
    xq, beta = oracle.quantize_act(x)
    t = torch.from_numpy(x)
    b = t.abs().amax(dim=1, keepdim=True) + 1e-8
    ref = torch.clamp(torch.round(t * 127.0 / b), -127, 127).to(torch.int8).numpy()
    assert np.array_equal(xq, ref)
    assert np.array_equal(beta, b.squeeze(1).numpy())


def test_act_quant_single_spike_and_zero_token():
    x = np.zeros((2, 40), dtype=np.float32)
    x[0, 7] = -3.25
    xq, beta = oracle.quantize_act(x)
    assert xq[0, 7] == -127 and np.count_nonzero(xq[0]) == 1
    assert np.count_nonzero(xq[1]) == 0 and beta[1] == np.float32(1e-8)


def test_act_quant_bf16_is_exact_widening():
    x = synth.activations(4, 3, 128)
    b = synth.f32_to_bf16_bits(x)
    xa, ba = oracle.quantize_act(b)
    xb, bb = oracle.quantize_act(synth.bf16_bits_to_f32(b))
    assert np.array_equal(xa, xb) and np.array_equal(ba, bb)


# ---------------------------------------------------------------- integer product
@pytest.mark.parametrize("M,N,K", [(1, 1, 1), (3, 7, 5), (4, 16, 64), (2, 9, 33)])
def test_matmul_brute_force(M, N, K):
    rng = np.random.default_rng(M * 100 + N * 10 + K)
    xq = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    codes = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    acc = oracle.ternary_matmul(xq, codes)
    ref = np.zeros((M, N), dtype=np.int64)
    for m in range(M):
        for n in range(N):
            ref[m, n] = sum(int(xq[m, k]) * int(codes[n, k]) for k in range(K))
    assert np.array_equal(acc, ref)
    dense = xq.astype(np.float64) @ codes.astype(np.float64).T  # exact in binary64
    assert np.array_equal(acc, dense)


def test_matmul_equals_page_float_emulation():
    """[BitNet 三值权重实战] §4.2 emulates the integer product with a float32
    F.linear on integer-valued tensors; while 127·K < 2^24 every partial sum is
    an exact float32 integer, so it must equal the add/sub/skip accumulator."""
    rng = np.random.default_rng(9)
    xq = rng.integers(-127, 128, size=(5, 4096)).astype(np.int8)
    codes = rng.integers(-1, 2, size=(33, 4096)).astype(np.int8)
    acc = oracle.ternary_matmul(xq, codes, threads=4)
    ref = torch.nn.functional.linear(torch.from_numpy(xq).float(), torch.from_numpy(codes).float())
    assert np.array_equal(acc, ref.numpy().astype(np.int32))


def test_matmul_extreme_magnitude():
    K = 28672
    xq = np.full((1, K), -127, dtype=np.int8)
    codes = np.full((2, K), 1, dtype=np.int8)
    codes[1] = -1
    acc = oracle.ternary_matmul(xq, codes)
    assert acc.tolist() == [[-127 * K, 127 * K]]


# ---------------------------------------------------------------- dequant and identity
def test_dequant_error_bound_and_bias():
    rng = np.random.default_rng(3)
    acc = rng.integers(-3_000_000, 3_000_000, size=(4, 50)).astype(np.int32)
    beta = np.array([0.3, 7.5, 1e-8, 40.0], dtype=np.float32)
    alpha = np.float32(0.0123)
    bias = rng.standard_normal(50).astype(np.float32)
    y = oracle.dequant(acc, beta, alpha)
    exact = acc.astype(np.float64) * (float(alpha) * beta.astype(np.float64)[:, None] / 127.0)
    # two binary32 roundings (the scale, then the product) → within 2 ulp
    assert np.all(np.abs(y - exact) <= 2 * np.spacing(np.abs(exact).astype(np.float32)) + 1e-45)
    yb = oracle.dequant(acc, beta, alpha, bias)
    assert np.array_equal(yb, (y + bias).astype(np.float32))


def test_identity_cosine_closed_form():
    """[BitNet 三值权重实战] §2.5: x·Wᵀ ≈ (β·α/127)(x̃·Ŵᵀ).  For Gaussian W the
    ternarised product has cosine 2φ(τ)/sqrt(1-erf(τ/√2)) with τ = ½·sqrt(2/π),
    about 0.887, with the float product (int8 activations change it < 0.01)."""
    tau = 0.5 * math.sqrt(2 / math.pi)
    phi = math.exp(-tau * tau / 2) / math.sqrt(2 * math.pi)
    cos_ref = 2 * phi / math.sqrt(1 - math.erf(tau / math.sqrt(2)))
    assert abs(cos_ref - 0.887) < 0.001
    W = synth.weights(0, 256, 256, 0.02)
    x = synth.activations(0, 16, 256)
    packed, alpha, codes = oracle.quantize_weights(W)
    _, _, _, y = oracle.forward(x, codes, alpha)
    yf = x.astype(np.float64) @ W.astype(np.float64).T
    cos = float(np.sum(y * yf) / np.linalg.norm(y) / np.linalg.norm(yf))
    assert abs(cos - cos_ref) < 0.03
    # magnitude: E[y_q²]/E[y²] = α²·P(ŵ≠0)/σ² = (2/π)(1 - P(code 0)) for Gaussian W
    p0 = math.erf(tau / math.sqrt(2))
    ratio_ref = math.sqrt(2 / math.pi * (1 - p0))
    assert abs(float(np.linalg.norm(y) / np.linalg.norm(yf)) / ratio_ref - 1) < 0.03

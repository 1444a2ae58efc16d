"""Pins of the oracle's rotation, scale-granularity and 4-bit-activation
functions against what the pages and the mathematics fix: hand-worked
examples (tests/golden/), the definitions written as brute force, exact
rational arithmetic, closed forms and invariants.  No expected value comes
from the CUDA library.

Rotation ("1.58-bit 大模型极限量化实战" §6.2): x·H with H block-diagonal
Sylvester Hadamard; the weights take W·H/b, so the product is unchanged.
Granularity: per row ("1.58 位大模型" §3.1, §4.2) and per block of 128 input
features (2kiu.com/news/4928193 §2.3, §4.2).  4-bit activations ("BitNet CPU
实测" §2.1)."""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from bitlinear_w1_a8_03_b200 import synth


def _sylvester(b):
    i = np.arange(b)
    pc = np.vectorize(lambda v: bin(v).count("1"))(i[:, None] & i[None, :])
    return np.where(pc % 2 == 0, 1, -1).astype(np.int64)


# ----------------------------------------------------------------------------- rotation
def test_hadamard_worked_example(golden):
    g = golden("hadamard_4.txt")
    x = np.array([g["x"]], dtype=np.float32)
    assert np.array_equal(oracle.hadamard(x, 4)[0], np.float32(g["xH_block4"]))
    assert np.array_equal(oracle.hadamard(x, 2)[0], np.float32(g["xH_block2"]))
    w = oracle.hadamard(x, 4, 0.25)[0]
    assert np.array_equal(w, np.float32(g["wH_block4"]))
    assert float(np.dot(oracle.hadamard(x, 4)[0].astype(np.float64), w)) == g["dot"][0]


@pytest.mark.parametrize("block,K", [(1, 5), (2, 6), (8, 24), (64, 128), (512, 512), (4096, 8192)])
def test_hadamard_equals_definition_on_integers(block, K):
    """Small integers keep every partial sum exact in binary32, so the
    butterfly must equal Σ_i x_i·(-1)^popcount(i & j) per block exactly."""
    rng = np.random.default_rng(block + K)
    x = rng.integers(-1000, 1001, size=(3, K)).astype(np.float32)
    got = oracle.hadamard(x, block)
    H = _sylvester(block) if block <= 512 else None
    for m in range(3):
        for s in range(0, K, block):
            seg = x[m, s:s + block].astype(np.int64)
            if H is not None:
                ref = seg @ H
            else:  # large block: a few outputs from the definition
                js = rng.choice(block, size=16, replace=False)
                pc = np.array([[bin(i & j).count("1") & 1 for j in js] for i in range(block)])
                ref_js = seg @ np.where(pc == 0, 1, -1)
                assert np.array_equal(got[m, s + js].astype(np.int64), ref_js)
                continue
            assert np.array_equal(got[m, s:s + block].astype(np.int64), ref)


@pytest.mark.parametrize("b", [2, 16, 128])
def test_hadamard_orthogonal_and_involutive(b):
    """The rows of the identity rotate to the rows of H: H·Hᵀ = b·I; rotating
    twice gives b·x, and the weight-side scale 1/b undoes it exactly."""
    H = oracle.hadamard(np.eye(b, dtype=np.float32), b).astype(np.int64)
    assert np.array_equal(H @ H.T, b * np.eye(b, dtype=np.int64))
    rng = np.random.default_rng(b)
    x = rng.integers(-50, 51, size=(2, 4 * b)).astype(np.float32)
    twice = oracle.hadamard(oracle.hadamard(x, b), b)
    assert np.array_equal(twice, b * x)
    assert np.array_equal(oracle.hadamard(oracle.hadamard(x, b), b, 1.0 / b), x)


@pytest.mark.parametrize("block", [128, 4096])
def test_hadamard_float_error_bound_and_parseval(block):
    """On real data the binary32 network is within log2(b)·2^-24·Σ|x| (plus
    second order) of the exact transform, and ‖xH‖² = b‖x‖²."""
    K = 2 * block
    x = synth.activations(5, 4, K, outliers=True)
    got = oracle.hadamard(x, block).astype(np.float64)
    d = int(np.log2(block))
    for m in range(4):
        for s in range(0, K, block):
            seg = x[m, s:s + block].astype(np.float64)
            exact = np.array([np.sum(seg * (1 - 2 * (np.vectorize(lambda i: bin(i & j).count('1') & 1)(np.arange(block)))))
                              for j in range(0, block, max(1, block // 32))])
            bound = 1.01 * d * 2.0 ** -24 * np.sum(np.abs(seg))
            assert np.all(np.abs(got[m, s:s + block:max(1, block // 32)] - exact) <= bound)
        assert abs(np.sum(got[m] ** 2) / (block * np.sum(x[m].astype(np.float64) ** 2)) - 1) < 1e-5


def test_rotation_keeps_the_product():
    """(x·H)·(W·H/b)ᵀ = x·Wᵀ: the weight side uses the same H and 1/b."""
    K, N, b = 256, 8, 128
    x = synth.activations(1, 3, K).astype(np.float64)
    W = synth.weights(2, N, K, 0.02).astype(np.float64)
    xr = oracle.hadamard(x.astype(np.float32), b).astype(np.float64)
    Wr = oracle.hadamard(W.astype(np.float32), b, 1.0 / b).astype(np.float64)
    ref = x @ W.T
    assert np.allclose(xr @ Wr.T, ref, rtol=0, atol=1e-5 * np.abs(x).sum() * np.abs(W).max())


def test_rotation_tames_outliers():
    """The reason for the rotation: with 0.1 % ×20 outlier channels, the int8
    quantisation error of a token is far smaller after rotating it."""
    K = 4096
    x = synth.activations(7, 8, K, outliers=True)
    xq, beta = oracle.quantize_act(x)
    plain = xq.astype(np.float64) * (beta[:, None] / 127.0)
    err_plain = np.linalg.norm(plain - x, axis=1)
    xq_r, beta_r, _ = oracle.quantize_act_rotated(x, K)
    back = oracle.hadamard((xq_r.astype(np.float64) * (beta_r[:, None] / 127.0)).astype(np.float32), K, 1.0 / K)
    err_rot = np.linalg.norm(back.astype(np.float64) - x, axis=1)
    assert np.all(err_rot < 0.5 * err_plain)


def test_hadamard_block_rule():
    assert oracle.hadamard_block(4096) == 4096
    assert oracle.hadamard_block(11008) == 256  # 11008 = 2^8·43
    assert oracle.hadamard_block(28672) == 4096
    assert oracle.hadamard_block(16384) == 8192
    assert oracle.hadamard_block(7) == 1


# ----------------------------------------------------------------------------- granularity
def _exact_mean(vals):
    s = sum(Fraction(abs(float(v))) for v in vals)
    return np.float32(float(s / len(vals)))  # Fraction → float rounds correctly to binary64


@pytest.mark.parametrize("group", [1, 3, 64, 128, 1000])
def test_absmean_groups_exact(group):
    rng = np.random.default_rng(group)
    K = 300 if group < 1000 else 1000
    W = (rng.standard_normal((3, K)) * 0.02).astype(np.float32)
    W[0, :5] = np.float32(1e-45)   # denormals
    W[1, 7] = np.float32(3e38)     # a huge value next to small ones
    W[2, ::7] = 0.0
    a = oracle.absmean_groups(W, group)
    G = -(-K // group)
    assert a.shape == (3, G)
    for n in range(3):
        for g in range(G):
            assert a[n, g] == _exact_mean(W[n, g * group:(g + 1) * group]), (n, g)


def test_absmean_groups_double_rounding():
    """α is the exact mean rounded to binary64, then to binary32.  Three values
    whose exact mean m lies 5.6e-22 below a binary32 midpoint: RN64(m) is the
    midpoint itself, and RN32 of it is the even neighbour above, while a
    truncating or directly rounding mean gives the neighbour below.  (Built by
    taking x + y just short of 3·midpoint by one ulp of y and filling that gap
    with z, one binary32 ulp short of it.)"""
    x, y, z = 2.209782838821411, 3.8743016261832963e-07, 2.8421707736338113e-14
    W = np.array([[x, y, z]], dtype=np.float32)
    assert [float(v) for v in W[0]] == [x, y, z]
    m = (Fraction(x) + Fraction(y) + Fraction(z)) / 3
    spec = np.float32(float(m))                    # RN32(RN64(m))
    below = np.nextafter(spec, np.float32(0))
    assert Fraction(float(below)) < m < Fraction(float(spec))
    assert m - Fraction(float(below)) < Fraction(float(spec)) - m  # m is nearer the value below
    assert oracle.absmean_groups(W, 3)[0, 0] == spec


def test_absmean_groups_whole_row_equals_tensor_mean():
    W = synth.weights(3, 1, 777, 0.02)
    assert oracle.absmean_groups(W, 777)[0, 0] == oracle.absmean(W)
    assert oracle.absmean_groups(W, 10 ** 6)[0, 0] == oracle.absmean(W)


def test_per_row_worked_example():
    """Per-row α ([1.58 位大模型] §3.1: the row's mean |w|): the pages' worked
    row [0.9, -0.3, 0.05, -1.2] next to the tie row [0.25, 0.75, -0.25, -0.75]."""
    W = np.array([[0.9, -0.3, 0.05, -1.2], [0.25, 0.75, -0.25, -0.75]], dtype=np.float32)
    a = oracle.absmean_groups(W, 4)
    assert a[0, 0] == np.float32(0.6125) and a[1, 0] == np.float32(0.5)
    assert np.array_equal(oracle.ternarize_groups(W, a, 4), [[1, 0, 0, -1], [0, 1, 0, -1]])


def test_ternarize_groups_uses_each_groups_alpha():
    """Element k of row n is divided by α[n][k // group] (not k % G, not the
    column's)."""
    N, K, group = 2, 12, 4
    alpha = np.array([[1.0, 2.0, 4.0], [8.0, 16.0, 32.0]], dtype=np.float32)
    W = np.repeat(alpha, group, axis=1) * np.float32(0.6)   # W/α = 0.6 everywhere → +1
    W[:, 1::group] *= np.float32(0.5)                        # W/α = 0.3 → 0
    codes = oracle.ternarize_groups(W, alpha, group)
    expect = np.ones((N, K), dtype=np.int8)
    expect[:, 1::group] = 0
    assert np.array_equal(codes, expect)


def test_forward_groups_closed_form():
    """Power-of-two group scales and small integer activations keep every step
    exact, so y = RN32(RN32(Σ_b α_b·Σ_{k∈b} x̃·ŵ)·RN32(β/127)) can be written down."""
    K, group = 8, 4
    xq = np.array([[3, -2, 5, 1, 7, 0, -4, 2]], dtype=np.int8)
    codes = np.array([[1, 1, -1, 0, -1, 1, 0, 1], [0, -1, 1, 1, 1, 1, 1, 1]], dtype=np.int8)
    alpha = np.array([[0.5, 2.0], [0.25, 4.0]], dtype=np.float32)
    beta = np.array([127.0], dtype=np.float32)  # s = 1 exactly
    y = oracle.forward_groups(xq, beta, codes, alpha, group)
    # row 0: blocks (3 - 2 - 5) = -4 and (-7 + 0 + 2) = -5 → 0.5·-4 + 2·-5 = -12
    # row 1: blocks (2 + 5 + 1) = 8 and (7 + 0 - 4 + 2) = 5 → 0.25·8 + 4·5 = 22
    assert np.array_equal(y, np.array([[-12.0, 22.0]], dtype=np.float32))


def test_forward_groups_against_dense_float64():
    M, N, K, group = 3, 5, 384, 128
    W = synth.weights(9, N, K, 0.02)
    x = synth.activations(9, M, K)
    _, alpha, codes = oracle.quantize_weights_groups(W, group)
    xq, beta = oracle.quantize_act(x)
    y = oracle.forward_groups(xq, beta, codes, alpha, group).astype(np.float64)
    wdq = codes.astype(np.float64) * np.repeat(alpha.astype(np.float64), group, axis=1)
    S = xq.astype(np.float64) @ wdq.T
    s = (beta.astype(np.float64) / 127.0).astype(np.float32).astype(np.float64)
    ref = S * s[:, None]
    assert np.all(np.abs(y - ref) <= 3 * 2.0 ** -24 * np.abs(ref) + 1e-30)


def test_per_row_forward_is_the_integer_product_scaled():
    """With one group per row: y = RN32(RN32(α_n·acc)·s_m), acc from the
    add/subtract/skip product."""
    M, N, K = 2, 6, 200
    W = synth.weights(4, N, K, 0.02)
    x = synth.activations(4, M, K)
    _, alpha, codes = oracle.quantize_weights_groups(W, K)
    xq, beta = oracle.quantize_act(x)
    acc = oracle.ternary_matmul(xq, codes)
    s = np.float32(beta.astype(np.float64) / 127.0)
    ref = (acc.astype(np.float32) * alpha[:, 0][None, :]).astype(np.float32) * s[:, None]
    assert np.array_equal(oracle.forward_groups(xq, beta, codes, alpha, K), ref.astype(np.float32))


def test_finer_scales_fit_uneven_rows_better():
    """Rows whose blocks differ in spread: per-block scales quantise the weights
    with less error than per-row, and per-row less than per-tensor."""
    rng = np.random.default_rng(11)
    N, K = 16, 1024
    spread = np.exp(rng.uniform(-2, 2, size=(N, K // 128)))
    W = (rng.standard_normal((N, K)) * np.repeat(spread, 128, axis=1) * 0.02).astype(np.float32)

    def err(group):
        _, a, c = oracle.quantize_weights_groups(W, group)
        dq = c.astype(np.float64) * np.repeat(a.astype(np.float64), group, axis=1)[:, :K]
        return np.linalg.norm(dq - W)
    a_t = oracle.absmean(W)
    c_t = oracle.ternarize(W, a_t)
    e_tensor = np.linalg.norm(c_t.astype(np.float64) * float(a_t) - W)
    assert err(128) < err(K) < e_tensor


# ----------------------------------------------------------------------------- 4-bit activations
def test_act_int4_ties_and_packing(golden):
    g = golden("act_int4_ties.txt")
    x = np.array([g["x"]], dtype=np.float32)
    xq4, beta = oracle.quantize_act_a4(x)
    assert beta[0] == np.float32(g["beta"][0])
    assert np.array_equal(oracle.unpack_a4(xq4, 5)[0], np.int8(g["xq"]))
    assert np.array_equal(xq4[0], np.uint8(g["packed"]))


def test_act_int4_bounds_spike_and_roundtrip():
    rng = np.random.default_rng(3)
    x = synth.activations(3, 5, 301, outliers=True)
    x[2] = 0.0
    x[3] = 0.0
    x[3, 17] = -2.5
    xq4, beta = oracle.quantize_act_a4(x)
    q = oracle.unpack_a4(xq4, 301)
    assert np.all(np.abs(q) <= 7)
    assert not np.any(q[2]) and beta[2] == np.float32(1e-8)
    assert q[3, 17] == -7 and np.count_nonzero(q[3]) == 1
    assert np.all(xq4[:, -1] >> 4 == 0)  # odd K: the last high nibble is zero
    # every value within half a step of x·7/β
    assert np.all(np.abs(q - x * 7.0 / beta[:, None]) <= 0.5 + 1e-5)
    vals = rng.integers(-7, 8, size=(4, 64)).astype(np.int8)
    packed = (vals[:, 0::2].astype(np.uint8) & 15) | ((vals[:, 1::2].astype(np.uint8) & 15) << 4)
    assert np.array_equal(oracle.unpack_a4(packed, 64), vals)


def test_act_int4_forward_worked_example():
    """The pages' worked weights with x = [1, 0.5, -0.5, -1]: β = 1 + 1e-8 = 1,
    x̃ = [7, 4, -4, -7] (3.5 rounds to 4 either way), acc = 7 + 7 = 14,
    y = 14·RN32(0.6125·1/7)."""
    W = np.array([[0.9, -0.3, 0.05, -1.2]], dtype=np.float32)
    _, alpha, codes = oracle.quantize_weights(W)
    xq4, beta, acc, y = oracle.forward_a4(np.array([[1.0, 0.5, -0.5, -1.0]], dtype=np.float32), codes, alpha)
    assert np.array_equal(oracle.unpack_a4(xq4, 4), [[7, 4, -4, -7]])
    assert acc[0, 0] == 14
    assert y[0, 0] == np.float32(14.0) * np.float32(float(Fraction(float(np.float32(0.6125))) / 7))

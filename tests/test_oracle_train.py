"""Pins of the oracle's training step with the straight-through estimator
("1.58-bit 大模型极限量化实战" §3.3 and §6.3; "1.58 位大模型" §3.4): the forward
quantises the latent weights afresh, the backward passes the gradient
straight through the quantisers except for weights outside the clip range.

Independent checks: the pages' worked layer (tests/golden/ste_worked_example.txt),
finite differences of the dequantised layer (a linear map, so a central
difference in binary64 is exact up to rounding), the clip mask against its
definition, linearity in g, and planted mistakes."""
import ctypes
import shutil
import subprocess
from fractions import Fraction

import numpy as np
import pytest

import oracle
from bitlinear_w1_a8_03_b200 import synth
from tests.conftest import read_golden


def test_ste_worked_example(golden):
    d = golden("ste_worked_example.txt")
    W = np.array([d["W"]], dtype=np.float32)
    x = np.array([d["x"]], dtype=np.float32)
    g = np.array([d["g"]], dtype=np.float32)
    y, gx, gw, alpha, codes, xq, beta = oracle.train_step(W, x, g)
    assert alpha == np.float32(0.6125) and np.array_equal(codes, [[1, 0, 0, -1]])
    assert np.array_equal(gx[0], np.float32(d["grad_x"]))
    s = np.float32(1.0 / 127.0)  # β = 1
    want = [np.float32(v * s) * 2 if v else 0.0 for v in (0, 64, -64, 0)]
    assert np.array_equal(gw[0], np.float32(want))
    assert abs(float(gw[0, 1]) - d["grad_W_num"][1] / d["grad_W_den"][0]) < 1e-6


def _dequant(codes, alpha, xq, beta):
    Wd = codes.astype(np.float64) * float(alpha)
    s = np.float32(beta.astype(np.float64) / 127.0).astype(np.float64)
    Xd = xq.astype(np.float64) * s[:, None]
    return Wd, Xd


def test_ste_gradients_are_finite_differences_of_the_dequantised_layer():
    """L(Xd, Wd) = Σ g ⊙ (Xd·Wdᵀ) is linear in each argument, so a central
    difference gives its derivative exactly up to rounding: ∂L/∂x through the
    STE is ∂L/∂Xd, and ∂L/∂W is ∂L/∂Wd where the weight is inside the clip range."""
    M, N, K = 3, 5, 7
    rng = np.random.default_rng(1)
    W = synth.weights(3, N, K, 0.02)
    W[0, 0] = 0.2  # far outside the clip range
    x = synth.activations(3, M, K)
    g = rng.standard_normal((M, N)).astype(np.float32)
    y, gx, gw, alpha, codes, xq, beta = oracle.train_step(W, x, g)
    Wd, Xd = _dequant(codes, alpha, xq, beta)
    L = lambda X, Wm: float(np.sum(g.astype(np.float64) * (X @ Wm.T)))
    h = 1e-3
    for m in range(M):
        for k in range(K):
            E = np.zeros_like(Xd)
            E[m, k] = h
            fd = (L(Xd + E, Wd) - L(Xd - E, Wd)) / (2 * h)
            assert abs(gx[m, k] - fd) <= 1e-6 * (1 + abs(fd)), (m, k)
    mask = np.abs(W / np.float32(alpha)) <= 1
    assert not mask[0, 0]
    for n in range(N):
        for k in range(K):
            E = np.zeros_like(Wd)
            E[n, k] = h
            fd = (L(Xd, Wd + E) - L(Xd, Wd - E)) / (2 * h)
            want = fd if mask[n, k] else 0.0
            assert abs(gw[n, k] - want) <= 1e-6 * (1 + abs(fd)), (n, k)


def test_ste_clip_mask_matches_definition():
    """Exactly the weights with |W/α| <= 1 (the forward's binary32 quotient)
    receive a gradient; the boundary W = ±α is inside."""
    N, K = 4, 64
    W = synth.weights(8, N, K, 0.02)
    alpha = oracle.absmean(W)
    W[0, 0] = alpha
    W[1, 1] = -alpha
    W[2, 2] = np.nextafter(alpha, np.float32(1))
    alpha2 = oracle.absmean(W)
    codes = oracle.ternarize(W, alpha2)
    xq = np.ones((1, K), dtype=np.int8)
    beta = np.array([127.0], dtype=np.float32)
    g = np.ones((1, N), dtype=np.float32)
    gw = oracle.ste_grad_w(g, xq, beta, W, alpha2)
    q = W / np.float32(alpha2)
    assert np.array_equal(gw != 0, np.abs(q) <= 1)
    assert np.all(gw[np.abs(q) <= 1] == np.float32(1.0))  # g·s·x̃ = 1·1·1
    # on the boundary: α = 0.5 exactly and W/α = ±1, all inside the range
    Wb = np.array([[0.5, -0.5, 0.5, -0.5]], dtype=np.float32)
    ab = oracle.absmean(Wb)
    assert ab == np.float32(0.5)
    gb = oracle.ste_grad_w(np.ones((1, 1), np.float32), np.ones((1, 4), np.int8), beta, Wb, ab)
    assert np.all(gb == np.float32(1.0))


def test_ste_linear_in_g_and_exact_scaling():
    M, N, K = 2, 6, 33
    W = synth.weights(5, N, K, 0.02)
    x = synth.activations(5, M, K)
    g = synth.activations(6, M, N)
    _, gx, gw, *_ = oracle.train_step(W, x, g)
    _, gx2, gw2, *_ = oracle.train_step(W, x, 2 * g)
    assert np.array_equal(gx2, 2 * gx) and np.array_equal(gw2, 2 * gw)


SRC_MUTANTS = [
    ("ste_mask_strict", "if (!(fabsf(q) <= 1.0f)) {", "if (!(fabsf(q) < 1.0f)) {", ["test_ste_clip_mask_matches_definition"]),
    ("ste_mask_uses_codes", "if (!(fabsf(q) <= 1.0f)) {", "if (!(fabsf(rintf(q)) <= 1.0f)) {",
     ["test_ste_worked_example", "test_ste_gradients_are_finite_differences_of_the_dequantised_layer"]),
    ("ste_grad_x_no_alpha", "gx[m * K + k] = (float)((double)alpha * s);", "gx[m * K + k] = (float)s;",
     ["test_ste_worked_example"]),
    ("ste_grad_x_wrong_sign", "else if (w == -1) s -= (double)g[m * N + n];",
     "else if (w == -1) s += (double)g[m * N + n];", ["test_ste_worked_example"]),
    ("ste_grad_w_no_beta", "double sm = (double)beta[m] / 127.0;", "double sm = 1.0 / 127.0;",
     ["test_ste_gradients_are_finite_differences_of_the_dequantised_layer"]),
    ("ste_grad_w_transposed", "s += (double)gs * (double)xq[m * K + k];", "s += (double)gs * (double)xq[m * K + (k % M)];",
     ["test_ste_gradients_are_finite_differences_of_the_dequantised_layer"]),
]


@pytest.mark.parametrize("name,orig,mut,catchers", SRC_MUTANTS, ids=[m[0] for m in SRC_MUTANTS])
def test_train_mutant_is_caught(name, orig, mut, catchers, tmp_path, monkeypatch):
    from tests.test_oracle_mutants import HDR, SRC
    src = open(SRC, encoding="utf-8").read()
    assert src.count(orig) == 1, f"mutation site for {name} not unique"
    shutil.copy(HDR, tmp_path / "bitlinear_oracle.h")
    (tmp_path / "bitlinear_oracle.c").write_text(src.replace(orig, mut), encoding="utf-8")
    so = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", *oracle.CFLAGS, "-o", str(so), str(tmp_path / "bitlinear_oracle.c"), "-lm"])
    monkeypatch.setattr(oracle, "_lib", oracle.configure(ctypes.CDLL(str(so))))
    caught = []
    for pin in catchers:
        fn = globals()[pin]
        try:
            fn(read_golden) if "golden" in fn.__code__.co_varnames[: fn.__code__.co_argcount] else fn()
        except Exception:
            caught.append(pin)
    assert caught, f"mutant {name} survived every pin in {catchers}"

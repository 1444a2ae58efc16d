"""Pins of the oracle's layer stack (the synthetic decoder-layer dataflow).

Each pin ties the composition to something outside it: an independent
recomputation of the products with float64 matrix products on tiny shapes,
the exact power-of-two scale invariance of per-token absmax quantisation, and
which of the seven products the next layer's input can depend on."""
import numpy as np
import pytest

import oracle
from bitlinear_w1_a8_03_b200 import synth

H, F = 24, 40


def _layer(seed, H=H, F=F):
    shapes = {"q": (H, H), "k": (H, H), "v": (H, H), "o": (H, H), "gate": (F, H), "up": (F, H), "down": (H, F)}
    layer = {}
    for i, name in enumerate(oracle.STACK_MATRICES):
        N, K = shapes[name]
        W = synth.weights(seed * 7 + i, N, K, 0.02)
        alpha = oracle.absmean(W)
        layer[name] = (oracle.ternarize(W, alpha), alpha)
    return layer


def _h0(M, seed=1):
    return synth.activations(seed, M, H, outliers=False)


def _product_f64(x_f32, codes, alpha):
    """x̃, β and y of one BitLinear, the product as a float64 matrix product
    of the integer codes (exact here: |acc| < 2^53)."""
    x = x_f32.astype(np.float32)
    beta = (np.abs(x).max(axis=1) + np.float32(1e-8)).astype(np.float32)
    xq = np.clip(np.rint((x * np.float32(127.0)).astype(np.float32) / beta[:, None]), -127, 127)
    acc = xq.astype(np.float64) @ codes.astype(np.float64).T
    s = (np.float64(alpha) * beta.astype(np.float64) / 127.0).astype(np.float32)
    return (acc.astype(np.float32) * s[:, None]).astype(np.float32)


def test_stack_matches_float64_recomposition():
    layers = [_layer(10), _layer(11)]
    h = _h0(3)
    outs = oracle.stack_forward(h, layers)
    for layer, o in zip(layers, outs):
        ys = {n: _product_f64(h, *layer[n]) for n in ("q", "k", "v", "gate", "up")}
        ys["o"] = _product_f64(ys["v"], *layer["o"])
        ys["down"] = _product_f64(ys["up"], *layer["down"])
        for n in oracle.STACK_MATRICES:
            assert np.array_equal(o[n], ys[n]), n
        h = (ys["o"] + ys["down"]).astype(np.float32)
        assert np.array_equal(o["h_next"], h)


@pytest.mark.parametrize("k", [3, -5])
def test_stack_scales_by_powers_of_two(k):
    """When every quantised input has max|x| ≥ 1/4, the 1e-8 in β = max|x| + 1e-8
    is below half an ulp and vanishes, so scaling h0 by 2^k leaves every x̃
    unchanged and scales every output exactly by 2^k.  (At these tiny widths
    the activations shrink ~100x per layer, hence the large h0.)"""
    layers = [_layer(20), _layer(21)]
    h = (_h0(4, seed=5) * np.float32(2.0 ** 24)).astype(np.float32)
    base = oracle.stack_forward(h, layers)
    scaled = oracle.stack_forward((h * np.float32(2.0 ** k)).astype(np.float32), layers)
    for b, s in zip(base, scaled):
        for n in ("v", "up", "h_next"):  # every quantised input of the stack
            assert np.abs(b[n]).max(axis=1).min() * min(1.0, 2.0 ** k) >= 0.25
        for n in (*oracle.STACK_MATRICES, "h_next"):
            assert np.array_equal(s[n], (b[n] * np.float32(2.0 ** k)).astype(np.float32)), n


def test_stack_output_depends_on_v_o_up_down_only():
    layer = _layer(30)
    h = _h0(2, seed=7)
    ref = oracle.stack_layer(h, layer)["h_next"]
    other = _layer(31)
    for n in ("q", "k", "gate"):
        changed = dict(layer, **{n: other[n]})
        assert np.array_equal(oracle.stack_layer(h, changed)["h_next"], ref), n
    for n in ("v", "o", "up", "down"):
        changed = dict(layer, **{n: other[n]})
        assert not np.array_equal(oracle.stack_layer(h, changed)["h_next"], ref), n


def _mutant_layer(kind):
    """A stack layer with one plausible wiring mistake planted."""
    def layer_fn(h, layer):
        h = np.ascontiguousarray(h, dtype=np.float32)
        out = {n: oracle.forward(h, *layer[n])[3] for n in ("q", "k", "v", "gate", "up")}
        src_o = out["k"] if kind == "o_reads_k" else out["v"]
        src_down = out["gate"] if kind == "down_reads_gate" else out["up"]
        out["o"] = oracle.forward(src_o, *layer["o"])[3]
        out["down"] = oracle.forward(src_down, *layer["down"])[3]
        if kind == "no_residual_down":
            out["h_next"] = out["o"].copy()
        elif kind == "sum_after_quant_of_parts":
            # quantising y_o and y_down separately and adding the dequantised
            # codes instead of quantising their float sum
            xo, bo = oracle.quantize_act(out["o"])
            xd, bd = oracle.quantize_act(out["down"])
            out["h_next"] = (xo * (bo[:, None] / np.float32(127)) + xd * (bd[:, None] / np.float32(127))
                             ).astype(np.float32)
        else:
            out["h_next"] = np.add(out["o"], out["down"], dtype=np.float32)
        return out
    return layer_fn


@pytest.mark.parametrize("kind", ["o_reads_k", "down_reads_gate", "no_residual_down", "sum_after_quant_of_parts"])
def test_stack_pins_reject_planted_wiring_mistakes(kind):
    """Each mutant disagrees with the independent float64 recomposition
    (the pin the real stack_layer passes)."""
    layer = _layer(40)
    h = _h0(3, seed=9)
    mutant = _mutant_layer(kind)(h, layer)
    ys = {n: _product_f64(h, *layer[n]) for n in ("q", "k", "v", "gate", "up")}
    ys["o"] = _product_f64(ys["v"], *layer["o"])
    ys["down"] = _product_f64(ys["up"], *layer["down"])
    h_next = (ys["o"] + ys["down"]).astype(np.float32)
    agree = all(np.array_equal(mutant[n], ys[n]) for n in oracle.STACK_MATRICES) and \
        np.array_equal(mutant["h_next"], h_next)
    assert not agree
    real = oracle.stack_layer(h, layer)
    assert all(np.array_equal(real[n], ys[n]) for n in oracle.STACK_MATRICES)
    assert np.array_equal(real["h_next"], h_next)

"""Host-side logic without a GPU: the layer stack's call wiring, the binding's
problem arrays, and the benchmark's byte accounting.  Tensors live on the
CPU; nothing here calls into the CUDA library."""
import ctypes

import numpy as np
import pytest

import torch

import bitlinear_w1_a8_03_b200 as bl
from bitlinear_w1_a8_03_b200.stack import MATRICES, LinearStack, shapes


def _cpu_layers(hidden, ffn, L):
    sh = shapes(hidden, ffn)
    layers = []
    for _ in range(L):
        layers.append({n: (torch.zeros((sh[n][0], 16 * ((sh[n][1] + 63) // 64)), dtype=torch.uint8),
                           torch.zeros(1, dtype=torch.float32)) for n in MATRICES})
    return layers


def test_stack_wiring():
    """Per layer: call 1 quantises h (layer 0: h0; later: y_o + y_down of the
    previous layer) for q, k, v, gate, up; call 2 quantises y_v and y_up for o
    and down; a last call materialises y_o + y_down into h_final."""
    hidden, ffn, L, M = 64, 128, 3, 2
    layers = _cpu_layers(hidden, ffn, L)
    st = LinearStack(layers, hidden, ffn, M, torch.device("cpu"), keep_all=True)
    assert len(st.calls) == 2 * L + 1
    assert st.launches() == 4 * L + 1
    ptr = lambda t: t.data_ptr()
    for l in range(L):
        acts1, n_a1, fwd1, n_f1 = st.calls[2 * l]
        acts2, n_a2, fwd2, n_f2 = st.calls[2 * l + 1]
        assert (n_a1, n_f1, n_a2, n_f2) == (1, 5, 2, 2)
        a = acts1[0]
        if l == 0:
            assert a.a == ptr(st.h0) and a.b is None
        else:
            assert a.a == ptr(st.y[l - 1]["o"]) and a.b == ptr(st.y[l - 1]["down"])
        assert a.x_sum == ptr(st.h_in[l]) and a.x_q == ptr(st.xq["h"]) and a.M == M and a.K == hidden
        for f, n in zip(fwd1, ("q", "k", "v", "gate", "up")):
            assert f.x_q == ptr(st.xq["h"]) and f.y == ptr(st.y[l][n])
            assert f.W_packed == ptr(layers[l][n][0]) and f.N == shapes(hidden, ffn)[n][0] and f.K == hidden
        assert acts2[0].a == ptr(st.y[l]["v"]) and acts2[0].x_q == ptr(st.xq["v"]) and acts2[0].K == hidden
        assert acts2[1].a == ptr(st.y[l]["up"]) and acts2[1].x_q == ptr(st.xq["up"]) and acts2[1].K == ffn
        assert fwd2[0].x_q == ptr(st.xq["v"]) and fwd2[0].y == ptr(st.y[l]["o"]) and fwd2[0].K == hidden
        assert fwd2[1].x_q == ptr(st.xq["up"]) and fwd2[1].y == ptr(st.y[l]["down"]) and fwd2[1].K == ffn
    acts, n_a, fwd, n_f = st.calls[-1]
    assert (n_a, n_f, fwd) == (1, 0, None)
    assert acts[0].a == ptr(st.y[L - 1]["o"]) and acts[0].b == ptr(st.y[L - 1]["down"])
    assert acts[0].x_sum == ptr(st.h_final)
    assert st.weight_bytes == L * sum(16 * ((shapes(hidden, ffn)[n][1] + 63) // 64) * shapes(hidden, ffn)[n][0]
                                      for n in MATRICES)


def test_stack_without_keep_all_reuses_buffers():
    st = LinearStack(_cpu_layers(64, 128, 2), 64, 128, 1, torch.device("cpu"))
    assert len(st.y) == 1 and st.h_in is None
    acts, _, _, _ = st.calls[2]  # layer 1 reads the shared y_o / y_down
    assert acts[0].a == st.y[0]["o"].data_ptr() and acts[0].x_sum is None


def test_problem_arrays_carry_shapes_and_pointers():
    x = torch.zeros((3, 128), dtype=torch.bfloat16)
    xq = torch.zeros((3, 128), dtype=torch.int8)
    beta = torch.zeros(3)
    W = torch.zeros((40, 32), dtype=torch.uint8)
    alpha = torch.zeros(1)
    y = torch.zeros((3, 40))
    lin = bl.make_linear_problems([dict(x=x, x_q=xq, beta=beta, W_packed=W, alpha=alpha, N=40, y=y)])
    assert (lin[0].M, lin[0].N, lin[0].K) == (3, 40, 128)
    assert lin[0].x == x.data_ptr() and lin[0].y == y.data_ptr() and lin[0].bias is None
    fwd = bl.make_forward_problems([dict(x_q=xq, beta=beta, W_packed=W, alpha=alpha, N=40, y=y)])
    assert (fwd[0].M, fwd[0].N, fwd[0].K) == (3, 40, 128) and fwd[0].acc_out is None
    acts = bl.make_act_sum_problems([dict(a=y, b=y, x_q=xq, beta=beta)])
    assert (acts[0].M, acts[0].K) == (3, 40) and acts[0].b == y.data_ptr() and acts[0].x_sum is None
    assert isinstance(acts, ctypes.Array) and len(acts) == 1


def test_decode_bytes_per_step():
    """The decode leg's algorithmic bytes: packed weights once, plus per matrix
    the act quant (bf16 x in, x̃ and β out) and the product (x̃, β in; y out)."""
    import bench
    specs = bench.workload_specs()
    w = sum(s.N * 16 * ((s.K + 63) // 64) for s in specs)
    assert w == 50_593_792
    acts = sum(2 * s.K + s.K + 4 + s.K + 4 + 4 * s.N for s in specs)
    assert bench.bytes_per_step(specs) == w + acts == 50_906_168


def test_kernel_attribute_set_once_per_device(tmp_path):
    """The opt-in shared-memory attribute is per device: the bookkeeping in
    csrc/bl_attr.h must run the setting once for each (kernel, device) pair,
    retry a failed setting, and refuse devices outside its table.  Compiled
    with the host compiler only (no CUDA)."""
    import os
    import subprocess
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    exe = str(tmp_path / "attr_once_check")
    subprocess.check_call(["g++", "-std=c++17", "-O1", "-I", os.path.join(root, "bitlinear_w1_a8_03_b200", "csrc"),
                           os.path.join(root, "tests", "native", "attr_once_check.cpp"), "-o", exe, "-pthread"])
    out = subprocess.run([exe], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout


def _exact_code(v, beta, scale):
    """clip(rint(RN(RN(scale·v) / β)), ±scale) in binary32 (the definition)."""
    a = np.float32(v) * np.float32(scale)
    return np.clip(np.rint(a / np.float32(beta)), -scale, scale)


def _fast_code(v, beta, scale):
    """The kernels' path: q = RN(v·RN(scale·RN(1/β))); t = RN(q + 1.5·2^23)
    and r = t - 1.5·2^23; r is kept when q is farther than 1e-4 from every
    half-integer, else the definition is taken.  The code is read from the
    low byte of t's bits, as the kernels do."""
    magic = np.float32(1.5 * 2.0 ** 23)
    with np.errstate(invalid="ignore", over="ignore"):
        c = np.float32(scale) * (np.float32(1.0) / np.float32(beta)) if beta < np.float32(2.0 ** 120) else np.float32(np.nan)
        q = np.float32(v) * np.float32(c)
        t = (q + magic).astype(np.float32)
        r = (t - magic).astype(np.float32)
        ok = np.abs(q - r) < np.float32(0.4999)
        exact = _exact_code(v, beta, scale)
        exact = np.where(np.isnan(exact), -scale, exact)  # fminf(fmaxf(NaN, -s), s) is -s
        t = np.where(ok, t, (exact.astype(np.float32) + magic).astype(np.float32))
    code = (t.astype(np.float32).view(np.uint32) & 0xFF).astype(np.uint8).view(np.int8).astype(np.float64)
    return code, ok


@pytest.mark.parametrize("scale", [127, 7])
def test_fast_quantisation_matches_the_definition(scale):
    """The per-element fast path of the activation quantisers (one multiply by
    a per-row factor, checked against the half-integers) gives the defined
    code for every element: random rows over many binades, rows with
    outliers, and values built to land within a few ulps of a half-integer."""
    rng = np.random.default_rng(scale)
    total = fast = 0
    for trial in range(400):
        K = 4096
        x = (rng.standard_normal(K) * np.exp2(rng.integers(-60, 60))).astype(np.float32)
        if trial % 3 == 0:
            x[rng.integers(0, K, 4)] *= np.float32(50.0)
        beta = np.float32(np.max(np.abs(x)) + np.float32(1e-8))
        if trial % 2 == 1:  # near ties: v with v·scale/β = j + 1/2 + a few ulps
            j = rng.integers(-scale, scale, K).astype(np.float64)
            t = j + 0.5 + rng.integers(-6, 7, K) * 2.0 ** -19
            x = np.clip((t * np.float64(beta) / scale), -np.float64(beta) * 0.9999999, np.float64(beta) * 0.9999999)
            x = x.astype(np.float32)
        got, ok = _fast_code(x, beta, scale)
        want = _exact_code(x, beta, scale)
        assert np.array_equal(got, want), trial
        if trial % 2 == 0:
            total += K
            fast += int(ok.sum())
    assert fast > 0.99 * total  # on ordinary rows the fast path does nearly all the work


def test_fast_quantisation_non_finite_and_huge_rows():
    for beta in (np.float32(np.inf), np.float32(np.nan), np.float32(3e38), np.float32(2.0 ** 121)):
        x = np.array([0.0, 1.0, -2.5, 3e38, -np.inf, np.nan], dtype=np.float32)
        for scale in (127, 7):
            got, _ = _fast_code(x, beta, scale)
            with np.errstate(invalid="ignore", over="ignore"):
                want = _exact_code(x, beta, scale)
            want = np.where(np.isnan(want), -scale, want)  # the kernels' clip maps NaN to -scale
            assert np.array_equal(got, want)


def test_exact_sum_limb_positions_cover_every_exponent():
    """The weight quantiser's exact Σ|W| adds |w|·2^149 (a 24-bit significand
    at bit position p = max(e, 1) - 1) into limbs p // 32 and p // 32 + 1 of a
    ten-limb (320-bit) integer, dispatching on p // 32 with cases 0 … 7.
    Every exponent field, subnormals and e = 255 included, lands in a case
    that exists, and the value's top bit stays inside the two limbs it
    touches (so no bit of any |w| is dropped)."""
    seen = set()
    for e in range(256):
        p = max(e, 1) - 1
        li = p >> 5
        assert 0 <= li <= 7 and li + 1 < 10
        top = (p & 31) + 23  # highest significand bit within the 64-bit two-limb window
        assert top < 64
        seen.add(li)
    assert seen == set(range(8))
    # a normal w = 1.0 (e = 127): 2^149 = 2^(32·4 + 21), i.e. limb 4, bit 21
    p = 127 - 1
    assert (p >> 5, (p & 31) + 23) == (3, 53)  # significand bit 23 of limb pair (3, 4) = bit 21 of limb 4

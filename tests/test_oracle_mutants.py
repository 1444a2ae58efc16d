"""Planted mistakes: each mutant is a copy of the oracle's C source with one
plausible slip, compiled on the CPU; at least one pin must fail on it.  This
shows the pins in test_oracle_pins.py constrain every step of the oracle."""
import ctypes
import os
import shutil
import subprocess

import pytest

import oracle
import tests.test_oracle_pins as pins
from tests.conftest import read_golden

SRC = os.path.join(os.path.dirname(oracle.__file__), "bitlinear_oracle.c")
HDR = os.path.join(os.path.dirname(oracle.__file__), "bitlinear_oracle.h")

# (name, original text, mutated text, pins that must catch it)
MUTANTS = [
    ("weight_round_half_away", "float r = rintf(q);", "float r = roundf(q);",
     ["test_weight_ties_round_half_even"]),
    ("act_round_half_away", "float r = rintf(t);", "float r = roundf(t);",
     ["test_activation_ties_round_half_even", "test_act_quant_against_torch_ops"]),
    ("absmean_drops_implicit_one", "if (e != 0) sig |= 0x800000u;", "",
     ["test_absmean_equals_exact_rational_mean", "test_worked_example_alpha_and_codes"]),
    ("absmean_drops_negative_terms", "float w = orc_load(W, dtype, i);",
     "float w = orc_load(W, dtype, i); if (w < 0) continue;",
     ["test_absmean_equals_exact_rational_mean", "test_worked_example_alpha_and_codes"]),
    ("matmul_wrong_sign", "else if (wr[k] == -1) s -= xr[k];", "else if (wr[k] == -1) s += xr[k];",
     ["test_matmul_brute_force", "test_worked_example_forward"]),
    ("matmul_ignores_token_row", "const int8_t* xr = xq + m * K;", "const int8_t* xr = xq;",
     ["test_matmul_brute_force"]),
    ("pack_transposed_fields", "row[4 * g + b] |= (uint8_t)(code << (2 * s));",
     "row[4 * g + s] |= (uint8_t)(code << (2 * b));", ["test_pack_worked_example_bytes"]),
    ("pack_padding_minus_one", "int code = (k < K) ? (int)codes[n * K + k] + 1 : 1;",
     "int code = (k < K) ? (int)codes[n * K + k] + 1 : 0;", ["test_pack_roundtrip_and_padding"]),
    ("act_no_epsilon", "float b = mx + 1e-8f;", "float b = mx;",
     ["test_act_quant_single_spike_and_zero_token", "test_act_quant_per_token_and_bounds"]),
    ("act_scale_128", "float t = orc_load(x, dtype, m * K + k) * 127.0f;",
     "float t = orc_load(x, dtype, m * K + k) * 128.0f;", ["test_act_quant_against_torch_ops"]),
    ("dequant_divides_by_128", "sd = sd / 127.0;", "sd = sd / 128.0;",
     ["test_dequant_error_bound_and_bias", "test_worked_example_forward"]),
    ("dequant_drops_beta", "double sd = (double)alpha * (double)beta[m];", "double sd = (double)alpha;",
     ["test_dequant_error_bound_and_bias"]),
    ("ternarize_no_clip_low", "if (r < -1.0f) r = -1.0f;", "",
     ["test_worked_example_alpha_and_codes", "test_ternarize_thresholds_match_definition"]),
]

ARGS = {
    "test_matmul_brute_force": [(3, 7, 5)],
    "test_pack_roundtrip_and_padding": [(17,)],
    "test_absmean_equals_exact_rational_mean": [(0,)],
}


@pytest.fixture(scope="module")
def workdir(tmp_path_factory):
    return tmp_path_factory.mktemp("mutants")


@pytest.mark.parametrize("name,orig,mut,catchers", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, orig, mut, catchers, workdir, monkeypatch):
    src = open(SRC, encoding="utf-8").read()
    assert src.count(orig) == 1, f"mutation site for {name} not unique"
    d = workdir / name
    d.mkdir()
    shutil.copy(HDR, d / "bitlinear_oracle.h")
    (d / "bitlinear_oracle.c").write_text(src.replace(orig, mut), encoding="utf-8")
    so = d / "libmut.so"
    subprocess.check_call(["gcc", *oracle.CFLAGS, "-o", str(so), str(d / "bitlinear_oracle.c"), "-lm"])
    monkeypatch.setattr(oracle, "_lib", oracle.configure(ctypes.CDLL(str(so))))
    caught = []
    for pin in catchers:
        fn = getattr(pins, pin)
        for args in ARGS.get(pin, [()]):
            try:
                if "golden" in fn.__code__.co_varnames[: fn.__code__.co_argcount]:
                    fn(*args, read_golden) if args else fn(read_golden)
                else:
                    fn(*args)
            except Exception:  # an assertion or a downstream error both count as caught
                caught.append(pin)
    assert caught, f"mutant {name} survived every pin in {catchers}"

"""Planted mistakes in the oracle's rotation, scale-granularity and 4-bit
functions: each mutant is a copy of the oracle's C source with one plausible
slip, compiled on the CPU; at least one pin in test_oracle_variants.py must
fail on it."""
import ctypes
import shutil
import subprocess

import pytest

import oracle
import tests.test_oracle_variants as pins
from tests.conftest import read_golden
from tests.test_oracle_mutants import HDR, SRC

MUTANTS = [
    ("hadamard_wrong_sign", "b[i + h] = p - q;", "b[i + h] = q - p;",
     ["test_hadamard_worked_example", "test_hadamard_equals_definition_on_integers"]),
    ("hadamard_wrong_partner", "float p = b[i], q = b[i + h];", "float p = b[i], q = b[(i + 2 * h) % block];",
     ["test_hadamard_equals_definition_on_integers", "test_hadamard_worked_example"]),
    ("hadamard_skips_last_stage", "for (int64_t h = 1; h < block; h <<= 1) {",
     "for (int64_t h = 1; 2 * h < block; h <<= 1) {", ["test_hadamard_worked_example"]),
    ("hadamard_ignores_blocks", "float* b = v + s;", "float* b = v;", ["test_hadamard_worked_example"]),
    ("hadamard_drops_scale", "if (scale != 1.0f)", "if (0)",
     ["test_hadamard_worked_example", "test_rotation_keeps_the_product"]),
    ("groups_alpha_wrong_index", "alpha[n * G + k / group]", "alpha[n * G + k % G]",
     ["test_ternarize_groups_uses_each_groups_alpha"]),
    ("groups_mean_full_count_for_last_group", "(uint64_t)(k1 - k0)", "(uint64_t)group",
     ["test_absmean_groups_exact"]),
    ("groups_mean_truncates", "if (round_bit && (sticky || (mant & 1ull))) {", "if (0) {",
     ["test_absmean_groups_double_rounding"]),
    ("groups_forward_drops_alpha", "S += (double)alpha[n * G + g] * (double)a;", "S += (double)a;",
     ["test_forward_groups_closed_form"]),
    ("groups_forward_divides_by_128", "double sd = (double)beta[m] / 127.0;", "double sd = (double)beta[m] / 128.0;",
     ["test_forward_groups_closed_form", "test_per_row_forward_is_the_integer_product_scaled"]),
    ("a4_scale_8", "float t = orc_load(x, dtype, m * K + k) * 7.0f;",
     "float t = orc_load(x, dtype, m * K + k) * 8.0f;", ["test_act_int4_ties_and_packing"]),
    ("a4_round_half_away", "float r4 = rintf(t);", "float r4 = roundf(t);", ["test_act_int4_ties_and_packing"]),
    ("a4_nibble_order", "(uint8_t)(nib << (4 * (k % 2)))", "(uint8_t)(nib << (4 * (1 - k % 2)))",
     ["test_act_int4_ties_and_packing"]),
    ("a4_unpack_unsigned", "(int8_t)(nib >= 8 ? nib - 16 : nib)", "(int8_t)nib",
     ["test_act_int4_ties_and_packing", "test_act_int4_bounds_spike_and_roundtrip"]),
    ("a4_dequant_127", "s4 = s4 / 7.0;", "s4 = s4 / 127.0;", ["test_act_int4_forward_worked_example"]),
]

ARGS = {
    "test_hadamard_equals_definition_on_integers": [(8, 24), (64, 128)],
    "test_absmean_groups_exact": [(3,), (64,)],
}


@pytest.fixture(scope="module")
def workdir(tmp_path_factory):
    return tmp_path_factory.mktemp("variant_mutants")


@pytest.mark.parametrize("name,orig,mut,catchers", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_variant_mutant_is_caught(name, orig, mut, catchers, workdir, monkeypatch):
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

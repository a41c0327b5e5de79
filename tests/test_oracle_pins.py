"""The oracle against what the pages and the mathematics fix (CPU only)."""
import os
import subprocess

import numpy as np
import pytest

import oracle
import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.PINS, ids=lambda p: p.__name__)
def test_pin(pin, oracle_lib):
    pin(oracle_lib)


def test_centered_mod():
    p = 2013265921
    xs = np.array([0, 1, -1, (p - 1) // 2, (p + 1) // 2, -(p - 1) // 2, p, -p, 2 ** 27, -(2 ** 27),
                   3 * p + 5, -3 * p - 5], np.int64)
    got = oracle.centered_mod(xs, p)
    for x, y in zip(xs.tolist(), got.tolist()):
        m = x % p
        ref = m - p if m > (p - 1) // 2 else m
        assert y == ref and -(p - 1) // 2 <= y <= (p - 1) // 2
        assert (y - x) % p == 0


# Planted mistakes: each mutant of the C source must fail at least one pin.
MUTANTS = {
    "dropped_last_term": ("for (int64_t j = 0; j <= t; ++j)", "for (int64_t j = 0; j < t; ++j)"),
    "dropped_first_term": ("for (int64_t j = 0; j <= t; ++j)", "for (int64_t j = (t > 0); j <= t; ++j)"),
    "wrong_sign": ("acc += p;", "acc += (j == 1) ? -p : p;"),
    "index_typo": ("g[IDX(b, t - j, d)]", "g[IDX(b, j, d)]"),
    "flipped_kernel": ("g[IDX(b, t - j, d)]", "g[IDX(b, L - 1 - (t - j), d)]"),
    "transposed_layout": ("#define IDX(b, t, d) (((int64_t)(b) * L + (t)) * D + (d))",
                          "#define IDX(b, t, d) (((int64_t)(b) * D + (d)) * L + (t))"),
    "den_signed": ("mag += fabs(p);", "mag += p;"),
    "int_narrow_accumulator": ("int64_t acc = 0;", "int16_t acc = 0;"),
    "bwd_dropped_term": ("for (int64_t t = j; t < L; ++t) {", "for (int64_t t = j + 1; t < L; ++t) {"),
    "bwd_correlation_flip": ("(double)k[IDX(b, t - j, d)]", "(double)k[IDX(b, L - 1 - (t - j), d)]"),
    "bwd_swapped_kernels": ("point_bwd_f32in(dr, g, L, D, b, j, d, &dv[i], &den_dv[i]);",
                            "point_bwd_f32in(dr, v, L, D, b, j, d, &dv[i], &den_dv[i]);"),
}


MUTANT_DIR = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_build", "mutants")  # git-ignored


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    old, new = MUTANTS[name]
    src = open(oracle._SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    os.makedirs(MUTANT_DIR, exist_ok=True)
    mut = os.path.join(MUTANT_DIR, f"mut_{name}.c")
    with open(mut, "w") as f:
        f.write(src.replace(old, new))
    so = os.path.join(MUTANT_DIR, f"libmut_{name}.so")
    oracle.build(str(mut), str(so), force=True)
    lib = oracle.load(str(so))
    failed = oracle_pins.run_all(lib)
    assert failed, f"mutant {name} passed every pin"

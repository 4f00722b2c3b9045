"""The oracle's pins catch plausible mistakes.

Each case compiles a copy of ``oracle/nl_oracle.c`` with one planted mistake
(on the CPU, in a temporary directory), swaps it in for the real library and
checks that at least one of the named pin tests now fails.
"""
import importlib
import os
import shutil
import subprocess
import tempfile

import pytest

import oracle as oracle_pkg

SRC = os.path.join(os.path.dirname(oracle_pkg.__file__), "nl_oracle.c")

MUTANTS = {
    "summation_order": ("float s = xx + yy;\n    return s + zz;",
                        "float s = yy + zz;\n    return xx + s;",
                        [("test_oracle_geometry", "test_r2_summation_order_is_pinned")]),
    "min_image_sign": ("return d - lr;", "return d + lr;",
                       [("test_oracle_geometry", "test_min_image_matches_exact_model")]),
    "cutoff_not_strict": ("if (oracle_r2(&w[3 * i], &w[3 * j], box) < rl2)",
                          "if (oracle_r2(&w[3 * i], &w[3 * j], box) <= rl2)",
                          [("test_oracle_golden", "test_oracle_reproduces_golden")]),
    "no_gray_encode": ("for (i = 1; i < 3; i++) X[i] ^= X[i - 1];", "",
                       [("test_oracle_curve", "test_hilbert_first_order_exhaustive")]),
    "interleave_transposed": ("for (d = 0; d < 3; d++)\n            key = (key << 1)",
                              "for (d = 2; d >= 0; d--)\n            key = (key << 1)",
                              [("test_oracle_curve", "test_hilbert_first_order_exhaustive")]),
    "wrap_no_second_fold": ("if (w >= L) w = w - L;", "",
                            [("test_oracle_geometry", "test_wrap_special_cases")]),
    "skin_not_strict": ("*rebuild = m > h2 ? 1 : 0;", "*rebuild = m >= h2 ? 1 : 0;",
                        [("test_oracle_skin", "test_exactly_half_skin_is_not_a_rebuild")]),
    "cell_stencil_too_small": ("for (ox = -1; ox <= 1; ox++)", "for (ox = 0; ox <= 1; ox++)",
                               [("test_oracle_geometry", "test_cell_list_equals_bruteforce_water")]),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, monkeypatch):
    old, new, checks = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    mutated = src.replace(old, new)
    d = tempfile.mkdtemp(prefix="oracle_mutant_")
    try:
        c = os.path.join(d, "m.c")
        so = os.path.join(d, "libm.so")
        open(c, "w").write(mutated)
        subprocess.check_call(["gcc", *oracle_pkg.CFLAGS, "-o", so, c, "-lm"])
        monkeypatch.setattr(oracle_pkg, "_lib", None)
        monkeypatch.setattr(oracle_pkg, "compile_library", lambda force=False: so)
        oracle_pkg.lib()
        caught = False
        for mod_name, fn_name in checks:
            mod = importlib.import_module(mod_name)
            fn = getattr(mod, fn_name)
            try:
                if fn_name == "test_oracle_reproduces_golden":
                    for p in mod.GOLDEN:
                        fn(oracle_pkg, p)
                else:
                    fn(oracle_pkg)
            except AssertionError:
                caught = True
        assert caught, f"planted mistake {name} was not caught"
    finally:
        monkeypatch.setattr(oracle_pkg, "_lib", None)
        shutil.rmtree(d, ignore_errors=True)

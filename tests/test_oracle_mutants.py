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
    "keys_quantize_unwrapped": ("q[a] = oracle_quantize(oracle_wrap(pos4[4 * i + a], box[a]), S[a]);",
                                "q[a] = oracle_quantize(pos4[4 * i + a], S[a]);",
                                [("test_oracle_curve", "test_keys_compose_wrap_quantize_per_axis",
                                  (oracle_pkg, "hilbert", (30.5, 47.25, 91.75)))]),
    "keys_scale_of_axis0": ("q[a] = oracle_quantize(oracle_wrap(pos4[4 * i + a], box[a]), S[a]);",
                            "q[a] = oracle_quantize(oracle_wrap(pos4[4 * i + a], box[a]), S[0]);",
                            [("test_oracle_curve", "test_keys_compose_wrap_quantize_per_axis",
                              (oracle_pkg, "hilbert", (30.5, 47.25, 91.75)))]),
    "keys_wrap_by_axis0": ("q[a] = oracle_quantize(oracle_wrap(pos4[4 * i + a], box[a]), S[a]);",
                           "q[a] = oracle_quantize(oracle_wrap(pos4[4 * i + a], box[0]), S[a]);",
                           [("test_oracle_curve", "test_keys_special_coordinates", (oracle_pkg, "morton"))]),
    "skin_not_strict": ("*rebuild = m > h2 ? 1 : 0;", "*rebuild = m >= h2 ? 1 : 0;",
                        [("test_oracle_skin", "test_exactly_half_skin_is_not_a_rebuild")]),
    "cell_stencil_too_small": ("for (ox = -1; ox <= 1; ox++)", "for (ox = 0; ox <= 1; ox++)",
                               [("test_oracle_geometry", "test_cell_list_equals_bruteforce_water")]),
    "edge_direction_reversed": ("float dx = oracle_min_image(wj[0] - wi[0], box[0]);",
                                "float dx = oracle_min_image(wi[0] - wj[0], box[0]);",
                                [("test_oracle_edges", "test_edges_planted_across_the_face", (0,))]),
    "edge_length_squared": ("o[3] = sqrtf(r2);", "o[3] = r2;",
                            [("test_oracle_edges", "test_edges_exact_pythagorean_length", ())]),
    "edge_reads_past_count": ("int64_t j = s < c ? nbr[i * (int64_t)K + s] : -1;",
                              "int64_t j = nbr[i * (int64_t)K + s];",
                              [("test_oracle_edges", "test_edges_ignore_entries_past_the_count",
                                ())]),
    "close_not_strict": ("if (r2 < close_d2) nc++;", "if (r2 <= close_d2) nc++;",
                         [("test_oracle_close", "test_planted_pairs_exact", ())]),
    "close_half_pairs": ("            float r2 = oracle_r2(&w[3 * i], &w[3 * j], box);\n"
                         "            if (r2 < mn) mn = r2;",
                         "            float r2 = oracle_r2(&w[3 * i], &w[3 * j], box);\n"
                         "            if (j < i) continue;\n"
                         "            if (r2 < mn) mn = r2;",
                         [("test_oracle_close", "test_planted_pairs_exact", ())]),
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
        for check in checks:
            mod = importlib.import_module(check[0])
            fn = getattr(mod, check[1])
            try:
                if len(check) > 2:        # a pin with its own arguments
                    fn(*check[2])
                elif check[1] == "test_oracle_reproduces_golden":
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


# The CSR form is numpy code in the oracle package: its mistakes are planted
# in a copy of the function's source.
CSR_MUTANTS = {
    "csr_counts_not_clipped": ("v = np.clip(np.asarray(counts, np.int64), 0, K)",
                               "v = np.asarray(counts, np.int64)"),
    "csr_offsets_shifted": ("np.cumsum(v, out=row_ptr[1:])", "np.cumsum(v, out=row_ptr[:-1])"),
}


@pytest.mark.parametrize("name", sorted(CSR_MUTANTS))
def test_planted_csr_mistake_is_caught(name, monkeypatch):
    import inspect
    import textwrap
    old, new = CSR_MUTANTS[name]
    src = textwrap.dedent(inspect.getsource(oracle_pkg.csr))
    assert src.count(old) == 1, f"mutation anchor for {name} not found"
    ns = dict(vars(oracle_pkg))
    exec(compile(src.replace(old, new), "<csr mutant>", "exec"), ns)
    monkeypatch.setattr(oracle_pkg, "csr", ns["csr"])
    mod = importlib.import_module("test_oracle_edges")
    with pytest.raises(AssertionError):
        mod.test_csr_matches_a_loop_over_rows()

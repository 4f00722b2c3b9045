"""The workload table that the benchmark and the reference arm report from
agrees with the generators: the small workloads generated here, the 10 M
ones by the recipes' closed forms (rigid water on n^3 sites with P = round(
0.15 M x L^3) sites turned into single Na+ and Cl- atoms: 3 n^3 - 4 P atoms;
the shell workload by construction)."""
import math

import numpy as np
import pytest

from neighbor_list_construction_b200 import workloads as W


@pytest.mark.parametrize("name", ["uniform4k", "lattice60k", "saltwater1m"])
def test_generated_workloads_match_the_table(name):
    w = W.make(name)
    n, cutoff, skin, K, desc = W.INFO[name]
    assert (w.n, w.cutoff, w.skin, w.capacity) == (n, cutoff, skin, K)
    assert w.pos.shape == (n, 4) and w.pos.dtype == np.float32
    assert np.all(np.asarray(w.box) > 0)
    assert f"{n:,}" in desc
    again = W.make(name)
    np.testing.assert_array_equal(again.pos, w.pos)       # seeded: the same every time


@pytest.mark.parametrize("name,nside", [("saltwater1m", 69), ("saltwater10m", 151)])
def test_salt_solution_counts_follow_the_recipe(name, nside):
    L = nside * 0.0334 ** (-1.0 / 3.0)
    P = int(round(0.15 * W.AVOGADRO_PER_A3_M * L ** 3))
    assert W.INFO[name][0] == 3 * nside ** 3 - 4 * P
    assert f"{nside}^3 sites" in W.INFO[name][4]


def test_small_salt_solution_composition():
    pos, L = W.salt_water(12, seed=3)
    P = int(round(0.15 * W.AVOGADRO_PER_A3_M * L ** 3))
    assert pos.shape[0] == 3 * 12 ** 3 - 4 * P
    assert math.isclose(L, 12 * 0.0334 ** (-1.0 / 3.0))


def test_shell_workload_total_is_fixed():
    assert W.INFO["shell10m"][0] == 10_060_000

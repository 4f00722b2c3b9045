"""Pins for the oracle's wrap, minimum image, distance predicate and
neighbor lists (CPU only).

What fixes the expected values:
* an exact-rational model of binary32 arithmetic (tests/fp32model.py) for the
  written fp32 definition, bit for bit;
* geometry in float64 (minimum over the 27 periodic images) for pairs whose
  distance is far from the cutoff;
* O(N^2) brute force for the cell-list enumeration;
* symmetry, which holds bitwise for the definition.
"""
import math

import numpy as np
import pytest

import fp32model as m32

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def f32(x):
    return float(np.float32(x))


def test_wrap_special_cases(oracle):
    L = 34.47
    Lf = f32(L)
    # -0.0 wraps to +0.0
    w = oracle.wrap(-0.0, L)
    assert w == 0.0 and math.copysign(1.0, w) == 1.0
    assert oracle.wrap(0.0, L) == 0.0
    assert oracle.wrap(Lf, L) == 0.0
    below = float(np.nextafter(np.float32(Lf), np.float32(0)))
    assert oracle.wrap(below, L) == below
    # a tiny negative coordinate rounds onto L and must come back to 0
    assert oracle.wrap(-1e-7, L) == 0.0
    # exact cases on a power-of-two box
    assert oracle.wrap(10.0, 4.0) == 2.0
    assert oracle.wrap(-1.0, 4.0) == 3.0
    assert oracle.wrap(-4.0, 4.0) == 0.0
    assert oracle.wrap(4.0 * 7 + 0.25, 4.0) == 0.25
    # far from the box the product L*t rounds so that x - L*t lands at or
    # above L; one more fold brings it back (here 34.5 - 34.47)
    w = oracle.wrap(2109564.0, L)
    assert w == m32.sub(34.5, L) and 0.0 < w < 0.05


def test_wrap_matches_exact_model_and_range(oracle):
    rng = np.random.default_rng(11)
    for L in (34.47, 84.023, 468.88, 4.0, 7.25):
        Lf = f32(L)
        xs = np.concatenate([rng.uniform(-3 * L, 4 * L, 300),
                             np.array([Lf, -Lf, 2 * Lf, -0.0, 1e-30, -1e-30])]).astype(np.float32)
        for x in xs:
            w = oracle.wrap(float(x), L)
            assert 0.0 <= w < Lf
            assert w == m32.wrap(float(x), L)
            # w is congruent to x modulo L up to fp32 rounding of the product
            k = round((float(x) - w) / Lf)
            assert abs((float(x) - w) - k * Lf) <= 4 * max(abs(float(x)), Lf) * 2 ** -23


def test_min_image_matches_exact_model(oracle):
    rng = np.random.default_rng(12)
    for L in (34.47, 84.023, 5.0, 468.88):
        ds = rng.uniform(-L, L, 400).astype(np.float32)
        half = np.float32(L) / np.float32(2)
        extra = np.array([half, -half, np.nextafter(half, np.float32(0)),
                          np.nextafter(half, np.float32(L)), 0.0, np.float32(L) * np.float32(0.999)],
                         np.float32)
        for d in np.concatenate([ds, extra]):
            assert oracle.min_image(float(d), L) == m32.min_image(float(d), L)


def test_min_image_ties_to_even(oracle):
    # d/L == 0.5 exactly: rintf(0.5) == 0, so d is left unchanged; -0.5 too.
    assert oracle.min_image(2.0, 4.0) == 2.0
    assert oracle.min_image(-2.0, 4.0) == -2.0
    # d/L == 1.5 -> rintf = 2
    assert oracle.min_image(6.0, 4.0) == -2.0


def test_r2_matches_exact_model(oracle):
    rng = np.random.default_rng(13)
    box = np.array([34.47, 41.5, 29.0], np.float32)
    for _ in range(400):
        a = (rng.random(3) * box).astype(np.float32)
        b = (rng.random(3) * box).astype(np.float32)
        assert oracle.r2(a, b, box) == m32.r2(a, b, box)


def test_r2_summation_order_is_pinned(oracle):
    """Find operands where ((x+y)+z) and (x+(y+z)) round differently and
    check the oracle gives the left-nested value defined for the path."""
    rng = np.random.default_rng(14)
    box = np.array([64.0, 64.0, 64.0], np.float32)
    found = 0
    for _ in range(20000):
        a = np.zeros(3, np.float32)
        b = rng.uniform(-3, 3, 3).astype(np.float32)
        d = [float(x) for x in b]
        left = m32.add(m32.add(m32.mul(d[0], d[0]), m32.mul(d[1], d[1])), m32.mul(d[2], d[2]))
        right = m32.add(m32.mul(d[0], d[0]), m32.add(m32.mul(d[1], d[1]), m32.mul(d[2], d[2])))
        if left != right:
            assert oracle.r2(a, b, box) == left
            found += 1
            if found >= 20:
                break
    assert found >= 20


def _exact_periodic_d2(a, b, box):
    best = math.inf
    for kx in (-1, 0, 1):
        for ky in (-1, 0, 1):
            for kz in (-1, 0, 1):
                d = [float(b[i]) - float(a[i]) + k * float(box[i]) for i, k in enumerate((kx, ky, kz))]
                best = min(best, d[0] ** 2 + d[1] ** 2 + d[2] ** 2)
    return best


def test_r2_agrees_with_periodic_geometry(oracle):
    """Away from rounding, the fp32 value is the true minimum-image distance."""
    rng = np.random.default_rng(15)
    box = np.array([30.0, 33.5, 47.25], np.float32)
    for _ in range(2000):
        a = (rng.random(3) * box).astype(np.float32)
        b = (rng.random(3) * box).astype(np.float32)
        exact = _exact_periodic_d2(a, b, box)
        got = oracle.r2(a, b, box)
        assert abs(got - exact) <= 1e-5 * max(exact, 1.0)


def test_r2_symmetric_bitwise(oracle):
    rng = np.random.default_rng(16)
    box = np.array([34.47, 34.47, 34.47], np.float32)
    for _ in range(2000):
        a = (rng.random(3) * box).astype(np.float32)
        b = (rng.random(3) * box).astype(np.float32)
        assert oracle.r2(a, b, box) == oracle.r2(b, a, box)


def _rows_as_sets(nbr, cnt):
    return [set(int(v) for v in nbr[i, :min(cnt[i], nbr.shape[1])]) for i in range(nbr.shape[0])]


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_cell_list_equals_bruteforce_uniform(oracle, seed):
    from neighbor_list_construction_b200 import workloads
    w = workloads.make("uniform4k", seed=seed)
    a_nbr, a_cnt, a_ov = oracle.build(w.pos, w.box, w.cutoff, w.skin, w.capacity)
    b_nbr, b_cnt, b_ov = oracle.bruteforce(w.pos, w.box, w.cutoff, w.skin, w.capacity)
    assert not a_ov and not b_ov
    np.testing.assert_array_equal(a_cnt, b_cnt)
    np.testing.assert_array_equal(a_nbr, b_nbr)
    # statistical sanity: mean directed neighbors ~ rho * 4/3 pi rl^3 = 128.8
    assert abs(a_cnt.mean() - 128.8) < 4.0


def test_cell_list_equals_bruteforce_water(oracle):
    from neighbor_list_construction_b200 import workloads
    w = workloads.make("saltwater_n12")
    a = oracle.build(w.pos, w.box, w.cutoff, w.skin, w.capacity)
    b = oracle.bruteforce(w.pos, w.box, w.cutoff, w.skin, w.capacity)
    np.testing.assert_array_equal(a[1], b[1])
    np.testing.assert_array_equal(a[0], b[0])


def test_adversarial_small_box(oracle):
    """Atoms on the faces, at -0.0, L, beyond L, exactly at rl, across the
    periodic corner; a box exactly 3 rl wide and an orthorhombic one."""
    rl = 2.5  # cutoff 2.0 + skin 0.5, exact
    for box in ([7.5, 7.5, 7.5], [7.5, 9.0, 11.25], [8.0, 8.0, 8.0]):
        box = np.array(box, np.float32)
        L = box
        pts = [
            [0, 0, 0], [-0.0, 0, 0], [L[0], 0, 0], [L[0] + 2.0, 0, 0], [rl, 0, 0],
            [0, rl, 0], [L[0] - 1.0, L[1] - 1.0, L[2] - 1.0], [L[0] - 0.25, 0.5, L[2] - 0.25],
            [L[0] / 2, L[1] / 2, L[2] / 2], [float(np.nextafter(np.float32(L[0]), np.float32(0))), 0, 0],
            [-2.4999, 0, 0], [1.25, 1.25, 1.25], [-1e-8, -1e-8, -1e-8],
        ]
        rng = np.random.default_rng(17)
        pts += list(rng.uniform(-1, 1, (40, 3)) * box + box / 2)
        pos = np.array(pts, np.float32)
        a = oracle.build(pos, box, 2.0, 0.5, 64)
        b = oracle.bruteforce(pos, box, 2.0, 0.5, 64)
        np.testing.assert_array_equal(a[1], b[1])
        np.testing.assert_array_equal(a[0], b[0])
        # every listed pair is within rl under the exact model; symmetric lists
        sets = _rows_as_sets(a[0], a[1])
        for i, s in enumerate(sets):
            for j in s:
                assert i in sets[j]
                wi = [m32.wrap(pos[i, k], box[k]) for k in range(3)]
                wj = [m32.wrap(pos[j, k], box[k]) for k in range(3)]
                assert m32.r2(wi, wj, box) < m32.mul(rl, rl)
        # a pair at exactly rl along an axis is excluded: atoms 0 and 4
        assert 4 not in sets[0]


def test_overflow_counts_true_and_rows_truncated(oracle):
    rng = np.random.default_rng(18)
    box = np.array([20.0, 20.0, 20.0], np.float32)
    pos = (rng.random((300, 3)) * 3.0 + 5.0).astype(np.float32)  # dense clump
    nbr, cnt, ov = oracle.build(pos, box, 2.0, 0.5, 16)
    assert ov
    full, fcnt, fov = oracle.build(pos, box, 2.0, 0.5, 400)
    assert not fov
    np.testing.assert_array_equal(cnt, fcnt)
    np.testing.assert_array_equal(nbr, full[:, :16])


def test_rows_subset_matches_full(oracle):
    from neighbor_list_construction_b200 import workloads
    w = workloads.make("lattice60k")
    which = np.array([0, 1, 77, 4242, w.n - 1])
    nbr, cnt, _ = oracle.rows(w.pos, w.box, w.cutoff, w.skin, w.capacity, which)
    full, fcnt, _ = oracle.build(w.pos, w.box, w.cutoff, w.skin, w.capacity)
    np.testing.assert_array_equal(cnt, fcnt[which])
    np.testing.assert_array_equal(nbr, full[which])
    assert 60 < fcnt.mean() < 200


def test_threaded_oracle_equals_single_threaded(oracle):
    """The OpenMP loops (keys, wrap, rows) give the same result on 1 and on
    many threads: rows are independent and each is sorted before it is
    written."""
    from neighbor_list_construction_b200 import workloads
    w = workloads.make("saltwater_n20")
    old = oracle.set_threads(1)
    try:
        one = oracle.build(w.pos, w.box, w.cutoff, w.skin, w.capacity)
        k1 = oracle.sort(w.pos, w.box)
        oracle.set_threads(max(4, old))
        many = oracle.build(w.pos, w.box, w.cutoff, w.skin, w.capacity)
        km = oracle.sort(w.pos, w.box)
    finally:
        oracle.set_threads(old)
    np.testing.assert_array_equal(one[0], many[0])
    np.testing.assert_array_equal(one[1], many[1])
    assert one[2] == many[2]
    np.testing.assert_array_equal(k1[0], km[0])
    np.testing.assert_array_equal(k1[1], km[1])

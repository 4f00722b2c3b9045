"""Pins for the oracle's space-filling-curve keys and curve order (CPU only).

What fixes the expected values: the defining properties of a Hilbert curve
(a bijection onto the grid whose consecutive cells are face-adjacent, which
refines itself level by level), the closed form of Morton interleaving,
the quantization's own bounds, and numpy's lexicographic sort as a textbook
routine for the (key, index) order.
"""
import numpy as np
import pytest


def test_hilbert_first_order_exhaustive(oracle):
    """Orders b = 1..5: keys 0..8^b-1 visit every cell once and consecutive
    cells differ by one step along one axis."""
    for b in range(1, 6):
        n = 8 ** b
        cells = np.array([oracle.hilbert_axes(k, b) for k in range(n)], np.int64)
        assert cells.min() == 0 and cells.max() == 2 ** b - 1
        flat = (cells[:, 2] << (2 * b)) | (cells[:, 1] << b) | cells[:, 0]
        assert np.unique(flat).size == n, "not a bijection"
        steps = np.abs(np.diff(cells, axis=0)).sum(axis=1)
        assert np.all(steps == 1), f"non-adjacent consecutive cells at order {b}"
        fwd = np.array([oracle.hilbert_key(*map(int, c), b) for c in cells], np.uint64)
        np.testing.assert_array_equal(fwd, np.arange(n, dtype=np.uint64))
        # the curve starts at the origin and ends at a corner one edge away
        assert tuple(cells[0]) == (0, 0, 0)
        end = cells[-1]
        assert sorted(end.tolist()) == [0, 0, 2 ** b - 1]


def test_hilbert_order6_bijection(oracle):
    b = 6
    n = 8 ** b
    rng = np.random.default_rng(3)
    ks = rng.choice(n - 1, size=4000, replace=False)
    for k in ks:
        c0 = np.array(oracle.hilbert_axes(int(k), b))
        c1 = np.array(oracle.hilbert_axes(int(k) + 1, b))
        assert np.abs(c1 - c0).sum() == 1
        assert oracle.hilbert_key(*map(int, c0), b) == k


def test_hilbert_nesting(oracle):
    """key_21(q) >> 3(21-b) == key_b(q >> (21-b)): coarser curves are prefixes."""
    rng = np.random.default_rng(4)
    for _ in range(3000):
        q = rng.integers(0, 2 ** 21, 3)
        b = int(rng.integers(1, 21))
        k21 = oracle.hilbert_key(int(q[0]), int(q[1]), int(q[2]), 21)
        kb = oracle.hilbert_key(int(q[0]) >> (21 - b), int(q[1]) >> (21 - b),
                                int(q[2]) >> (21 - b), b)
        assert k21 >> (3 * (21 - b)) == kb


def test_hilbert_order21_adjacency_and_roundtrip(oracle):
    rng = np.random.default_rng(5)
    top = 8 ** 21
    for _ in range(20000):
        k = int(rng.integers(0, top - 1, dtype=np.uint64))
        c0 = np.array(oracle.hilbert_axes(k, 21), np.int64)
        c1 = np.array(oracle.hilbert_axes(k + 1, 21), np.int64)
        assert np.abs(c1 - c0).sum() == 1
        assert oracle.hilbert_key(*map(int, c0), 21) == k
    # keys use 63 bits: bit 63 is always clear
    assert oracle.hilbert_key(2 ** 21 - 1, 2 ** 21 - 1, 2 ** 21 - 1, 21) < 2 ** 63


def test_morton_closed_form(oracle):
    for l in range(21):
        assert oracle.morton_key(1 << l, 0, 0) == 1 << (3 * l + 2)
        assert oracle.morton_key(0, 1 << l, 0) == 1 << (3 * l + 1)
        assert oracle.morton_key(0, 0, 1 << l) == 1 << (3 * l)
    rng = np.random.default_rng(6)
    for _ in range(200):
        q = [int(v) for v in rng.integers(0, 2 ** 21, 3)]
        k = oracle.morton_key(*q)
        assert k == (oracle.morton_key(q[0], 0, 0) | oracle.morton_key(0, q[1], 0)
                     | oracle.morton_key(0, 0, q[2]))


def test_quantize_bounds(oracle):
    for L in (34.47, 468.88, 84.023):
        S = oracle.quant_scale(L)
        assert S == float(np.float32(2097152.0) / np.float32(L))
        assert oracle.quantize(0.0, S) == 0
        below = float(np.nextafter(np.float32(L), np.float32(0)))
        assert oracle.quantize(below, S) == 2 ** 21 - 1
        rng = np.random.default_rng(7)
        ws = np.sort(rng.random(5000).astype(np.float32) * np.float32(L))
        qs = np.array([oracle.quantize(float(w), S) for w in ws])
        assert np.all(np.diff(qs) >= 0)
        # within one cell of the real-valued grid coordinate
        exact = np.floor(ws.astype(np.float64) * 2 ** 21 / float(np.float32(L)))
        assert np.all(np.abs(qs - exact) <= 1)


@pytest.mark.parametrize("curve", ["hilbert", "morton"])
def test_sort_matches_lexsort(oracle, curve):
    from neighbor_list_construction_b200 import workloads
    w = workloads.make("lattice60k")
    keys = oracle.keys(w.pos, w.box, curve)
    perm, ks = oracle.sort(w.pos, w.box, curve)
    ref = np.lexsort((np.arange(w.n), keys))
    np.testing.assert_array_equal(perm, ref.astype(np.int32))
    np.testing.assert_array_equal(ks, keys[ref])
    assert np.all(np.diff(ks.astype(np.float64)) >= 0)


def test_sort_ties_by_index(oracle):
    # identical positions -> identical keys -> order by original index
    pos = np.zeros((64, 4), np.float32)
    pos[::2, :3] = 5.0
    perm, ks = oracle.sort(pos, [10.0, 10.0, 10.0])
    zeros = perm[ks == ks.min()]
    assert np.all(np.diff(zeros) > 0)
    assert sorted(perm.tolist()) == list(range(64))


def test_hilbert_order_is_local(oracle):
    """Consecutive atoms along the curve are close (sanity, not a pin)."""
    from neighbor_list_construction_b200 import workloads
    w = workloads.make("uniform4k")
    perm, _ = oracle.sort(w.pos, w.box)
    p = w.pos[perm, :3].astype(np.float64)
    d_curve = np.linalg.norm(np.diff(p, axis=0), axis=1).mean()
    d_rand = np.linalg.norm(np.diff(w.pos[:, :3].astype(np.float64), axis=0), axis=1).mean()
    assert d_curve < 0.25 * d_rand

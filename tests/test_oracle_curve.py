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


# ---------------------------------------------------------------------------
# The key of an atom is the curve index of its grid cell, and the grid cell is
# fixed by the mathematics alone: per axis a, q_a = floor(frac(x_a / L_a) * 2^21)
# for the real-valued coordinate.  The oracle computes it in fp32 (wrap, then
# scale by fl(2^21 / L_a)), which agrees with the exact value except within a
# few fp32 roundings of a cell face.  The pins below take the exact value from
# rational arithmetic, skip only points that close to a face, and check the
# whole composition (wrap of each axis by its own side, quantization with that
# axis's own scale, the key of the three grid coordinates) on orthorhombic
# boxes with coordinates far outside [0, L).
# ---------------------------------------------------------------------------
from fractions import Fraction

_BOXES = [(30.5, 47.25, 91.75), (91.75, 30.5, 47.25), (47.25, 91.75, 30.5),
          (468.88, 214.256, 84.023)]


def _exact_cell(x: float, L: float):
    """(q, distance to the nearest cell face in units of a cell) from exact
    rationals: q = floor(frac(x / L) * 2^21)."""
    fx, fl_ = Fraction(float(np.float32(x))), Fraction(float(np.float32(L)))
    u = (fx / fl_) % 1 * 2 ** 21          # exact grid coordinate in [0, 2^21)
    q = int(u)                            # floor (u >= 0)
    frac = u - q
    return q, float(min(frac, 1 - frac))


def _coords(rng, L, n):
    """Coordinates inside the box and up to five box lengths either side."""
    span = rng.integers(-5, 6, size=n).astype(np.float64)
    return (rng.random(n) * L + span * L).astype(np.float32)


def _cells_of_keys(oracle, keys, curve):
    """Grid cells of keys: the oracle's inverse Hilbert transform (pinned by
    the curve tests above) or Morton de-interleaving (closed form)."""
    out = []
    for k in keys:
        k = int(k)
        if curve == "hilbert":
            out.append(oracle.hilbert_axes(k, 21))
        else:
            q = [0, 0, 0]
            for l in range(21):
                q[0] |= ((k >> (3 * l + 2)) & 1) << l
                q[1] |= ((k >> (3 * l + 1)) & 1) << l
                q[2] |= ((k >> (3 * l)) & 1) << l
            out.append(tuple(q))
    return np.array(out, np.int64)


@pytest.mark.parametrize("curve", ["hilbert", "morton"])
@pytest.mark.parametrize("box", _BOXES)
def test_keys_compose_wrap_quantize_per_axis(oracle, curve, box):
    """Per axis, the key's grid coordinate is floor(frac(x/L_a) * 2^21) of
    that axis's own side.  Error bound of the fp32 steps, in cells: the wrap
    L*floor(x/L) rounds by at most 2^-24 |x| + 2^-24 L (|x| <= 6 L here, so
    <= 7/8 cell), the scale fl(2^21/L) and the product by at most 1/4 cell:
    at most 2 cells apart anywhere (cyclically: a point just below a
    multiple of L may wrap to cell 0), and equal for in-box points more than
    0.4 cell from a face, where the wrap is exact."""
    rng = np.random.default_rng(11)
    n = 3000
    pos = np.zeros((n, 4), np.float32)
    for a in range(3):
        pos[:, a] = _coords(rng, box[a], n)
    pos[:300, :3] = (rng.random((300, 3)) * np.asarray(box)).astype(np.float32)  # in-box
    got = _cells_of_keys(oracle, oracle.keys(pos, box, curve), curve)
    exact_in = 0
    for i in range(n):
        for a in range(3):
            q, margin = _exact_cell(float(pos[i, a]), box[a])
            d = abs(int(got[i, a]) - q)
            d = min(d, 2 ** 21 - d)
            assert d <= 2, (i, a, float(pos[i, a]), q, int(got[i, a]))
            L = np.float32(box[a])
            if np.float32(0) <= pos[i, a] < L and margin > 0.4:
                assert int(got[i, a]) == q, (i, a, float(pos[i, a]))
                exact_in += 1
    assert exact_in > 100


def _interior(L):
    """The first float at or above 0.3 L whose exact grid coordinate is more
    than 0.4 cell from a face."""
    x = np.float32(L) * np.float32(0.3)
    while _exact_cell(float(x), L)[1] <= 0.4:
        x = np.nextafter(x, np.float32(np.inf))
    return x


@pytest.mark.parametrize("curve", ["hilbert", "morton"])
def test_keys_special_coordinates(oracle, curve):
    """-0, 0, L, multiples of L and the last float below L, on each axis of an
    orthorhombic box, with the other axes held at an interior cell."""
    box = (30.5, 47.25, 91.75)
    keyfn = oracle.hilbert_key if curve == "hilbert" else oracle.morton_key
    top = 2 ** 21 - 1
    for a in range(3):
        L = np.float32(box[a])
        cases = {0.0: 0, -0.0: 0, float(L): 0, float(2 * L): 0, float(-L): 0,
                 float(-3 * L): 0, float(np.nextafter(L, np.float32(0))): top}
        for x, qa in cases.items():
            pos = np.zeros((1, 4), np.float32)
            base = []
            for b in range(3):
                # an interior coordinate far from any cell face
                pos[0, b] = _interior(box[b])
                base.append(_exact_cell(float(pos[0, b]), box[b])[0])
            pos[0, a] = np.float32(x)
            base[a] = qa
            k = int(oracle.keys(pos, box, curve)[0])
            assert k == keyfn(*base), (a, x)


def test_sort_is_keys_then_index_on_orthorhombic_box(oracle):
    """oracle.sort orders by the composed keys of an orthorhombic box with
    out-of-box coordinates, ties by index (numpy lexsort as the textbook
    routine)."""
    box = (30.5, 47.25, 91.75)
    rng = np.random.default_rng(12)
    n = 5000
    pos = np.zeros((n, 4), np.float32)
    for a in range(3):
        pos[:, a] = _coords(rng, box[a], n)
    pos[n // 2:n // 2 + 50, :3] = pos[7, :3]       # a run of equal keys
    for curve in ("hilbert", "morton"):
        keyfn = oracle.hilbert_key if curve == "hilbert" else oracle.morton_key
        perm, ks = oracle.sort(pos, box, curve)
        # the sorted keys are the keys pinned above, taken along perm
        np.testing.assert_array_equal(ks, oracle.keys(pos, box, curve)[perm])
        assert sorted(perm.tolist()) == list(range(n))
        kk = ks.astype(object)
        for k in range(n - 1):
            assert kk[k] < kk[k + 1] or (kk[k] == kk[k + 1] and perm[k] < perm[k + 1])

"""Pins of the oracle's per-slot edge features (minimum-image displacement from
the row atom to its neighbor, and its length) against facts that do not go
through it: the same geometry in float64, exact antisymmetry of the pair,
planted pairs across a periodic face at exactly representable distances, and
the padding rule."""
import numpy as np
import pytest

import oracle


def rows(pos, box, cutoff, skin):
    """Oracle rows with the capacity of the largest row (complete sets)."""
    _, cnt, _ = oracle.build(pos, box, cutoff, skin, 1)
    K = max(int(cnt.max()), 1)
    nbr, cnt, ov = oracle.build(pos, box, cutoff, skin, K)
    assert not ov
    return nbr, cnt


@pytest.mark.parametrize("seed,box", [(1, [9.0, 9.0, 9.0]), (2, [7.6, 10.1, 13.0])])
def test_edges_match_float64_geometry(seed, box):
    rng = np.random.default_rng(seed)
    box = np.array(box, np.float32)
    n = 300
    pos = np.zeros((n, 4), np.float32)
    pos[:, :3] = (rng.random((n, 3)) * 1.6 - 0.3) * box   # some outside the box
    nbr, cnt = rows(pos, box, 2.0, 0.5)
    e = oracle.edge_features(pos, box, nbr, cnt)
    L = box.astype(np.float64)
    checked = 0
    for i in range(n):
        for s in range(cnt[i]):
            j = nbr[i, s]
            d = pos[j, :3].astype(np.float64) - pos[i, :3].astype(np.float64)
            d -= L * np.round(d / L)
            # wrap and subtraction round at most a few ulps of the box side
            assert np.all(np.abs(e[i, s, :3] - d) <= 4 * np.spacing(box)), (i, j)
            assert abs(float(e[i, s, 3]) - np.sqrt(d @ d)) <= 1e-5
            checked += 1
    assert checked == int(cnt.sum()) > 1000


def test_edges_length_is_the_membership_distance():
    rng = np.random.default_rng(5)
    box = np.array([12.0, 11.0, 10.0], np.float32)
    n = 250
    pos = np.zeros((n, 4), np.float32)
    pos[:, :3] = rng.random((n, 3)) * box
    cutoff, skin = 2.5, 0.5
    nbr, cnt = rows(pos, box, cutoff, skin)
    e = oracle.edge_features(pos, box, nbr, cnt)
    rl = np.float32(np.float32(cutoff) + np.float32(skin))
    for i in range(n):
        for s in range(cnt[i]):
            r2 = oracle.r2(pos[i, :3], pos[nbr[i, s], :3], box)
            # float32 square root is correctly rounded in numpy as in C
            assert e[i, s, 3] == np.sqrt(np.float32(r2))
            assert e[i, s, 3] <= rl


def test_edges_antisymmetric():
    rng = np.random.default_rng(9)
    box = np.array([10.0, 9.5, 11.0], np.float32)
    n = 200
    pos = np.zeros((n, 4), np.float32)
    pos[:, :3] = rng.random((n, 3)) * box
    nbr, cnt = rows(pos, box, 2.0, 0.75)
    e = oracle.edge_features(pos, box, nbr, cnt)
    slot = {}
    for i in range(n):
        for s in range(cnt[i]):
            slot[(i, int(nbr[i, s]))] = s
    for (i, j), s in slot.items():
        t = slot[(j, i)]
        np.testing.assert_array_equal(e[i, s, :3], -e[j, t, :3])
        assert e[i, s, 3] == e[j, t, 3]


@pytest.mark.parametrize("axis", [0, 1, 2])
def test_edges_planted_across_the_face(axis):
    box = np.array([10.0, 10.0, 10.0], np.float32)
    pos = np.zeros((3, 4), np.float32)
    pos[:, :3] = 5.0
    pos[0, axis] = 0.25
    pos[1, axis] = 9.75          # 0.5 away from atom 0 through the face
    pos[2, :3] = [2.5, 2.5, 2.5]
    pos[2, axis] = 0.625         # 0.375 from atom 0 on `axis`, 2.5 on the others
    nbr = np.array([[1, 2], [0, -1], [-1, -1]], np.int32)
    cnt = np.array([2, 1, 0], np.int32)
    e = oracle.edge_features(pos, box, nbr, cnt)
    want01 = np.zeros(4, np.float32)
    want01[axis] = -0.5
    want01[3] = 0.5
    np.testing.assert_array_equal(e[0, 0], want01)
    want10 = -want01
    want10[3] = 0.5
    np.testing.assert_array_equal(e[1, 0], want10)
    d = np.full(3, -2.5, np.float32)
    d[axis] = 0.375
    np.testing.assert_array_equal(e[0, 1, :3], d)
    # 0.375^2 + 2 * 2.5^2 = 12.640625 exactly; its root is not a dyadic, so
    # compare with the correctly rounded float32 root
    assert e[0, 1, 3] == np.sqrt(np.float32(12.640625))
    np.testing.assert_array_equal(e[1, 1], 0.0)
    np.testing.assert_array_equal(e[2], 0.0)


def test_edges_exact_pythagorean_length():
    box = np.array([16.0, 16.0, 16.0], np.float32)
    pos = np.zeros((2, 4), np.float32)
    pos[0, :3] = [1.0, 1.0, 1.0]
    pos[1, :3] = [1.375, 1.5, 1.0]     # (0.375, 0.5, 0): length 0.625 exactly
    e = oracle.edge_features(pos, box, np.array([[1], [0]], np.int32),
                             np.array([1, 1], np.int32))
    np.testing.assert_array_equal(e[0, 0], [0.375, 0.5, 0.0, 0.625])
    np.testing.assert_array_equal(e[1, 0], [-0.375, -0.5, 0.0, 0.625])


def test_edges_padding_overflow_and_bad_indices():
    rng = np.random.default_rng(3)
    box = np.array([8.0, 8.0, 8.0], np.float32)
    n = 120
    pos = np.zeros((n, 4), np.float32)
    pos[:, :3] = rng.random((n, 3)) * box
    K = 4
    nbr, cnt, ov = oracle.build(pos, box, 2.0, 0.5, K)
    assert ov                                   # some rows hold K of more
    full, fcnt = rows(pos, box, 2.0, 0.5)
    e = oracle.edge_features(pos, box, nbr, cnt)
    ef = oracle.edge_features(pos, box, full, fcnt)
    for i in range(n):
        c = min(int(cnt[i]), K)
        np.testing.assert_array_equal(e[i, c:], 0.0)
        for s in range(c):
            t = int(np.nonzero(full[i] == nbr[i, s])[0][0])
            np.testing.assert_array_equal(e[i, s], ef[i, t])
    bad = nbr.copy()
    bad[0, 0] = -1
    bad[1, 0] = n
    e2 = oracle.edge_features(pos, box, bad, np.maximum(cnt, 1))
    np.testing.assert_array_equal(e2[0, 0], 0.0)
    np.testing.assert_array_equal(e2[1, 0], 0.0)


def test_csr_matches_a_loop_over_rows():
    """The oracle's CSR form against a plain loop: offsets are the running
    sum of the valid entries, entries are the rows' valid prefixes."""
    rng = np.random.default_rng(12)
    for n, K in [(0, 4), (1, 1), (37, 5), (300, 16)]:
        nbr = rng.integers(-1, 1000, (n, K)).astype(np.int32)
        cnt = rng.integers(-2, K + 4, n).astype(np.int32)
        row_ptr, col = oracle.csr(nbr, cnt)
        want_ptr, want_col = [0], []
        for i in range(n):
            v = min(max(int(cnt[i]), 0), K)
            want_col.extend(int(x) for x in nbr[i, :v])
            want_ptr.append(want_ptr[-1] + v)
        assert row_ptr.dtype == np.int64 and col.dtype == np.int32
        np.testing.assert_array_equal(row_ptr, want_ptr)
        np.testing.assert_array_equal(col, np.array(want_col, np.int32))


def test_csr_of_built_rows_round_trips():
    """Rows rebuilt from the CSR form of an oracle build, padded with -1,
    are the build's rows."""
    rng = np.random.default_rng(13)
    box = np.array([9.0, 9.0, 9.0], np.float32)
    pos = np.zeros((200, 4), np.float32)
    pos[:, :3] = rng.random((200, 3)) * box
    for K in (8, 64):
        nbr, cnt, _ = oracle.build(pos, box, 2.0, 0.5, K)
        row_ptr, col = oracle.csr(nbr, cnt)
        back = np.full_like(nbr, -1)
        for i in range(nbr.shape[0]):
            seg = col[row_ptr[i]:row_ptr[i + 1]]
            back[i, :seg.size] = seg
        np.testing.assert_array_equal(back, nbr)


def test_edges_ignore_entries_past_the_count():
    """Slots at or past min(counts[i], K) are padding whatever they hold: stale
    valid indices there give zeros, as -1 does."""
    rng = np.random.default_rng(21)
    box = np.array([9.0, 9.0, 9.0], np.float32)
    n = 150
    pos = np.zeros((n, 4), np.float32)
    pos[:, :3] = rng.random((n, 3)) * box
    nbr, cnt = rows(pos, box, 2.0, 0.5)
    K = nbr.shape[1]
    stale = nbr.copy()
    pad = np.arange(K)[None, :] >= cnt[:, None]
    stale[pad] = rng.integers(0, n, int(pad.sum()))
    e = oracle.edge_features(pos, box, nbr, cnt)
    e_stale = oracle.edge_features(pos, box, stale, cnt)
    assert pad.sum() > 100
    np.testing.assert_array_equal(e_stale, e)
    np.testing.assert_array_equal(e_stale[pad], 0.0)

"""Pins of the oracle's close-pair detector (minimum squared pair distance and
the count of directed pairs below a threshold) against definitions that do not
go through it: brute force over all pairs and planted pairs at exactly
representable distances."""
import numpy as np
import pytest

import oracle


def brute(pos, box, cutoff, skin, close_d2):
    rl = np.float32(np.float32(cutoff) + np.float32(skin))
    rl2 = np.float32(rl * rl)
    n = pos.shape[0]
    mn, nc = np.inf, 0
    for i in range(n):
        for j in range(n):
            if i == j:
                continue
            r2 = oracle.r2(pos[i, :3], pos[j, :3], box)
            if r2 < rl2:
                mn = min(mn, r2)
                nc += r2 < np.float32(close_d2)
    return mn, nc


@pytest.mark.parametrize("seed,box", [(1, [9.0, 9.0, 9.0]), (2, [7.6, 10.1, 13.0]),
                                      (3, [20.0, 20.0, 20.0])])
def test_close_pairs_match_brute_force(seed, box):
    rng = np.random.default_rng(seed)
    box = np.array(box, np.float32)
    n = 160
    pos = np.zeros((n, 4), np.float32)
    pos[:, :3] = rng.random((n, 3)) * box
    for close in (0.25, 1.0, 4.0):
        mn, nc = oracle.close_pairs(pos, box, 2.0, 0.5, close)
        bmn, bnc = brute(pos, box, 2.0, 0.5, close)
        assert mn == np.float32(bmn) and nc == bnc


def test_planted_pairs_exact():
    """Atoms far apart except two planted pairs at separations 0.5 and 0.75
    (r2 = 0.25 and 0.5625 exactly); one pair straddles the periodic face."""
    box = np.array([30.0, 30.0, 30.0], np.float32)
    pos = np.array([[5.0, 5.0, 5.0, 0], [5.5, 5.0, 5.0, 0],
                    [29.625, 15.0, 15.0, 0], [0.375, 15.0, 15.0, 0],
                    [15.0, 5.0, 25.0, 0]], np.float32)
    mn, nc = oracle.close_pairs(pos, box, 2.0, 0.5, 0.3)
    assert mn == 0.25 and nc == 2
    mn, nc = oracle.close_pairs(pos, box, 2.0, 0.5, 1.0)
    assert mn == 0.25 and nc == 4
    mn, nc = oracle.close_pairs(pos, box, 2.0, 0.5, 0.25)   # strict
    assert nc == 0


def test_no_pairs():
    box = np.array([30.0, 30.0, 30.0], np.float32)
    pos = np.array([[1.0, 1.0, 1.0, 0], [15.0, 15.0, 15.0, 0]], np.float32)
    mn, nc = oracle.close_pairs(pos, box, 2.0, 0.5, 1.0)
    assert mn == np.inf and nc == 0
    mn, nc = oracle.close_pairs(np.zeros((0, 4), np.float32), box, 2.0, 0.5, 1.0)
    assert mn == np.inf and nc == 0

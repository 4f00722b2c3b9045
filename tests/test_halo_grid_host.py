"""The coarse grid of the halo selection (nl_halo_grid: host code of the
library, callable without a GPU).  Two atoms closer than rl, by the fp32
minimum-image r2 of the build, must land in the same or adjacent coarse
cells (periodically) under the fp32 cell assignment of the halo kernels:
T = fl(dims / L) and c = min(floor(fl(w * T)), dims - 1) of the wrapped
coordinate w.  Pairs include partners just under rl across a cell face, in a
box whose cells are barely wider than rl plus the grid's margin."""
import math

import numpy as np
import pytest

import oracle
from neighbor_list_construction_b200 import nl


def coarse(w, L, dims):
    T = np.float32(np.float32(dims) / np.float32(L))
    c = int(np.floor(np.float32(np.float32(w) * T)))
    return min(max(c, 0), dims - 1)


def adjacent(a, b, dims):
    d = (a - b) % dims
    return d in (0, 1, dims - 1)


def tight_box(rl):
    """A box side whose grid has 3 cells, each wider than rl by little more
    than the margin."""
    w = rl * (1.0 + 2.0 ** -10)
    L = 3.0 * w / (1.0 - 3.0 * 2.0 ** -16) * (1.0 + 1e-6)
    return float(np.float32(L))


def check_pairs(box, cutoff, skin, seed, n=3000):
    dims = nl.nl_halo_grid(box, cutoff, skin)
    rl = np.float32(np.float32(cutoff) + np.float32(skin))
    rl2 = np.float32(rl * rl)
    rng = np.random.default_rng(seed)
    box32 = np.array(box, np.float32)
    checked = 0
    for k in range(n):
        a = (rng.random(3) * box32).astype(np.float32)
        if k % 2:   # start on a coarse face: the first fp32 value of cell m on one axis
            ax = k % 3
            m = int(rng.integers(0, dims[ax]))
            a[ax] = np.float32(m * float(box32[ax]) / dims[ax])
        u = rng.normal(size=3)
        u /= np.linalg.norm(u)
        r = float(rl) * (1.0 - rng.random() * (1e-6 if k % 4 < 2 else 0.5))
        b = np.array([oracle.wrap(np.float32(a[i] + r * u[i]), box32[i]) for i in range(3)],
                     np.float32)
        aw = np.array([oracle.wrap(a[i], box32[i]) for i in range(3)], np.float32)
        if not oracle.r2(aw, b, box32) < rl2:
            continue
        for i in range(3):
            ca, cb = coarse(aw[i], box32[i], dims[i]), coarse(b[i], box32[i], dims[i])
            assert adjacent(ca, cb, dims[i]), (box, dims, i, aw, b)
        checked += 1
    return checked


@pytest.mark.parametrize("box,cutoff,skin", [
    ([30.0, 30.0, 30.0], 5.75, 1.0),
    ([468.88, 468.88, 468.88], 5.75, 1.0),
    ([20.0, 45.3, 101.7], 3.0, 1.0),
])
def test_pairs_within_rl_fall_in_adjacent_coarse_cells(box, cutoff, skin):
    assert check_pairs(box, cutoff, skin, seed=len(box) + int(box[1])) > 1000


def test_tight_cells_barely_wider_than_rl():
    rl = 6.75
    L = tight_box(rl)
    dims = nl.nl_halo_grid([L, L, L], 5.75, 1.0)
    assert dims == (3, 3, 3)
    assert L / 3 > rl
    assert check_pairs([L, L, L], 5.75, 1.0, seed=7) > 1000


def test_grid_follows_the_stated_width_and_clamps():
    for L, rl in [(30.0, 6.75), (468.88, 6.75), (101.7, 4.0), (1e6, 1.0), (1.0, 5.0)]:
        want = math.floor(L / (float(np.float32(rl)) * (1 + 2.0 ** -10) + L * 2.0 ** -16))
        want = min(max(want, 1), 1024)
        cut = rl - 1.0
        dims = nl.nl_halo_grid([L, L, L], cut, 1.0)
        assert dims == (want,) * 3, (L, rl, dims)
    assert nl.nl_halo_grid([1e6, 1e6, 1e6], 0.5, 0.5) == (1024, 1024, 1024)
    assert nl.nl_halo_grid([1.0, 1.0, 1.0], 4.0, 1.0) == (1, 1, 1)


@pytest.mark.parametrize("box,cutoff,skin", [
    ([30.0, 30.0, 30.0], -1.0, 1.0),
    ([30.0, 30.0, 30.0], 5.0, -0.5),
    ([30.0, 30.0, 30.0], float("nan"), 1.0),
    ([30.0, 30.0, 30.0], 0.0, 0.0),
    ([0.0, 30.0, 30.0], 5.0, 1.0),
    ([30.0, float("inf"), 30.0], 5.0, 1.0),
])
def test_bad_arguments_are_refused(box, cutoff, skin):
    with pytest.raises(nl.NLError):
        nl.nl_halo_grid(box, cutoff, skin)

"""GPU path vs the CPU oracle, through the C ABI (bit-exact).

Curve order: the permutation (ties by index) and keys equal the oracle's at
every size, the 1M and 10M workloads included.  Neighbor lists: every
canonicalised row and count equals the oracle's, at full size too.  All inputs are the seeded workloads of
neighbor_list_construction_b200.workloads.
"""
import numpy as np
import pytest
import torch

import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nl():
    from neighbor_list_construction_b200 import nl as _nl
    return _nl


@pytest.fixture(scope="module")
def ctx(nl):
    c = nl.Context(10_400_000, 320)
    yield c
    c.close()


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def gpu_sort(ctx, pos, box, curve="hilbert"):
    perm, ps, ks = ctx.sort(dev(pos), box, curve, keys=True)
    assert ctx.sync_status() == 0
    return perm.cpu().numpy(), ps.cpu().numpy(), ks.cpu().numpy().view(np.uint64)


def gpu_build(ctx, pos, box, cutoff, skin, K):
    nbr, cnt = ctx.build(dev(pos), box, cutoff, skin, K)
    st = ctx.sync_status()
    return nbr.cpu().numpy(), cnt.cpu().numpy(), st


# ------------------------------------------------------------------ curve order
@pytest.mark.parametrize("name", ["uniform4k", "lattice60k", "saltwater_n20"])
@pytest.mark.parametrize("curve", ["hilbert", "morton"])
def test_sort_matches_oracle(ctx, oracle, name, curve):
    w = gu.workload(name)
    perm, ps, ks = gpu_sort(ctx, w.pos, w.box, curve)
    o_perm, o_ks = oracle.sort(w.pos, w.box, curve)
    np.testing.assert_array_equal(ks, o_ks)
    np.testing.assert_array_equal(perm, o_perm)
    np.testing.assert_array_equal(ps[:, :3], w.pos[o_perm, :3])
    np.testing.assert_array_equal(ps[:, 3].view(np.int32), o_perm)


@pytest.mark.parametrize("n", [1, 2, 3, 31, 33, 4095, 4096, 4097, 12289, 65537])
def test_sort_ragged_sizes(ctx, oracle, n):
    rng = np.random.default_rng(n)
    box = np.array([50.0, 61.5, 43.25], np.float32)
    pos = np.zeros((n, 4), np.float32)
    pos[:, :3] = rng.uniform(-0.5, 1.5, (n, 3)) * box  # some outside the box
    if n > 8:
        pos[: n // 4, :3] = pos[n // 4: 2 * (n // 4), :3]  # duplicates -> equal keys
    perm, ps, ks = gpu_sort(ctx, pos, box)
    o_perm, o_ks = oracle.sort(pos, box)
    np.testing.assert_array_equal(ks, o_ks)
    np.testing.assert_array_equal(perm, o_perm)


# The sort finishes short runs of equal top-24-bit key prefixes in place and
# falls back to all eight digit passes when a run is longer than 64 keys:
# identical points give runs of exactly 64 and 65, a dense cluster gives runs
# of thousands, and an all-equal input is one run of n.
@pytest.mark.parametrize("case", ["run64", "run65", "cluster", "all_equal"])
def test_sort_long_prefix_runs(ctx, oracle, case):
    rng = np.random.default_rng(7)
    box = np.array([40.0, 40.0, 40.0], np.float32)
    n = 20000
    pos = np.zeros((n, 4), np.float32)
    pos[:, :3] = rng.uniform(0.0, 1.0, (n, 3)) * box
    if case == "run64":
        pos[100:164, :3] = pos[5000, :3]
        pos[5000, :3] = pos[3000, :3]
    elif case == "run65":
        pos[100:165, :3] = pos[5000, :3]
        pos[5000, :3] = pos[3000, :3]
    elif case == "cluster":
        c = rng.uniform(0.0, 1.0, 3).astype(np.float32) * box
        pos[: n // 4, :3] = c + rng.uniform(0.0, 0.02, (n // 4, 3)).astype(np.float32)
    else:
        pos[:, :3] = box * np.float32(0.3)
    perm, ps, ks = gpu_sort(ctx, pos, box)
    o_perm, o_ks = oracle.sort(pos, box)
    np.testing.assert_array_equal(ks, o_ks)
    np.testing.assert_array_equal(perm, o_perm)
    np.testing.assert_array_equal(ps[:, :3], pos[o_perm, :3])


@pytest.mark.parametrize("name", ["saltwater1m", "saltwater10m", "shell10m"])
@pytest.mark.parametrize("curve", ["hilbert", "morton"])
def test_sort_full_size(ctx, oracle, name, curve):
    """The whole permutation, sorted keys and sorted positions of the 1M and
    10M workloads, both curves."""
    w = gu.workload(name)
    perm, ps, ks = gpu_sort(ctx, w.pos, w.box, curve)
    o_perm, o_ks = oracle.sort(w.pos, w.box, curve)
    np.testing.assert_array_equal(ks, o_ks)
    np.testing.assert_array_equal(perm, o_perm)
    np.testing.assert_array_equal(ps[:, :3], w.pos[o_perm, :3])


# --------------------------------------------------------------- neighbor lists
def test_build_uniform4k_equals_bruteforce(ctx, oracle):
    w = gu.workload("uniform4k")
    nbr, cnt, st = gpu_build(ctx, w.pos, w.box, w.cutoff, w.skin, w.capacity)
    o_nbr, o_cnt, o_ov = oracle.bruteforce(w.pos, w.box, w.cutoff, w.skin, w.capacity)
    assert st == 0 and not o_ov
    gu.assert_rows_match(nbr, cnt, o_nbr, o_cnt)


@pytest.mark.parametrize("name", ["lattice60k", "saltwater_n20", "uniform4k"])
def test_build_matches_oracle_on_sorted_positions(ctx, oracle, name):
    w = gu.workload(name)
    ps = gu.oracle_sorted(name)
    nbr, cnt, st = gpu_build(ctx, ps, w.box, w.cutoff, w.skin, w.capacity)
    o_nbr, o_cnt, o_ov = oracle.build(ps, w.box, w.cutoff, w.skin, w.capacity)
    assert st == (1 if o_ov else 0)
    gu.assert_rows_match(nbr, cnt, o_nbr, o_cnt)


@pytest.mark.parametrize("box,cutoff,skin", [
    ([7.5, 7.5, 7.5], 2.0, 0.5),        # exactly 3 rl: 2 cells -> error (margin)
    ([7.6, 7.6, 7.6], 2.0, 0.5),        # 3 cells per axis, literal min image
    ([10.1, 10.1, 10.1], 2.0, 0.5),     # 4 cells per axis, literal
    ([13.0, 10.1, 7.6], 2.0, 0.5),      # orthorhombic, mixed
    ([12.6, 20.0, 31.0], 2.0, 0.5),     # >= 5 cells everywhere: shifted path
])
def test_build_small_boxes(ctx, oracle, box, cutoff, skin):
    rng = np.random.default_rng(5)
    box = np.array(box, np.float32)
    n = int(0.1 * np.prod(box)) + 7
    pos = np.zeros((n, 4), np.float32)
    pos[:, :3] = rng.random((n, 3)) * box
    edge = np.array([[0, 0, 0], [-0.0, 0, 0], [box[0], 0, 0], [box[0] + 2.0, 0, 0],
                     [2.5, 0, 0], [box[0] - 1e-3, box[1] - 1e-3, box[2] - 1e-3],
                     [-1e-8, -1e-8, -1e-8]], np.float32)
    pos[:7, :3] = edge
    o_nbr, o_cnt, o_ov = oracle.bruteforce(pos, box, cutoff, skin, 64)
    if box[0] == np.float32(7.5):
        from neighbor_list_construction_b200 import nl as _nl
        with pytest.raises(_nl.NLError) as e:
            ctx.build(dev(pos), box, cutoff, skin, 64)
        assert e.value.status == _nl.NL_ERR_BOX
        return
    nbr, cnt, st = gpu_build(ctx, pos, box, cutoff, skin, 64)
    gu.assert_rows_match(nbr, cnt, o_nbr, o_cnt)


@pytest.mark.parametrize("case", ["one_atom", "two_coincident", "all_coincident",
                                  "on_the_faces", "far_outside", "cutoff_zero_skin"])
def test_build_degenerate_inputs(ctx, oracle, case):
    """Inputs at the edges of the definition: a single atom, coincident atoms
    (r2 = 0 < rl2: neighbors of each other), every atom at one point (rows of
    n - 1), atoms exactly on the box faces (x = 0 and x = L wrap together),
    coordinates many boxes away, and rl = skin alone (cutoff 0)."""
    rng = np.random.default_rng(31)
    box = np.array([20.0, 22.0, 24.0], np.float32)
    cutoff, skin, K = 2.5, 0.5, 64
    if case == "one_atom":
        pos = np.zeros((1, 4), np.float32)
        pos[0, :3] = [3.0, 4.0, 5.0]
    elif case == "two_coincident":
        pos = np.zeros((2, 4), np.float32)
        pos[:, :3] = [7.0, 7.0, 7.0]
    elif case == "all_coincident":
        pos = np.zeros((50, 4), np.float32)
        pos[:, :3] = [1.0, 21.5, 0.0]
    elif case == "on_the_faces":
        n = 600
        pos = np.zeros((n, 4), np.float32)
        pos[:, :3] = rng.random((n, 3)) * box
        face = rng.integers(0, 3, n)
        side = rng.integers(0, 2, n).astype(np.float32)
        pos[np.arange(n), face] = side * box[face]
    elif case == "far_outside":
        n = 800
        pos = np.zeros((n, 4), np.float32)
        pos[:, :3] = (rng.random((n, 3)) * 2.0 - 1.0) * box * 40.0
    else:
        cutoff, skin = 0.0, 3.0
        n = 900
        pos = np.zeros((n, 4), np.float32)
        pos[:, :3] = rng.random((n, 3)) * box
    nbr, cnt, st = gpu_build(ctx, pos, box, cutoff, skin, K)
    o_nbr, o_cnt, o_ov = oracle.build(pos, box, cutoff, skin, K)
    assert st == (1 if o_ov else 0)
    gu.assert_rows_match(nbr, cnt, o_nbr, o_cnt)
    if case == "all_coincident":
        assert np.all(cnt == 49)


def test_build_golden_fixtures(ctx):
    import glob
    import json
    import os
    for path in sorted(glob.glob(os.path.join(os.path.dirname(__file__), "golden", "tiny_*.json"))):
        g = json.load(open(path))
        pos = np.zeros((len(g["positions"]), 4), np.float32)
        pos[:, :3] = np.array(g["positions"], np.float32)
        # the fixtures' boxes hold 3-4 cells: they exercise the literal path
        nbr, cnt, st = gpu_build(ctx, pos, g["box"], g["cutoff"], g["skin"], g["capacity"])
        np.testing.assert_array_equal(cnt, np.array(g["counts"], np.int32))
        exp = np.array(g["rows"], np.int32)
        ok = cnt <= g["capacity"]
        np.testing.assert_array_equal(gu.canonical(nbr)[ok], exp[ok])
        assert st == (1 if g.get("overflow") else 0)


def test_overflow_status_and_rows(ctx, oracle):
    rng = np.random.default_rng(18)
    box = np.array([20.0, 20.0, 20.0], np.float32)
    pos = np.zeros((300, 4), np.float32)
    pos[:, :3] = rng.random((300, 3)) * 3.0 + 5.0
    nbr, cnt, st = gpu_build(ctx, pos, box, 2.0, 0.5, 16)
    o_nbr, o_cnt, o_ov = oracle.build(pos, box, 2.0, 0.5, 16)
    full, fcnt, _ = oracle.build(pos, box, 2.0, 0.5, 400)
    sets = [set(full[i, :fcnt[i]].tolist()) for i in range(300)]
    assert o_ov and st == 1
    gu.assert_rows_match(nbr, cnt, o_nbr, o_cnt, full_sets=sets)


@pytest.mark.parametrize("m", [255, 256, 700, 800])
def test_build_crowded_cell(ctx, oracle, m):
    """One cell holding m atoms among a uniform background: 255 is the
    largest cell the in-cell sort orders (its sub-bin counts fill a byte),
    256 stays in scatter order and sends the build to the per-atom search,
    700 still fits the sort's shared-memory stage (768 atoms), 800 does
    not.  Rows past the capacity must be members of the full sets."""
    rng = np.random.default_rng(m)
    L, cutoff, skin, K = 30.0, 2.5, 0.5, 320
    bg = 2000
    pos = np.zeros((bg + m, 4), np.float32)
    pos[:bg, :3] = rng.random((bg, 3)) * L
    # cells are 30/9 wide in x and 30/19 in y and z: the crowd sits inside
    # cell (4, 9, 9), whose centre is (15, 15, 15)
    pos[bg:, :3] = 14.8 + rng.random((m, 3)) * 0.4
    box = np.array([L, L, L], np.float32)
    nbr, cnt, st = gpu_build(ctx, pos, box, cutoff, skin, K)
    full, fcnt, _ = oracle.build(pos, box, cutoff, skin, 1024)
    assert fcnt.max() < 1024
    o_nbr, o_cnt, o_ov = oracle.build(pos, box, cutoff, skin, K)
    assert st == (1 if o_ov else 0)
    sets = [set(full[i, :fcnt[i]].tolist()) for i in range(pos.shape[0])]
    gu.assert_rows_match(nbr, cnt, o_nbr, o_cnt, full_sets=sets)


@pytest.mark.parametrize("K", [102, 104])
def test_build_capacity_not_multiple_of_vector(ctx, oracle, K):
    """A box large enough for the staged kernel, with a capacity that is
    (104) or is not (102) a whole number of 16-byte row vectors: the second
    goes to the per-atom kernel; both must equal the oracle, overflowing
    rows included."""
    rng = np.random.default_rng(23)
    L = 40.0
    n = 7000
    pos = np.zeros((n, 4), np.float32)
    pos[:, :3] = rng.random((n, 3)) * L
    box = np.array([L, L, L], np.float32)
    nbr, cnt, st = gpu_build(ctx, pos, box, 5.75, 1.0, K)
    o_nbr, o_cnt, o_ov = oracle.build(pos, box, 5.75, 1.0, K)
    assert st == (1 if o_ov else 0)
    gu.assert_rows_match(nbr, cnt, o_nbr, o_cnt)


def test_build_cutoff_shell_pairs(ctx, oracle):
    """Partners placed within a few ulps of the cutoff radius: every pair
    decision sits on the r2 < rl2 boundary, so any change in rounding (a
    fused multiply-add, a reordered sum) flips some of them."""
    rng = np.random.default_rng(17)
    L, cutoff, skin = 48.0, 5.75, 1.0
    rl = np.float64(np.float32(cutoff + skin))
    nb = 6000
    base = rng.random((nb, 3)) * L
    u = rng.normal(size=(nb, 3))
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    r = rl * (1.0 + rng.uniform(-3e-7, 3e-7, size=(nb, 1)))
    pos = np.zeros((2 * nb, 4), np.float32)
    pos[:nb, :3] = base
    pos[nb:, :3] = base + r * u
    box = np.array([L, L, L], np.float32)
    nbr, cnt, st = gpu_build(ctx, pos, box, cutoff, skin, 256)
    o_nbr, o_cnt, o_ov = oracle.build(pos, box, cutoff, skin, 256)
    assert st == (1 if o_ov else 0)
    gu.assert_rows_match(nbr, cnt, o_nbr, o_cnt)


def test_build_pairs_that_a_fused_sum_would_flip(ctx, oracle):
    """The predicate is r2 = (dx*dx + dy*dy) + dz*dz with every product and
    sum rounded to fp32.  Pairs are chosen (from many near the cutoff radius)
    whose decision r2 < rl2 changes if either sum were fused with the product
    before it (one rounding instead of two); the GPU rows must equal the
    oracle's (unfused) on all of them."""
    rng = np.random.default_rng(29)
    L, cutoff, skin = 96.0, 5.75, 1.0
    rl2 = np.float32(np.float32(cutoff + skin) * np.float32(cutoff + skin))
    rl = np.float64(np.float32(cutoff + skin))
    nb = 20000
    base = rng.random((nb, 3)) * L
    u = rng.normal(size=(nb, 3))
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    r = rl * (1.0 + rng.uniform(-3e-7, 3e-7, size=(nb, 1)))
    a = np.float32(base)
    b = np.float32(base + r * u) % np.float32(L)
    d = (b - a).astype(np.float32)                       # fp32 differences
    d -= np.float32(L) * np.round(d / np.float32(L)).astype(np.float32)
    sq = (d * d).astype(np.float32)
    s_xy = (sq[:, 0] + sq[:, 1]).astype(np.float32)
    plain = (s_xy + sq[:, 2]).astype(np.float32)

    def fma(x, y, z):   # one rounding (exact product in fp64, then to fp32)
        return np.float32(np.float64(x) * np.float64(y) + np.float64(z))

    f_xy = fma(d[:, 0], d[:, 0], sq[:, 1])
    fused = [(f_xy + sq[:, 2]).astype(np.float32), fma(d[:, 2], d[:, 2], s_xy),
             fma(d[:, 2], d[:, 2], f_xy)]
    flips = np.zeros(nb, bool)
    for f in fused:
        flips |= (f < rl2) != (plain < rl2)
    assert flips.sum() >= 50                              # the test has teeth
    pos = np.zeros((2 * nb, 4), np.float32)
    pos[:nb, :3] = a
    pos[nb:, :3] = b
    box = np.array([L, L, L], np.float32)
    nbr, cnt, st = gpu_build(ctx, pos, box, cutoff, skin, 256)
    o_nbr, o_cnt, o_ov = oracle.build(pos, box, cutoff, skin, 256)
    assert st == (1 if o_ov else 0)
    gu.assert_rows_match(nbr, cnt, o_nbr, o_cnt)
    # each flip-prone pair: the oracle's r2 is the plain sum, and the pair is
    # in both rows exactly when that sum is below rl2
    can = gu.canonical(np.asarray(nbr))
    for k in np.nonzero(flips)[0]:
        assert oracle.r2(a[k], b[k], box) == plain[k]
        inside = plain[k] < rl2
        assert (nb + k in can[k]) == inside and (k in can[nb + k]) == inside


def test_build_mixed_density_uses_both_paths(ctx, nl, oracle):
    """A dense slab whose tiles overflow the shared-memory stage (listed for
    the per-atom search) beside sparse tiles that are staged; rows with more
    neighbors than the capacity are checked as subsets."""
    rng = np.random.default_rng(44)
    box = np.array([25.0, 25.0, 25.0], np.float32)
    # 9 cells of 2.78 A per axis; the slab fills x-cells 0 and 1 with ~200
    # atoms per cell, so a tile's 9 rows hold ~3,600 atoms (over the stage)
    sparse = rng.random((1600, 3)) * box
    dense = rng.random((32400, 3)) * np.array([5.5, 25.0, 25.0])
    pos = np.zeros((34000, 4), np.float32)
    pos[:, :3] = np.concatenate([sparse, dense])[rng.permutation(34000)]
    K = 256
    nbr, cnt, st = gpu_build(ctx, pos, box, 2.0, 0.5, K)
    info = nl.nl_last_build_info(ctx.handle)
    assert info[3] == 1  # staged kernel ran (dense tiles went to the listed path)
    full, fcnt, _ = oracle.build(pos, box, 2.0, 0.5, 1024)
    o_nbr = full[:, :K]
    sets = [set(full[i, :fcnt[i]].tolist()) for i in range(pos.shape[0])]
    assert st == (1 if (fcnt > K).any() else 0)
    gu.assert_rows_match(nbr, cnt, np.where(np.arange(K) < fcnt[:, None], o_nbr, -1), fcnt,
                         full_sets=sets)


@pytest.mark.parametrize("name", ["saltwater1m", "saltwater10m", "shell10m"])
def test_build_full_size(ctx, oracle, name):
    """Full-size workloads in the order the benchmark uses (curve-sorted):
    every row and count against the oracle, and the overflow status."""
    w = gu.workload(name)
    ps = gu.oracle_sorted(name)
    nbr_t, cnt_t = ctx.build(dev(ps), w.box, w.cutoff, w.skin, w.capacity)
    st = ctx.sync_status()
    over = gu.assert_all_rows_match(oracle, nbr_t, cnt_t, ps, w.box, w.cutoff, w.skin,
                                    w.capacity)
    assert st == (1 if over else 0)


@pytest.mark.parametrize("name", ["saltwater10m", "shell10m"])
def test_build_full_size_unsorted_input(ctx, oracle, name):
    """The same workloads in their shuffled input order (no curve sort): the
    cell binning alone decides the staging, every row is compared."""
    w = gu.workload(name)
    nbr_t, cnt_t = ctx.build(dev(w.pos), w.box, w.cutoff, w.skin, w.capacity)
    st = ctx.sync_status()
    over = gu.assert_all_rows_match(oracle, nbr_t, cnt_t, w.pos, w.box, w.cutoff, w.skin,
                                    w.capacity)
    assert st == (1 if over else 0)


# ------------------------------------------------------------------ skin check
def test_skin_special_cases(ctx, nl):
    box = [10.0, 10.0, 10.0]
    ref = np.zeros((10, 4), np.float32)
    ref[:, :3] = 1.0
    r = dev(ref)
    ctx.build(r, box, 2.0, 1.0, 32)
    rb, md = ctx.skin_check(r, box, 1.0)
    assert rb.item() == 0 and md.item() == 0.0
    p = ref.copy()
    p[3, 0] = 1.5  # exactly h = 0.5 -> r2 = 0.25 = h^2, strict -> no rebuild
    rb, md = ctx.skin_check(dev(p), box, 1.0)
    assert rb.item() == 0 and md.item() == 0.25
    p[3, 0] = np.nextafter(np.float32(1.5), np.float32(2))
    rb, md = ctx.skin_check(dev(p), box, 1.0)
    assert rb.item() == 1 and md.item() > 0.25
    assert ctx.sync_status() == 0


def test_skin_matches_oracle(ctx, oracle):
    w = gu.workload("lattice60k")
    p0 = dev(w.pos)
    ctx.build(p0, w.box, w.cutoff, w.skin, w.capacity)
    rng = np.random.default_rng(9)
    for scale in (0.05, 0.2, 0.35, 0.6):
        moved = w.pos.copy()
        moved[:, :3] += rng.normal(0, scale, (w.n, 3)).astype(np.float32)
        moved[:5, :3] += w.box  # a few atoms crossed the box: min image
        rb, md = ctx.skin_check(dev(moved), w.box, w.skin)
        o_m, o_rb = oracle.skin_check(moved, w.pos, w.box, w.skin)
        assert md.item() == o_m and bool(rb.item()) == o_rb


def test_displacement_stand_in_matches_oracle(ctx, nl, oracle):
    w = gu.workload("lattice60k")
    p = dev(w.pos)
    for step in (1, 2, 17):
        nl.nls_displace(p, 77, step, 0.02)
    exp = w.pos.copy()
    for step in (1, 2, 17):
        exp = oracle.displace(exp, 77, step, 0.02)
    np.testing.assert_array_equal(p.cpu().numpy()[:, :3], exp[:, :3])


# ------------------------------------------------------------------ replay
def _replay(ctx, nl, oracle, name, steps, seed=2024, check_lists=True):
    """nl_replay of `steps` steps against the oracle's loop: the decisions, the
    final positions and every row of the lists of the last rebuild."""
    w = gu.workload(name)
    ps = gu.oracle_sorted(name)
    p = dev(ps)
    nbr, cnt = ctx.build(p, w.box, w.cutoff, w.skin, w.capacity)
    g = nl.nls_step_graph(p, seed, nl.nl_step_counter(ctx.handle), w.sigma_step)
    dec = torch.full((steps,), -1, dtype=torch.int32, device="cuda")
    try:
        nl.nl_replay(ctx.handle, g, steps, p, w.box, w.cutoff, w.skin, w.capacity, nbr, cnt, dec)
        st = ctx.sync_status()
    finally:
        nl.nls_graph_destroy(g)
    o_dec, o_final, o_ref = oracle.md_decisions(ps, w.box, w.skin, seed, w.sigma_step, steps)
    np.testing.assert_array_equal(dec.cpu().numpy(), o_dec)
    np.testing.assert_array_equal(p.cpu().numpy()[:, :3], o_final[:, :3])
    if check_lists:
        # the lists of the last rebuild: built on the positions of that step
        over = gu.assert_all_rows_match(oracle, nbr, cnt, o_ref, w.box, w.cutoff, w.skin,
                                        w.capacity)
        assert st == (1 if over else 0)
    return o_dec


def test_replay_lattice60k_50_steps(ctx, nl, oracle):
    dec = _replay(ctx, nl, oracle, "lattice60k", 50)
    assert dec.sum() >= 1


def test_replay_twice_reuses_graph(ctx, nl, oracle):
    _replay(ctx, nl, oracle, "uniform4k", 30, seed=5)
    _replay(ctx, nl, oracle, "uniform4k", 30, seed=5)


def test_replay_salt_solution_200_steps(ctx, nl, oracle):
    dec = _replay(ctx, nl, oracle, "saltwater10m", 200)
    assert 3 <= dec.sum() <= 40


# ---------------------------------------------------------- replay, re-sorted
def _replay_resort(ctx, nl, oracle, name, steps, start, seed=2024):
    """nl_replay_resort against the oracle's plain interval: with the stand-in
    keyed by atom id, re-sorting only permutes the trajectory, so decisions
    are equal and every array is the oracle's, permuted by the final ids."""
    w = gu.workload(name)
    p0 = gu.oracle_sorted(name) if start == "curve" else w.pos
    n = w.n
    p = dev(p0)
    ids = torch.arange(n, dtype=torch.int32, device="cuda")
    aux0 = np.random.default_rng(1).random((n, 4)).astype(np.float32)
    aux = dev(aux0)
    nbr, cnt = ctx.build(p, w.box, w.cutoff, w.skin, w.capacity)
    g = nl.nls_step_graph_ids(p, ids, seed, nl.nl_step_counter(ctx.handle), w.sigma_step)
    dec = torch.full((steps,), -1, dtype=torch.int32, device="cuda")
    try:
        nl.nl_replay_resort(ctx.handle, g, steps, p, ids, aux, w.box, w.cutoff, w.skin,
                            w.capacity, nbr, cnt, dec)
        st = ctx.sync_status()
    finally:
        nl.nls_graph_destroy(g)
    o_dec, o_final, o_ref = oracle.md_decisions(p0, w.box, w.skin, seed, w.sigma_step, steps)
    np.testing.assert_array_equal(dec.cpu().numpy(), o_dec)
    idh = ids.cpu().numpy()
    np.testing.assert_array_equal(np.sort(idh), np.arange(n))
    np.testing.assert_array_equal(p.cpu().numpy(), o_final[idh])
    np.testing.assert_array_equal(aux.cpu().numpy(), aux0[idh])
    if o_dec.any():
        # the last rebuild put the atoms in curve order of their positions then
        k = oracle.keys(o_ref, w.box)[idh]
        assert np.all(k[1:] >= k[:-1])
    else:
        np.testing.assert_array_equal(idh, np.arange(n))
    # rows by atom id: slot k holds atom idh[k], its entries are slots too
    g_nbr = nbr.cpu().numpy()
    by_id = np.full_like(g_nbr, -1)
    by_id[idh] = np.where(g_nbr >= 0, idh[np.maximum(g_nbr, 0)], -1)
    by_cnt = np.zeros(n, np.int32)
    by_cnt[idh] = cnt.cpu().numpy()
    o_nbr, o_cnt, o_ov = oracle.build(o_ref, w.box, w.cutoff, w.skin, w.capacity)
    assert st == (1 if o_ov else 0)
    gu.assert_rows_match(by_id, by_cnt, o_nbr, o_cnt)
    return o_dec, idh


@pytest.mark.parametrize("name,steps,start", [("lattice60k", 50, "input"),
                                              ("saltwater_n20", 120, "input"),
                                              ("saltwater_n20", 120, "curve"),
                                              ("uniform4k", 1, "input")])
def test_replay_resort(ctx, nl, oracle, name, steps, start):
    dec, ids = _replay_resort(ctx, nl, oracle, name, steps, start)
    if steps > 1:
        assert dec.sum() >= 1
    if start == "input" and dec.any():
        assert not np.array_equal(ids, np.arange(ids.size))


def test_replay_resort_without_ids_or_aux(ctx, nl, oracle):
    """ids and aux are optional; pos alone is permuted.  The stand-in is keyed
    by slot here, so after the first re-sort the trajectory is no longer the
    oracle's: decisions are compared up to and including the first rebuild."""
    w = gu.workload("lattice60k")
    p = dev(w.pos)
    nbr, cnt = ctx.build(p, w.box, w.cutoff, w.skin, w.capacity)
    g = nl.nls_step_graph(p, 11, nl.nl_step_counter(ctx.handle), w.sigma_step)
    dec = torch.full((40,), -1, dtype=torch.int32, device="cuda")
    try:
        nl.nl_replay_resort(ctx.handle, g, 40, p, None, None, w.box, w.cutoff, w.skin,
                            w.capacity, nbr, cnt, dec)
        assert ctx.sync_status() == 0
    finally:
        nl.nls_graph_destroy(g)
    d = dec.cpu().numpy()
    o_dec, _, _ = oracle.md_decisions(w.pos, w.box, w.skin, 11, w.sigma_step, 40)
    first = int(np.argmax(o_dec)) if o_dec.any() else 40
    np.testing.assert_array_equal(d[: first + 1], o_dec[: first + 1])
    assert set(np.unique(d)) <= {0, 1}


# ------------------------------------------------------------------ errors
def test_argument_errors(ctx, nl):
    p = dev(np.zeros((10, 4), np.float32))
    with pytest.raises(nl.NLError) as e:
        ctx.build(p, [10, 10, 10], 2.0, 0.5, 400)
    assert e.value.status == nl.NL_ERR_CAPACITY
    with pytest.raises(nl.NLError) as e:
        ctx.build(p, [10, 10, 10], -1.0, 0.5, 16)
    assert e.value.status == nl.NL_ERR_ARG
    with pytest.raises(nl.NLError) as e:
        ctx.build(p, [10, 0, 10], 2.0, 0.5, 16)
    assert e.value.status == nl.NL_ERR_ARG
    with pytest.raises(nl.NLError) as e:
        ctx.build(p, [5, 10, 10], 2.0, 0.5, 16)
    assert e.value.status == nl.NL_ERR_BOX
    assert ctx.sync_status() == 0


def test_empty_input(ctx, nl):
    p = torch.zeros((0, 4), dtype=torch.float32, device="cuda")
    nbr, cnt = ctx.build(p, [10, 10, 10], 2.0, 0.5, 16)
    perm, ps, _ = ctx.sort(p, [10, 10, 10])
    rb, md = ctx.skin_check(p, [10, 10, 10], 0.5)
    assert rb.item() == 0 and ctx.sync_status() == 0

"""nl_edge_features on the GPU against the oracle's per-slot edge features:
rows built on the GPU (any slot order) carry, slot by slot, the features the
oracle gives the same (i, j); synthetic rows with arbitrary pairs, padding,
overflowing and negative counts and out-of-range indices match bit for bit;
and a full-size salt solution matches on sampled rows."""
import numpy as np
import pytest
import torch

import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ctx():
    from neighbor_list_construction_b200 import nl
    c = nl.Context(10_400_000, 320)
    yield c
    c.close()


@pytest.fixture(scope="module")
def nl():
    from neighbor_list_construction_b200 import nl as _nl
    return _nl


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bits(a):
    return np.ascontiguousarray(a, np.float32).view(np.uint32)


def full_features(pos, box, cutoff, skin, oracle):
    """Oracle rows with room for every neighbor, and their features."""
    _, cnt, _ = oracle.build(pos, box, cutoff, skin, 1)
    K = max(int(cnt.max()), 1)
    o_nbr, o_cnt, _ = oracle.build(pos, box, cutoff, skin, K)
    return o_nbr, o_cnt, oracle.edge_features(pos, box, o_nbr, o_cnt)


def test_edges_of_gpu_rows(ctx, oracle):
    for name in ("uniform4k", "lattice60k", "saltwater_n20"):
        w = gu.workload(name)
        p = dev(w.pos)
        nbr, cnt = ctx.build(p, w.box, w.cutoff, w.skin, w.capacity)
        e = ctx.edge_features(p, w.box, nbr, cnt)
        assert ctx.sync_status() == 0
        g_nbr, g_cnt, g_e = nbr.cpu().numpy(), cnt.cpu().numpy(), e.cpu().numpy()
        # the rows are the oracle's rows, and each slot carries the oracle
        # feature of its own pair (looked up in the oracle's ascending rows)
        o_nbr, o_cnt, o_ov = oracle.build(w.pos, w.box, w.cutoff, w.skin, w.capacity)
        assert not o_ov
        gu.assert_rows_match(g_nbr, g_cnt, o_nbr, o_cnt)
        o_e = oracle.edge_features(w.pos, w.box, o_nbr, o_cnt)
        order = np.argsort(np.where(g_nbr < 0, np.iinfo(np.int32).max, g_nbr), axis=1,
                           kind="stable")
        g_sorted = np.take_along_axis(g_e, order[:, :, None], axis=1)
        np.testing.assert_array_equal(bits(g_sorted), bits(o_e))
        valid = np.arange(w.capacity)[None, :] < g_cnt[:, None]
        np.testing.assert_array_equal(bits(g_e[~valid]), 0)


def test_edges_overflowing_rows(ctx, oracle):
    w = gu.workload("saltwater_n20")
    p = dev(w.pos)
    K = 48                                # below most counts: every row overflows
    nbr, cnt = ctx.build(p, w.box, w.cutoff, w.skin, K)
    e = ctx.edge_features(p, w.box, nbr, cnt)
    assert ctx.sync_status() == 1
    g_nbr, g_cnt, g_e = nbr.cpu().numpy(), cnt.cpu().numpy(), e.cpu().numpy()
    assert (g_cnt > K).mean() > 0.5
    o_nbr, o_cnt, o_e = full_features(w.pos, w.box, w.cutoff, w.skin, oracle)
    np.testing.assert_array_equal(g_cnt, o_cnt)
    for i in range(g_nbr.shape[0]):
        c = min(int(g_cnt[i]), K)
        # slot of each GPU entry in the oracle's complete, ascending row
        t = np.searchsorted(o_nbr[i, : o_cnt[i]], g_nbr[i, :c])
        np.testing.assert_array_equal(o_nbr[i, t], g_nbr[i, :c])
        np.testing.assert_array_equal(bits(g_e[i, :c]), bits(o_e[i, t]))
        np.testing.assert_array_equal(bits(g_e[i, c:]), 0)


@pytest.mark.parametrize("K", [1, 7, 32, 33, 100])
def test_edges_arbitrary_rows(ctx, oracle, K):
    """Rows that are not neighbor lists: far pairs through every face,
    self-pairs, indices -1 and n inside the counted prefix, counts above K,
    zero and negative; positions partly outside the box."""
    rng = np.random.default_rng(K)
    n = 3001
    box = np.array([31.0, 17.5, 23.25], np.float32)
    pos = np.zeros((n, 4), np.float32)
    pos[:, :3] = (rng.random((n, 3)) * 2.2 - 0.6) * box
    pos[:, 3] = rng.random(n)                 # the fourth lane is ignored
    nbr = rng.integers(0, n, (n, K)).astype(np.int32)
    nbr[rng.random((n, K)) < 0.05] = -1
    nbr[rng.random((n, K)) < 0.02] = n
    nbr[::11, 0] = np.arange(0, n, 11)        # self-pairs: zero displacement
    cnt = rng.integers(-3, K + 5, n).astype(np.int32)
    e = ctx.edge_features(dev(pos), box, dev(nbr), dev(cnt))
    assert ctx.sync_status() == 0
    np.testing.assert_array_equal(bits(e.cpu().numpy()),
                                  bits(oracle.edge_features(pos, box, nbr, cnt)))


def test_edges_empty_and_arguments(ctx, nl):
    box = [10.0, 10.0, 10.0]
    p = torch.zeros(0, 4, dtype=torch.float32, device="cuda")
    nb = torch.zeros(0, 8, dtype=torch.int32, device="cuda")
    c = torch.zeros(0, dtype=torch.int32, device="cuda")
    e = ctx.edge_features(p, box, nb, c)
    assert e.shape == (0, 8, 4)
    p = torch.zeros(4, 4, dtype=torch.float32, device="cuda")
    nb = torch.zeros(4, 8, dtype=torch.int32, device="cuda")
    c = torch.zeros(4, dtype=torch.int32, device="cuda")
    out = torch.zeros(4, 8, 4, dtype=torch.float32, device="cuda")
    with pytest.raises(nl.NLError):
        nl.nl_edge_features(ctx.handle, p, [10.0, -1.0, 10.0], nb, c, out)
    with pytest.raises(ValueError):
        nl.nl_edge_features(ctx.handle, p, box, nb.float(), c, out)
    assert ctx.sync_status() == 0


def test_edges_full_size_sampled(ctx, oracle):
    """saltwater10m in curve order, as the benchmark runs it: zero padding
    everywhere, and sampled rows against the oracle's rows and features (the
    sampled atoms and their oracle neighbors gathered into a compact
    problem), bit for bit."""
    w = gu.workload("saltwater10m")
    ps = gu.oracle_sorted("saltwater10m")
    p = dev(ps)
    nbr, cnt = ctx.build(p, w.box, w.cutoff, w.skin, w.capacity)
    e = ctx.edge_features(p, w.box, nbr, cnt)
    assert ctx.sync_status() == 0
    K = w.capacity
    valid = torch.arange(K, device="cuda")[None, :] < cnt.clamp(max=K)[:, None]
    nz = (e.view(torch.int32) != 0).any(dim=2)
    assert not bool((nz & ~valid).any())
    assert bool(nz[valid].all())          # no two atoms coincide: r > 0
    del valid, nz
    rng = np.random.default_rng(321)
    n = w.n
    sample = np.unique(np.concatenate([rng.choice(n, 2000, replace=False),
                                       np.arange(0, 32), np.arange(n - 32, n)]))
    idx = torch.from_numpy(sample).cuda()
    g_nbr = nbr[idx].cpu().numpy()
    g_cnt = cnt[idx].cpu().numpy()
    g_e = e[idx].cpu().numpy()
    o_nbr, o_cnt, o_ov = oracle.rows(ps, w.box, w.cutoff, w.skin, K, sample)
    assert not o_ov
    gu.assert_rows_match(g_nbr, g_cnt, o_nbr, o_cnt)
    # compact problem: sampled atoms first, then every oracle neighbor
    others = np.setdiff1d(np.unique(o_nbr[o_nbr >= 0]), sample)
    ids = np.concatenate([sample, others])
    pos_of = np.searchsorted(np.sort(ids), o_nbr.clip(min=0))
    rank = np.argsort(ids)
    c_nbr = np.full((ids.size, K), -1, np.int32)
    c_nbr[: sample.size] = np.where(o_nbr >= 0, rank[pos_of], -1)
    c_cnt = np.zeros(ids.size, np.int32)
    c_cnt[: sample.size] = o_cnt
    o_e = oracle.edge_features(ps[ids], w.box, c_nbr, c_cnt)[: sample.size]
    order = np.argsort(np.where(g_nbr < 0, np.iinfo(np.int32).max, g_nbr), axis=1,
                       kind="stable")
    g_sorted = np.take_along_axis(g_e, order[:, :, None], axis=1)
    np.testing.assert_array_equal(bits(g_sorted), bits(o_e))


# -------------------------------------------- features of rows in every regime
def check_rows_and_edges(ctx, oracle, pos, box, cutoff, skin, K):
    """nl_build then nl_edge_features: slot by slot the oracle's feature of
    the same (i, j), looked up in the oracle's complete rows; zeros in the
    padding."""
    p = dev(pos)
    nbr, cnt = ctx.build(p, box, cutoff, skin, K)
    st = ctx.sync_status()
    e = ctx.edge_features(p, box, nbr, cnt)
    assert ctx.sync_status() == 0
    g_nbr, g_cnt, g_e = nbr.cpu().numpy(), cnt.cpu().numpy(), e.cpu().numpy()
    o_nbr, o_cnt, o_e = full_features(pos, box, cutoff, skin, oracle)
    np.testing.assert_array_equal(g_cnt, o_cnt)
    for i in range(g_nbr.shape[0]):
        c = min(int(g_cnt[i]), K)
        t = np.searchsorted(o_nbr[i, : o_cnt[i]], g_nbr[i, :c])
        np.testing.assert_array_equal(o_nbr[i, t], g_nbr[i, :c])
        np.testing.assert_array_equal(bits(g_e[i, :c]), bits(o_e[i, t]))
        np.testing.assert_array_equal(bits(g_e[i, c:]), 0)
    return st


@pytest.mark.parametrize("box", [[7.6, 7.6, 7.6], [13.0, 10.1, 7.6]])
def test_edges_small_boxes(ctx, oracle, box):
    """Rows from the per-atom kernel with the literal minimum image."""
    rng = np.random.default_rng(9)
    box = np.array(box, np.float32)
    n = int(0.1 * np.prod(box)) + 7
    pos = np.zeros((n, 4), np.float32)
    pos[:, :3] = rng.random((n, 3)) * box
    check_rows_and_edges(ctx, oracle, pos, box, 2.0, 0.5, 64)


def test_edges_dense_slab(ctx, oracle):
    """Rows from the listed (dense) tiles and the per-atom search next to a
    sparse region; planted pairs across the periodic face."""
    rng = np.random.default_rng(5)
    box = np.array([25.0, 25.0, 25.0], np.float32)
    sparse = rng.random((1600, 3)) * box
    dense = rng.random((20000, 3)) * np.array([5.5, 25.0, 25.0])
    pos = np.zeros((21604, 4), np.float32)
    pos[:21600, :3] = np.concatenate([sparse, dense])
    pos[21600:, :3] = [[15.0, 12.0, 12.0], [15.0625, 12.0, 12.0],
                       [24.9375, 3.0, 3.0], [0.0, 3.0, 3.0]]
    check_rows_and_edges(ctx, oracle, pos, box, 2.0, 0.5, 256)


def test_edges_cutoff_shell(ctx, oracle):
    """Partners within a few ulps of rl: lengths at the edge of the
    membership test."""
    rng = np.random.default_rng(17)
    L, cutoff, skin = 48.0, 5.75, 1.0
    rl = np.float64(np.float32(cutoff + skin))
    nb = 4000
    base = rng.random((nb, 3)) * L
    u = rng.normal(size=(nb, 3))
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    pos = np.zeros((2 * nb, 4), np.float32)
    pos[:nb, :3] = base
    pos[nb:, :3] = base + rl * (1.0 + rng.uniform(-3e-7, 3e-7, size=(nb, 1))) * u
    box = np.array([L, L, L], np.float32)
    check_rows_and_edges(ctx, oracle, pos, box, cutoff, skin, 256)


# ----------------------------------------------------------------- CSR form
@pytest.mark.parametrize("K", [1, 33, 100])
def test_csr_of_arbitrary_rows(ctx, oracle, K):
    """to_csr on synthetic rows (indices -1 and n, counts above K, zero and
    negative): offsets and entries equal the oracle's CSR form, and each
    entry's feature equals the oracle's feature of its slot."""
    rng = np.random.default_rng(100 + K)
    n = 2501
    box = np.array([31.0, 17.5, 23.25], np.float32)
    pos = np.zeros((n, 4), np.float32)
    pos[:, :3] = (rng.random((n, 3)) * 2.2 - 0.6) * box
    nbr = rng.integers(0, n, (n, K)).astype(np.int32)
    nbr[rng.random((n, K)) < 0.05] = -1
    nbr[rng.random((n, K)) < 0.02] = n
    cnt = rng.integers(-3, K + 5, n).astype(np.int32)
    row_ptr, col, e = ctx.to_csr(dev(nbr), dev(cnt), dev(pos), box)
    assert ctx.sync_status() == 0
    o_ptr, o_col = oracle.csr(nbr, cnt)
    np.testing.assert_array_equal(row_ptr.cpu().numpy(), o_ptr)
    np.testing.assert_array_equal(col.cpu().numpy(), o_col)
    keep = np.arange(K)[None, :] < np.clip(cnt, 0, K)[:, None]
    o_e = oracle.edge_features(pos, box, nbr, cnt)[keep]
    np.testing.assert_array_equal(bits(e.cpu().numpy()), bits(o_e))
    r2, c2 = ctx.to_csr(dev(nbr), dev(cnt))          # entries only
    assert torch.equal(r2, row_ptr) and torch.equal(c2, col)


def test_csr_empty(ctx):
    nbr = torch.zeros(0, 8, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(0, dtype=torch.int32, device="cuda")
    row_ptr, col = ctx.to_csr(nbr, cnt)
    assert row_ptr.tolist() == [0] and col.numel() == 0


def test_csr_full_size(ctx):
    """saltwater10m rows (1.29 G entries, past 2^30: the offsets are int64):
    the CSR form equals the rows' valid prefixes, row after row."""
    w = gu.workload("saltwater10m")
    p = dev(gu.oracle_sorted("saltwater10m"))
    nbr, cnt = ctx.build(p, w.box, w.cutoff, w.skin, w.capacity)
    row_ptr, col = ctx.to_csr(nbr, cnt)
    assert ctx.sync_status() == 0
    v = cnt.clamp(min=0, max=w.capacity).to(torch.int64)
    assert int(row_ptr[-1].item()) == int(v.sum().item()) > 2 ** 30
    assert torch.equal(row_ptr[1:], torch.cumsum(v, 0))
    keep = torch.arange(w.capacity, device="cuda")[None, :] < v[:, None]
    assert torch.equal(col, nbr[keep])

"""nl_build_close on the GPU against the oracle's close-pair detector: the
smallest pair r2 and the count of directed pairs below a threshold, over the
staged kernel, the listed (dense) path and the per-atom kernel with the
literal minimum image; its lists equal nl_build's."""
import numpy as np
import pytest
import torch

import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ctx():
    from neighbor_list_construction_b200 import nl
    c = nl.Context(200_000, 320)
    yield c
    c.close()


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def run(ctx, pos, box, cutoff, skin, K, close_d2):
    p = dev(pos)
    nbr, cnt, mn, nc = ctx.build_close(p, box, cutoff, skin, K, close_d2)
    st = ctx.sync_status()
    nbr2, cnt2 = ctx.build(p, box, cutoff, skin, K)
    assert ctx.sync_status() == st
    n = nbr.cpu().numpy()
    c = cnt.cpu().numpy()
    np.testing.assert_array_equal(c, cnt2.cpu().numpy())
    np.testing.assert_array_equal(gu.canonical(n), gu.canonical(nbr2.cpu().numpy()))
    return float(mn.item()), int(nc.item()), n, c, st


def check(ctx, oracle, pos, box, cutoff, skin, K, thresholds):
    for t in thresholds:
        mn, nc, n, c, st = run(ctx, pos, box, cutoff, skin, K, t)
        omn, onc = oracle.close_pairs(pos, box, cutoff, skin, t)
        assert mn == np.float32(omn), (t, mn, omn)
        assert nc == onc, (t, nc, onc)


@pytest.mark.parametrize("name", ["uniform4k", "saltwater_n20"])
def test_close_pairs_workloads(ctx, oracle, name):
    w = gu.workload(name)
    check(ctx, oracle, w.pos, w.box, w.cutoff, w.skin, w.capacity, [0.0, 1.0, 4.0, 9.0])


@pytest.mark.parametrize("box", [[7.6, 7.6, 7.6], [13.0, 10.1, 7.6], [12.6, 20.0, 31.0]])
def test_close_pairs_small_boxes(ctx, oracle, box):
    rng = np.random.default_rng(9)
    box = np.array(box, np.float32)
    n = int(0.1 * np.prod(box)) + 7
    pos = np.zeros((n, 4), np.float32)
    pos[:, :3] = rng.random((n, 3)) * box
    check(ctx, oracle, pos, box, 2.0, 0.5, 64, [0.5, 2.0])


def test_close_pairs_planted_and_dense(ctx, oracle):
    """A sparse box with planted close pairs (one across the periodic face)
    next to a dense slab whose tiles take the listed path."""
    rng = np.random.default_rng(5)
    box = np.array([25.0, 25.0, 25.0], np.float32)
    sparse = rng.random((1600, 3)) * box
    dense = rng.random((20000, 3)) * np.array([5.5, 25.0, 25.0])
    pos = np.zeros((21604, 4), np.float32)
    pos[:21600, :3] = np.concatenate([sparse, dense])
    pos[21600:, :3] = [[15.0, 12.0, 12.0], [15.0625, 12.0, 12.0],
                       [24.9375, 3.0, 3.0], [0.0, 3.0, 3.0]]
    check(ctx, oracle, pos, box, 2.0, 0.5, 256, [0.0, 0.004, 0.01, 1.0])


def test_close_pairs_cutoff_shell(ctx, oracle):
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
    check(ctx, oracle, pos, box, cutoff, skin, 256, [np.float32(rl * rl), 20.0])


def test_close_pairs_errors(ctx):
    from neighbor_list_construction_b200 import nl
    p = dev(np.zeros((10, 4), np.float32) + 1.0)
    nbr = torch.empty(10, 8, dtype=torch.int32, device="cuda")
    cnt = torch.empty(10, dtype=torch.int32, device="cuda")
    mn = torch.empty(1, dtype=torch.float32, device="cuda")
    nc = torch.empty(1, dtype=torch.int64, device="cuda")
    box = [10.0, 10.0, 10.0]
    with pytest.raises(nl.NLError):
        nl.nl_build_close(ctx.handle, p, box, 2.0, 0.5, 8, nbr, cnt, -1.0, mn, nc)
    with pytest.raises(nl.NLError):
        nl.nl_build_close(ctx.handle, p, box, 2.0, 0.5, 8, nbr, cnt, float("nan"), mn, nc)
    with pytest.raises(nl.NLError):
        nl.nl_build_close(ctx.handle, p, box, 2.0, 0.5, 8, nbr, cnt, 1.0, None, nc)

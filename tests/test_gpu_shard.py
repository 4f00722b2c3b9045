"""The sharded build on one GPU (all shards in one process, collectives
routed in memory): the rows of every shard's own atoms, as global ids, are
the oracle's rows of the whole system.  The halo moves in fixed blocks and
its size stays on the device; a block too small is reported as
NL_ERR_HALO."""
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
def shard():
    from neighbor_list_construction_b200 import shard as _shard
    return _shard


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def run_sharded(ctx, shard, pos, box, cutoff, skin, K, owner, block=None):
    """owner[k] = shard of atom k (global id k); returns rows by global id,
    the halo sizes and the halo block used."""
    p = shard.with_ids(dev(pos), 0)
    nranks = int(owner.max()) + 1
    ids = [np.nonzero(owner == r)[0] for r in range(nranks)]
    shards = [p[torch.from_numpy(i).cuda()] for i in ids]
    res = shard.build_sharded_local(ctx, shards, box, cutoff, skin, K, block)
    n = pos.shape[0]
    nbr = np.full((n, K), -1, np.int32)
    cnt = np.zeros(n, np.int32)
    halos = []
    for i, (nb, c, h, blk) in zip(ids, res):
        nbr[i] = nb.cpu().numpy()
        cnt[i] = c.cpu().numpy()
        halos.append(int(h.item()))
    assert len({r[3] for r in res}) == 1          # every rank agreed on one block
    return nbr, cnt, halos, res[0][3]


@pytest.mark.parametrize("name,nranks", [("uniform4k", 1), ("uniform4k", 3), ("lattice60k", 2),
                                         ("lattice60k", 8), ("saltwater_n20", 4),
                                         ("saltwater_n20", 7)])
def test_equal_count_shards_match_the_oracle(ctx, shard, oracle, name, nranks):
    w = gu.workload(name)
    ps = gu.oracle_sorted(name)                 # global id = place on the curve
    owner = np.zeros(w.n, np.int64)
    for r, (s, e) in enumerate(shard.shard_bounds(w.n, nranks)):
        owner[s:e] = r
    nbr, cnt, halos, blk = run_sharded(ctx, shard, ps, w.box, w.cutoff, w.skin, w.capacity,
                                       owner)
    st = ctx.sync_status()
    o_nbr, o_cnt, o_ov = oracle.build(ps, w.box, w.cutoff, w.skin, w.capacity)
    assert st == (1 if o_ov else 0)
    gu.assert_rows_match(nbr, cnt, o_nbr, o_cnt)
    sizes = [e - s for s, e in shard.shard_bounds(w.n, nranks)]
    for h, m in zip(halos, sizes):
        assert h <= w.n - m                     # never more than all other atoms
        assert (h > 0) == (nranks > 1)
    # a second build with the agreed block reads nothing on the host
    nbr2, cnt2, halos2, blk2 = run_sharded(ctx, shard, ps, w.box, w.cutoff, w.skin, w.capacity,
                                           owner, blk)
    assert blk2 == blk and halos2 == halos and ctx.sync_status() == st
    gu.assert_rows_match(nbr2, cnt2, o_nbr, o_cnt)


def test_scattered_shards_match_the_oracle(ctx, shard, oracle):
    """Owners drawn at random: every shard's halo is nearly everything."""
    w = gu.workload("lattice60k")
    owner = np.random.default_rng(5).integers(0, 5, w.n)
    nbr, cnt, halos, _ = run_sharded(ctx, shard, w.pos, w.box, w.cutoff, w.skin, w.capacity,
                                     owner)
    assert ctx.sync_status() == 0
    o_nbr, o_cnt, _ = oracle.build(w.pos, w.box, w.cutoff, w.skin, w.capacity)
    gu.assert_rows_match(nbr, cnt, o_nbr, o_cnt)
    assert min(halos) > 0.5 * w.n


def test_an_empty_shard(ctx, shard, oracle):
    w = gu.workload("uniform4k")
    owner = np.zeros(w.n, np.int64)
    owner[w.n // 2:] = 2                        # shard 1 owns nothing
    nbr, cnt, halos, _ = run_sharded(ctx, shard, w.pos, w.box, w.cutoff, w.skin, w.capacity,
                                     owner)
    o_nbr, o_cnt, _ = oracle.build(w.pos, w.box, w.cutoff, w.skin, w.capacity)
    gu.assert_rows_match(nbr, cnt, o_nbr, o_cnt)
    assert ctx.sync_status() == 0


def test_a_block_too_small_is_reported(ctx, shard, oracle):
    """Halo blocks smaller than the counts drop atoms: the status says
    NL_ERR_HALO (read on the host, no fault), and a build with the block the
    drivers agree on is complete again."""
    from neighbor_list_construction_b200 import nl
    w = gu.workload("lattice60k")
    ps = gu.oracle_sorted("lattice60k")
    owner = np.zeros(w.n, np.int64)
    for r, (s, e) in enumerate(shard.shard_bounds(w.n, 4)):
        owner[s:e] = r
    run_sharded(ctx, shard, ps, w.box, w.cutoff, w.skin, w.capacity, owner, 64)
    with pytest.raises(nl.NLError) as e:
        ctx.sync_status()
    assert e.value.status == nl.NL_ERR_HALO
    nbr, cnt, _, blk = run_sharded(ctx, shard, ps, w.box, w.cutoff, w.skin, w.capacity, owner)
    assert blk > 64 and ctx.sync_status() == 0
    o_nbr, o_cnt, _ = oracle.build(ps, w.box, w.cutoff, w.skin, w.capacity)
    gu.assert_rows_match(nbr, cnt, o_nbr, o_cnt)


def test_full_size_eight_shards(ctx, shard, oracle):
    """saltwater10m cut into 8 curve shards: every row of every shard, as
    global ids, against the oracle's rows of the whole system."""
    w = gu.workload("saltwater10m")
    ps = gu.oracle_sorted("saltwater10m")
    p = shard.with_ids(dev(ps), 0)
    bounds = shard.shard_bounds(w.n, 8)
    res = shard.build_sharded_local(ctx, [p[s:e] for s, e in bounds], w.box, w.cutoff, w.skin,
                                    w.capacity)
    assert ctx.sync_status() == 0
    for (s, e), (nb, c, h, _) in zip(bounds, res):
        gu.assert_all_rows_match(oracle, nb, c, ps, w.box, w.cutoff, w.skin, w.capacity,
                                 row_offset=s)
        assert 0 < int(h.item()) < (e - s)


@pytest.mark.parametrize("name", ["uniform4k", "saltwater_n20"])
def test_build_rows_prefix(ctx, oracle, name):
    """nl_build_rows: the rows of the first n_rows atoms are nl_build's rows
    (the oracle's) whatever n_rows is; out-of-range n_rows is an error."""
    from neighbor_list_construction_b200 import nl
    w = gu.workload(name)
    p = dev(w.pos)
    o_nbr, o_cnt, o_ov = oracle.build(w.pos, w.box, w.cutoff, w.skin, w.capacity)
    for n_rows in (0, 1, 777, w.n // 2, w.n):
        nbr, cnt = ctx.build_rows(p, n_rows, w.box, w.cutoff, w.skin, w.capacity)
        assert ctx.sync_status() == (1 if o_ov and o_cnt[:n_rows].max(initial=0) > w.capacity
                                     else 0)
        assert nbr.shape == (n_rows, w.capacity)
        gu.assert_rows_match(nbr.cpu().numpy(), cnt.cpu().numpy(), o_nbr[:n_rows],
                             o_cnt[:n_rows])
    with pytest.raises(nl.NLError):
        ctx.build_rows(p, w.n + 1, w.box, w.cutoff, w.skin, w.capacity)
    nb = torch.empty(1, w.capacity, dtype=torch.int32, device="cuda")
    c1 = torch.empty(1, dtype=torch.int32, device="cuda")
    with pytest.raises(nl.NLError):
        nl.nl_build_rows(ctx.handle, p, -1, w.box, w.cutoff, w.skin, w.capacity, nb, c1)
    assert ctx.sync_status() == 0


def test_dist_driver_over_nccl_one_rank(ctx, shard, oracle):
    """build_sharded through DistExchange on a one-rank NCCL group: the same
    collective calls the multi-GPU run makes, on CUDA tensors."""
    import os
    import socket
    import torch.distributed as dist
    if dist.is_initialized():
        pytest.skip("a process group already exists")
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("nccl", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = gu.workload("lattice60k")
        ps = gu.oracle_sorted("lattice60k")
        p = shard.with_ids(dev(ps), 0)
        nbr, cnt, halo, blk = shard.build_sharded(ctx, p, w.box, w.cutoff, w.skin, w.capacity,
                                                  shard.DistExchange())
        assert int(halo.item()) == 0 and blk >= 64
        assert ctx.sync_status() == 0
        o_nbr, o_cnt, _ = oracle.build(ps, w.box, w.cutoff, w.skin, w.capacity)
        gu.assert_rows_match(nbr.cpu().numpy(), cnt.cpu().numpy(), o_nbr, o_cnt)
    finally:
        dist.destroy_process_group()

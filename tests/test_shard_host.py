"""Host side of the sharded build, on CPU: the equal-count cut, the id lane,
and the collectives -- DistExchange over gloo with two and three ranks
must answer every request exactly as route_local (the single-process
routing that the one-GPU tests use) does."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from neighbor_list_construction_b200 import shard


def test_shard_bounds_equal_count():
    for n, k in [(0, 1), (1, 3), (10, 3), (10_291_605, 8), (7, 7), (100, 1)]:
        b = shard.shard_bounds(n, k)
        assert len(b) == k and b[0][0] == 0 and b[-1][1] == n
        sizes = [e - s for s, e in b]
        assert max(sizes) - min(sizes) <= 1 and sum(sizes) == n
        assert all(b[i][1] == b[i + 1][0] for i in range(k - 1))
        assert sizes == sorted(sizes, reverse=True)
    with pytest.raises(ValueError):
        shard.shard_bounds(5, 0)


def test_with_ids_puts_id_bits_in_the_fourth_float():
    p = torch.rand(5, 4)
    q = shard.with_ids(p, 1000)
    assert torch.equal(q[:, :3], p[:, :3])
    assert q[:, 3].view(torch.int32).tolist() == [1000, 1001, 1002, 1003, 1004]


BLOCK = 6


def fake_requests(rank, nranks):
    """The four collectives of one rank, with rank-dependent payloads: the
    occupancy marks, the per-destination counts, the local maximum count and
    the fixed blocks of atoms (BLOCK per destination)."""
    g = torch.Generator().manual_seed(rank)
    occ = (torch.randint(0, 2, (50,), generator=g, dtype=torch.int32) << rank).to(torch.int32)
    counts = torch.tensor([(rank * 3 + q * 5) % 7 if q != rank else 0 for q in range(nranks)],
                          dtype=torch.int32)
    top = counts.max().reshape(1)
    send = torch.rand(nranks * BLOCK, 4, generator=g)
    return occ, counts, top, send


def _gloo_rank(rank, nranks, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=nranks)
    try:
        ex = shard.DistExchange()
        occ, counts, top, send = fake_requests(rank, nranks)

        def steps():
            a = yield ("sum", occ)
            b = yield ("counts", counts)
            m = yield ("max", top)
            c = yield ("blocks", send)
            return a, b, m, c

        a, b, m, c = ex.run(steps())
        torch.save({"sum": a, "counts": b, "max": m, "blocks": c},
                   os.path.join(out_dir, f"r{rank}.pt"))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("nranks", [2, 3])
def test_dist_exchange_matches_local_routing(tmp_path, nranks):
    mp.start_processes(_gloo_rank, args=(nranks, _free_port(), str(tmp_path)), nprocs=nranks,
                       start_method="spawn")
    reqs = [fake_requests(r, nranks) for r in range(nranks)]
    sums = shard.route_local([("sum", r[0]) for r in reqs])
    cnts = shard.route_local([("counts", r[1]) for r in reqs])
    tops = shard.route_local([("max", r[2]) for r in reqs])
    blocks = shard.route_local([("blocks", r[3]) for r in reqs])
    for k in range(nranks):
        got = torch.load(os.path.join(tmp_path, f"r{k}.pt"))
        assert torch.equal(got["sum"], sums[k])
        assert torch.equal(got["counts"], cnts[k])
        assert torch.equal(got["max"], tops[k])
        assert torch.equal(got["blocks"], blocks[k])
        # block q of rank p's send is block p of rank q's receive
        for p in range(nranks):
            assert torch.equal(got["blocks"][p * BLOCK:(p + 1) * BLOCK],
                               reqs[p][3][k * BLOCK:(k + 1) * BLOCK])
        assert got["max"].item() == max(int(r[1].max()) for r in reqs)
        # the sum of distinct rank bits is their bitwise or
        ors = np.bitwise_or.reduce(np.stack([r[0].numpy() for r in reqs]), axis=0)
        assert np.array_equal(got["sum"].numpy(), ors)


def test_block_for_leaves_room():
    for top in (0, 1, 63, 64, 1000, 301_000):
        b = shard.block_for(top)
        assert b % 64 == 0 and b >= top + top // 4 and b >= 64

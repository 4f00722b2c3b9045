"""Equal-count shards along the curve, with a halo exchange between them.

Tessera abstract: the atoms are sorted along a space-filling curve and cut
into equal-count shards, one per GPU; a GPU builds the rows of its own atoms
from its shard plus the atoms of other shards within the search radius (its
halo).  One rank's build, in the order the steps run:

1. ``nl_halo_mark``: the coarse cells (wider than rl) its atoms occupy;
2. a sum over ranks of those marks (all-reduce): per cell, the ranks there;
3. ``nl_halo_needed``, ``nl_halo_count``: per destination rank, how many of
   its atoms lie next to a cell of that rank; the counts go round
   (all-to-all), so each rank knows how many atoms it will receive;
4. ``nl_halo_fill_blocks`` and an all-to-all of equal splits: every rank
   sends a fixed block of ``halo_block`` atoms to every other rank;
5. ``nl_halo_pack``: the received blocks are appended to the own atoms on
   the device, and the atom count stays in device memory;
6. ``nl_build_rows_dev`` over [own atoms; halo], rows for the own atoms only;
7. ``nl_map_ids``: row entries become global ids (carried in the fourth
   float of each position).

No step reads a count on the host, so a build enqueues without waiting for
the GPU.  The block size is agreed once: the first build of a driver (when
no block is given) takes the largest count over all ranks (an all-reduce of
maxima, one host read) with a quarter to spare, and later builds reuse it.
A count above the block drops atoms and makes ``sync_status`` report
``NL_ERR_HALO``; the caller then rebuilds with a larger block.

Every step that touches atoms runs in libnl's kernels; this module only
moves buffers between ranks.  The steps are written once, as a generator
that yields at each collective, and are driven either by
:class:`DistExchange` (one process per GPU over ``torch.distributed``: NCCL
on GPUs, gloo on CPU in tests) or by :func:`build_sharded_local`, which runs
all shards in one process on one GPU and routes their buffers itself, for
testing and measuring the sharded path where only one GPU is available.
"""
from __future__ import annotations

import torch

from . import nl


def shard_bounds(n: int, nranks: int) -> list[tuple[int, int]]:
    """Equal-count cut of n curve-ordered atoms: rank r gets [start, end),
    the first n % nranks ranks one atom more."""
    if nranks < 1 or n < 0:
        raise ValueError("need nranks >= 1 and n >= 0")
    q, r = divmod(n, nranks)
    out, s = [], 0
    for k in range(nranks):
        e = s + q + (1 if k < r else 0)
        out.append((s, e))
        s = e
    return out


def with_ids(pos: torch.Tensor, first_id: int) -> torch.Tensor:
    """A copy of pos (n x 4 float32) whose fourth float holds the int32 bits
    of the global ids first_id .. first_id + n - 1."""
    out = pos.clone()
    ids = torch.arange(first_id, first_id + pos.shape[0], dtype=torch.int32, device=pos.device)
    out[:, 3] = ids.view(torch.float32)
    return out


def block_for(max_count: int) -> int:
    """Halo block for a largest per-destination count: a quarter to spare,
    rounded up to 64 atoms."""
    want = int(max_count) + int(max_count) // 4 + 64
    return (want + 63) // 64 * 64


def _steps(ctx, pos_own, box, cutoff, skin, capacity, rank, nranks, block=None):
    """One rank's halo build; yields ("sum", occ), ("counts", counts),
    ("max", local max) when no block is given, and ("blocks", send) for the
    driver to answer with the combined result, and returns (nbr, counts,
    halo atoms as a device int64 tensor, block)."""
    dev = pos_own.device
    n_own = pos_own.shape[0]
    dims = nl.nl_halo_grid(box, cutoff, skin)
    nc = dims[0] * dims[1] * dims[2]
    occ = torch.empty(nc, dtype=torch.int32, device=dev)
    nl.nl_halo_mark(ctx.handle, pos_own, box, dims, rank, occ)
    occ_all = yield ("sum", occ)
    need = torch.empty(nc, dtype=torch.int32, device=dev)
    nl.nl_halo_needed(ctx.handle, box, dims, occ_all, need)
    counts = torch.empty(nranks, dtype=torch.int32, device=dev)
    nl.nl_halo_count(ctx.handle, pos_own, box, dims, need, rank, nranks, counts)
    recv_counts = yield ("counts", counts)
    if block is None:   # agree on a block: the one host read, first build only
        top = yield ("max", counts.max().reshape(1))
        block = block_for(int(top.item()))
    send = torch.empty(nranks * block, 4, dtype=torch.float32, device=dev)
    cursor = torch.empty(nranks, dtype=torch.int32, device=dev)
    nl.nl_halo_fill_blocks(ctx.handle, pos_own, box, dims, need, rank, nranks, block, counts,
                           cursor, send)
    recv = yield ("blocks", send)
    n_max = n_own + (nranks - 1) * block
    pos_all = torch.empty(n_max, 4, dtype=torch.float32, device=dev)
    pos_all[:n_own] = pos_own
    n_all = torch.empty(1, dtype=torch.int64, device=dev)
    nl.nl_halo_pack(ctx.handle, nranks, block, recv_counts, recv, n_own, pos_all, n_all)
    nbr = torch.empty(n_own, capacity, dtype=torch.int32, device=dev)
    cnt = torch.empty(n_own, dtype=torch.int32, device=dev)
    nl.nl_build_rows_dev(ctx.handle, pos_all, n_all, n_own, box, cutoff, skin, capacity,
                         nbr if n_own else None, cnt if n_own else None)
    if n_own:
        nl.nl_map_ids(ctx.handle, nbr, pos_all, cnt)
    return nbr, cnt, n_all - n_own, block


class DistExchange:
    """The collectives of the halo build over a torch.distributed group."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.size = dist.get_world_size(group)

    def sum(self, t: torch.Tensor) -> torch.Tensor:
        out = t.clone()
        self.dist.all_reduce(out, op=self.dist.ReduceOp.SUM, group=self.group)
        return out

    def counts(self, c: torch.Tensor) -> torch.Tensor:
        out = torch.empty_like(c)
        self.dist.all_to_all_single(out, c.contiguous(), group=self.group)
        return out

    def max(self, t: torch.Tensor) -> torch.Tensor:
        out = t.clone()
        self.dist.all_reduce(out, op=self.dist.ReduceOp.MAX, group=self.group)
        return out

    def blocks(self, send: torch.Tensor) -> torch.Tensor:
        """All-to-all of equal splits: block q of send goes to rank q."""
        out = torch.empty_like(send)
        self.dist.all_to_all_single(out, send.contiguous(), group=self.group)
        return out

    def run(self, gen):
        req = next(gen)
        while True:
            if req[0] == "sum":
                ans = self.sum(req[1])
            elif req[0] == "counts":
                ans = self.counts(req[1])
            elif req[0] == "max":
                ans = self.max(req[1])
            else:
                ans = self.blocks(req[1])
            try:
                req = gen.send(ans)
            except StopIteration as fin:
                return fin.value


def build_sharded(ctx, pos_own, box, cutoff, skin, capacity, comm: DistExchange,
                  halo_block: int | None = None):
    """This rank's rows over its own atoms (pos_own, global ids in the fourth
    float): (nbr [n_own, capacity] of global ids, counts [n_own], halo atoms
    (device int64 [1]), the halo block used).  Pass the returned block back
    to later builds: they then need no host read."""
    return comm.run(_steps(ctx, pos_own, box, cutoff, skin, capacity, comm.rank, comm.size,
                           halo_block))


def route_local(reqs):
    """Answers one collective for all ranks of one process: reqs[r] is rank
    r's request; returns each rank's answer, as DistExchange would."""
    nranks = len(reqs)
    kind = reqs[0][0]
    if any(r[0] != kind for r in reqs):
        raise RuntimeError("ranks disagree on the collective")
    if kind == "sum":
        total = reqs[0][1].clone()
        for r in reqs[1:]:
            total += r[1]
        return [total for _ in reqs]
    if kind == "counts":
        mat = torch.stack([r[1] for r in reqs])      # [source, destination]
        return [mat[:, q].contiguous() for q in range(nranks)]
    if kind == "max":
        top = reqs[0][1].clone()
        for r in reqs[1:]:
            top = torch.maximum(top, r[1])
        return [top for _ in reqs]
    # blocks: equal splits, block q of rank p's send goes to rank q
    pieces = [r[1].chunk(nranks) for r in reqs]
    return [torch.cat([pieces[p][q] for p in range(nranks)]) for q in range(nranks)]


def build_sharded_local(ctx, shards, box, cutoff, skin, capacity, halo_block: int | None = None):
    """All shards' halo builds in one process (one context, one GPU): the
    same steps as build_sharded, with the collectives answered by
    route_local.  Returns one (nbr, counts, halo atoms, block) per shard."""
    nranks = len(shards)
    gens = [_steps(ctx, p, box, cutoff, skin, capacity, r, nranks, halo_block)
            for r, p in enumerate(shards)]
    reqs = [next(g) for g in gens]
    while True:
        answers = route_local(reqs)
        nxt, done = [], []
        for g, a in zip(gens, answers):
            try:
                nxt.append(g.send(a))
            except StopIteration as fin:
                done.append(fin.value)
        if done:
            if len(done) != nranks:
                raise RuntimeError("ranks finished at different steps")
            return done
        reqs = nxt

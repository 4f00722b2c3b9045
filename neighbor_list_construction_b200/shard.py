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
4. ``nl_halo_fill`` and an all-to-all of those atoms: the halo;
5. ``nl_build_rows`` over [own atoms; halo], rows for the own atoms only;
6. ``nl_map_ids``: row entries become global ids (carried in the fourth
   float of each position).

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


def _steps(ctx, pos_own, box, cutoff, skin, capacity, rank, nranks):
    """One rank's halo build; yields ("sum", occ), ("counts", counts) and
    ("atoms", send, send_splits, recv_splits) for the driver to answer with
    the combined result, and returns (nbr, counts, n_halo)."""
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
    send_splits = [int(v) for v in counts.tolist()]
    recv_splits = [int(v) for v in recv_counts.tolist()]
    offsets = torch.zeros(nranks, dtype=torch.int32, device=dev)
    if nranks > 1:
        offsets[1:] = torch.cumsum(counts, 0, dtype=torch.int32)[:-1]
    send = torch.empty(max(sum(send_splits), 1), 4, dtype=torch.float32, device=dev)
    cursor = torch.empty(nranks, dtype=torch.int32, device=dev)
    nl.nl_halo_fill(ctx.handle, pos_own, box, dims, need, rank, nranks, offsets, counts, cursor,
                    send)
    send = send[: sum(send_splits)]
    halo = yield ("atoms", send, send_splits, recv_splits)
    pos_all = torch.cat([pos_own, halo]) if halo.shape[0] else pos_own
    nbr, cnt = ctx.build_rows(pos_all, n_own, box, cutoff, skin, capacity)
    if n_own:
        nl.nl_map_ids(ctx.handle, nbr, pos_all, cnt)
    return nbr, cnt, int(halo.shape[0])


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

    def atoms(self, send: torch.Tensor, send_splits, recv_splits) -> torch.Tensor:
        out = torch.empty(sum(recv_splits), 4, dtype=send.dtype, device=send.device)
        self.dist.all_to_all_single(out, send.contiguous(), output_split_sizes=list(recv_splits),
                                    input_split_sizes=list(send_splits), group=self.group)
        return out

    def run(self, gen):
        req = next(gen)
        while True:
            if req[0] == "sum":
                ans = self.sum(req[1])
            elif req[0] == "counts":
                ans = self.counts(req[1])
            else:
                ans = self.atoms(req[1], req[2], req[3])
            try:
                req = gen.send(ans)
            except StopIteration as fin:
                return fin.value


def build_sharded(ctx, pos_own, box, cutoff, skin, capacity, comm: DistExchange):
    """This rank's rows over its own atoms (pos_own, global ids in the fourth
    float): (nbr [n_own, capacity] of global ids, counts [n_own], halo size)."""
    return comm.run(_steps(ctx, pos_own, box, cutoff, skin, capacity, comm.rank, comm.size))


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
    pieces = []
    for r in reqs:
        send, splits = r[1], r[2]
        offs = [0]
        for v in splits:
            offs.append(offs[-1] + int(v))
        pieces.append([send[offs[q]:offs[q + 1]] for q in range(nranks)])
    return [torch.cat([pieces[p][q] for p in range(nranks)]) for q in range(nranks)]


def build_sharded_local(ctx, shards, box, cutoff, skin, capacity):
    """All shards' halo builds in one process (one context, one GPU): the
    same steps as build_sharded, with the collectives answered by
    route_local.  Returns one (nbr, counts, halo size) per shard."""
    nranks = len(shards)
    gens = [_steps(ctx, p, box, cutoff, skin, capacity, r, nranks) for r, p in enumerate(shards)]
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

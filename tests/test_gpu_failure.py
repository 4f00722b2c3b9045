"""Failure detection without a fault: a bounded device wait that runs out (it
polls a word that nothing writes) reports NL_ERR_TIMEOUT through the
context's status word; the report clears on reading, bad limits are refused
on the host, and the context stays usable: a build after it equals the
oracle's."""
import numpy as np
import pytest
import torch

import gpu_util as gu

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_stays_usable(oracle):
    from neighbor_list_construction_b200 import nl
    w = gu.workload("uniform4k")
    ctx = nl.Context(w.n, w.capacity)
    try:
        assert ctx.sync_status() == nl.NL_OK
        assert nl.nl_wait_selftest(ctx.handle, 1000) == nl.NL_OK   # enqueued
        with pytest.raises(nl.NLError) as e:
            ctx.sync_status()
        assert e.value.status == nl.NL_ERR_TIMEOUT
        assert ctx.sync_status() == nl.NL_OK                       # cleared by the read
        for bad in (0, -5, (1 << 22) + 1):
            with pytest.raises(nl.NLError) as e:
                nl.nl_wait_selftest(ctx.handle, bad)
            assert e.value.status == nl.NL_ERR_ARG
        assert ctx.sync_status() == nl.NL_OK
        pos = torch.from_numpy(np.ascontiguousarray(w.pos)).cuda()
        nbr, cnt = ctx.build(pos, w.box, w.cutoff, w.skin, w.capacity)
        assert ctx.sync_status() == nl.NL_OK
        o_nbr, o_cnt, o_ov = oracle.build(w.pos, w.box, w.cutoff, w.skin, w.capacity)
        assert not o_ov
        gu.assert_rows_match(nbr.cpu().numpy(), cnt.cpu().numpy(), o_nbr, o_cnt)
    finally:
        ctx.close()


def test_after_a_timeout_later_kernels_leave_their_outputs_alone(oracle):
    """Once a bounded wait has given up, the kernels that consume what a
    look-back pass produced (gather, scatter, in-cell sort, pair search)
    return at entry until the status is read: a sort and a build issued before
    the read leave their outputs as they were, so a partial prefix can never
    turn into an index or a copy size.  After the read, both equal the
    oracle's.  Only the self-test wait runs out; no real scan is made to."""
    from neighbor_list_construction_b200 import nl
    w = gu.workload("lattice60k")
    ctx = nl.Context(w.n, w.capacity)
    try:
        pos = torch.from_numpy(np.ascontiguousarray(w.pos)).cuda()
        assert nl.nl_wait_selftest(ctx.handle, 1000) == nl.NL_OK
        perm = torch.full((w.n,), -7, dtype=torch.int32, device="cuda")
        ps = torch.full((w.n, 4), -7.0, dtype=torch.float32, device="cuda")
        nl.nl_sort_hilbert(ctx.handle, pos, w.box, perm, ps)
        nbr = torch.full((w.n, w.capacity), -7, dtype=torch.int32, device="cuda")
        cnt = torch.full((w.n,), -7, dtype=torch.int32, device="cuda")
        ctx.build(pos, w.box, w.cutoff, w.skin, w.capacity, nbr=nbr, counts=cnt)
        torch.cuda.synchronize()
        assert bool((ps == -7.0).all()) and bool((nbr == -7).all()) and bool((cnt == -7).all())
        with pytest.raises(nl.NLError) as e:
            ctx.sync_status()
        assert e.value.status == nl.NL_ERR_TIMEOUT
        # the read cleared the status: the same calls now do their work
        nl.nl_sort_hilbert(ctx.handle, pos, w.box, perm, ps)
        ctx.build(pos, w.box, w.cutoff, w.skin, w.capacity, nbr=nbr, counts=cnt)
        assert ctx.sync_status() == nl.NL_OK
        o_perm, _ = oracle.sort(w.pos, w.box)
        np.testing.assert_array_equal(perm.cpu().numpy(), o_perm)
        np.testing.assert_array_equal(ps.cpu().numpy()[:, :3], w.pos[o_perm, :3])
        o_nbr, o_cnt, o_ov = oracle.build(w.pos, w.box, w.cutoff, w.skin, w.capacity)
        gu.assert_rows_match(nbr.cpu().numpy(), cnt.cpu().numpy(), o_nbr, o_cnt)
    finally:
        ctx.close()

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

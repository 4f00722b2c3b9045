"""nl_sort_hilbert_noalloc: the curve sort for callers that cannot allocate.

Some callers cannot call cudaMalloc (a framework that owns all device memory,
a plugin whose host forbids allocation).  The no-alloc entry point keeps its
scratch in a static device array inside libnl.so, so it needs no context.
This test calls it through the C ABI twice in a row, on two different inputs,
and checks each result against the context-based nl_sort_hilbert: the
permutation, keys and sorted positions are integers or copies, so they must
match exactly.  It also checks that sizes above the array's limit (2^20
atoms) are refused.  The file is named to be collected last.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _inputs():
    from neighbor_list_construction_b200 import workloads
    w1 = workloads.make("lattice60k")
    rng = np.random.default_rng(31)
    box2 = np.array([50.0, 61.5, 43.25], np.float32)
    p2 = np.zeros((70_001, 4), np.float32)
    p2[:, :3] = rng.uniform(-0.5, 1.5, (70_001, 3)) * box2
    return [(w1.pos, w1.box), (p2, box2)]


def test_noalloc_sort_matches_context_sort_on_two_calls():
    from neighbor_list_construction_b200 import nl
    ctx = nl.Context(100_000, 16)
    try:
        for pos_np, box in _inputs():
            pos = torch.from_numpy(pos_np).cuda()
            n = pos.shape[0]
            perm_ref, ps_ref, keys_ref = ctx.sort(pos, box, keys=True)
            assert ctx.sync_status() == nl.NL_OK
            perm = torch.full((n,), -1, dtype=torch.int32, device="cuda")
            ps = torch.zeros((n, 4), dtype=torch.float32, device="cuda")
            keys = torch.zeros(n, dtype=torch.int64, device="cuda")
            status = torch.full((1,), 99, dtype=torch.int32, device="cuda")
            nl.nl_sort_hilbert_noalloc(pos, box, perm, ps, keys, status)
            torch.cuda.synchronize()
            assert status.item() == nl.NL_OK
            assert torch.equal(perm, perm_ref)
            assert torch.equal(keys, keys_ref)
            assert torch.equal(ps, ps_ref)
    finally:
        ctx.close()


def test_noalloc_sort_rejects_sizes_above_its_limit():
    from neighbor_list_construction_b200 import nl
    n = (1 << 20) + 1
    pos = torch.zeros((n, 4), dtype=torch.float32, device="cuda")
    perm = torch.empty(n, dtype=torch.int32, device="cuda")
    ps = torch.empty((n, 4), dtype=torch.float32, device="cuda")
    with pytest.raises(nl.NLError) as e:
        nl.nl_sort_hilbert_noalloc(pos, [10.0, 10.0, 10.0], perm, ps)
    assert e.value.status == nl.NL_ERR_CAPACITY

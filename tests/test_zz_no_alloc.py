"""nl_sort_hilbert_noalloc: the curve sort for callers that cannot allocate.

Some callers cannot call cudaMalloc (a framework that owns all device memory,
a plugin whose host forbids allocation).  The no-alloc entry point keeps its
scratch in a static device array inside libnl.so, so it needs no context.
This test calls it through the C ABI several times in a row, on different
inputs, and checks each result against the context-based nl_sort_hilbert and
against the oracle: the permutation, keys and sorted positions are integers or
copies, so they must match exactly.  It also checks that sizes above the
array's limit (2^20 atoms) are refused.  The file is named to be collected last.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _inputs():
    """Two well-spread inputs, one whose 200 coincident atoms make a run of
    equal keys longer than the run finish takes (so the gated eight-pass sort
    runs on the static array), and one of exactly 2^20 atoms, the limit, where
    the look-back area's tile stride is largest."""
    from neighbor_list_construction_b200 import workloads
    w1 = workloads.make("lattice60k")
    rng = np.random.default_rng(31)
    box2 = np.array([50.0, 61.5, 43.25], np.float32)
    p2 = np.zeros((70_001, 4), np.float32)
    p2[:, :3] = rng.uniform(-0.5, 1.5, (70_001, 3)) * box2
    p3 = np.zeros((30_000, 4), np.float32)
    p3[:, :3] = rng.uniform(0.0, 1.0, (30_000, 3)) * box2
    p3[1000:1200, :3] = p3[7, :3]
    n4 = 1 << 20
    box4 = np.array([220.0, 215.5, 222.25], np.float32)
    p4 = np.zeros((n4, 4), np.float32)
    p4[:, :3] = rng.uniform(0.0, 1.0, (n4, 3)) * box4
    return [(w1.pos, w1.box), (p2, box2), (p3, box2), (p4, box4)]


def test_noalloc_sort_matches_context_sort_on_two_calls():
    """Calls in a row on different inputs, each against the context sort and
    against the oracle's (key, index) order."""
    import oracle
    from neighbor_list_construction_b200 import nl
    ctx = nl.Context(1 << 20, 16)
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
            o_perm, o_keys = oracle.sort(pos_np, box)
            np.testing.assert_array_equal(perm.cpu().numpy(), o_perm)
            np.testing.assert_array_equal(keys.cpu().numpy().view(np.uint64), o_keys)
            np.testing.assert_array_equal(ps.cpu().numpy()[:, :3], pos_np[o_perm, :3])
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

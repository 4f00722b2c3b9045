"""Helpers shared by the GPU parity tests (no GPU work at import)."""
from __future__ import annotations

import functools

import numpy as np


@functools.lru_cache(maxsize=None)
def workload(name: str, seed: int | None = None):
    from neighbor_list_construction_b200 import workloads
    return workloads.make(name, seed=seed)


@functools.lru_cache(maxsize=None)
def oracle_sorted(name: str) -> np.ndarray:
    """The workload's positions in the oracle's curve order (Hilbert), so that
    tests run the GPU build in the benchmark's order on inputs that owe
    nothing to the GPU path."""
    import oracle
    w = workload(name)
    perm, _ = oracle.sort(w.pos, w.box)
    return np.ascontiguousarray(w.pos[perm])


def canonical(nbr: np.ndarray) -> np.ndarray:
    big = np.iinfo(np.int32).max
    out = np.sort(np.where(nbr < 0, big, nbr), axis=1)
    return np.where(out == big, -1, out).astype(np.int32)


def assert_rows_match(g_nbr, g_cnt, o_nbr, o_cnt, full_sets=None):
    """GPU rows (any order) equal the oracle's ascending rows; rows whose
    count exceeds the capacity must be `capacity` distinct members of the
    atom's full neighbor set (given in full_sets[i] when present)."""
    g_nbr = np.asarray(g_nbr)
    g_cnt = np.asarray(g_cnt)
    np.testing.assert_array_equal(g_cnt, o_cnt)
    K = g_nbr.shape[1]
    ok = o_cnt <= K
    can = canonical(g_nbr)
    bad = np.nonzero(np.any(can[ok] != o_nbr[ok], axis=1))[0]
    assert bad.size == 0, f"{bad.size} rows differ, first local row {bad[:5]}"
    for r in np.nonzero(~ok)[0]:
        row = g_nbr[r]
        assert np.all(row >= 0) and np.unique(row).size == K
        if full_sets is not None:
            assert set(row.tolist()) <= full_sets[r]

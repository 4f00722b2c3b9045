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


def assert_all_rows_match(oracle, nbr_t, cnt_t, pos, box, cutoff, skin, K, chunk=1 << 21,
                          row_offset=0):
    """Every row and count of a GPU build (device tensors, any slot order)
    against the oracle, element by element, in chunks of rows.  Row r of the
    GPU tensors is atom row_offset + r of pos (a shard's rows).

    The GPU rows are put in canonical order (ascending, -1 padding last) with
    torch.sort on the device; the oracle's rows come from oracle.rows on the
    same positions.  Rows whose count passes K must hold K distinct members of
    the atom's full neighbor set.  Returns True when any row overflowed."""
    import torch
    n = nbr_t.shape[0]
    cnt = cnt_t.cpu().numpy()
    big = torch.iinfo(torch.int32).max
    overflow = False
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        which = np.arange(row_offset + s, row_offset + e, dtype=np.int64)
        o_nbr, o_cnt, o_ov = oracle.rows(pos, box, cutoff, skin, K, which)
        np.testing.assert_array_equal(cnt[s:e], o_cnt)
        g = nbr_t[s:e]
        g = torch.sort(torch.where(g < 0, big, g), dim=1).values
        g = torch.where(g == big, -1, g).cpu().numpy()
        ok = o_cnt <= K
        bad = np.nonzero(np.any(g[ok] != o_nbr[ok], axis=1))[0]
        assert bad.size == 0, f"{bad.size} rows differ, first {s + np.nonzero(ok)[0][bad[:5]]}"
        over = np.nonzero(~ok)[0]
        if over.size:
            overflow = True
            K2 = int(o_cnt[over].max())
            f_nbr, f_cnt, _ = oracle.rows(pos, box, cutoff, skin, K2, which[over])
            raw = nbr_t[s:e][torch.from_numpy(over).to(nbr_t.device)].cpu().numpy()
            for r, row in enumerate(raw):
                assert np.all(row >= 0) and np.unique(row).size == K
                assert set(row.tolist()) <= set(f_nbr[r, :f_cnt[r]].tolist())
    return overflow

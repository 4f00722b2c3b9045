"""CPU oracle for the periodic neighbor-list build -- TEST INFRASTRUCTURE ONLY.

A plain, slow restatement (``nl_oracle.c``, plain C, fp32 without fused
multiply-add; its per-atom and per-row loops may run on OpenMP threads, which
changes no result) of what the GPU hot path computes: Hilbert-curve order,
fixed-capacity padded neighbor rows, and the skin check.  Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` may import this
package; the product library never does, and shares no code with it.

Method source: "Ab Initio Accuracy Beyond the Cutoff: Distributed
Message-Passing Equivariant Attention at Tens-of-Millions-of-Atom Scale"
(Tessera), abstract -- space-filling-curve sort, conservative neighbor skin,
fixed tensor shapes between rebuilds.  Hilbert transform: J. Skilling,
"Programming the Hilbert curve", AIP Conf. Proc. 707 (2004).

Every function here is pinned by ``tests/test_oracle_*.py`` against brute
force, closed forms, exact rational arithmetic and curve invariants.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nl_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
          "-fPIC", "-shared"]


def compile_library(force: bool = False) -> str:
    """Compile the oracle with gcc if the shared library is missing or stale."""
    if (force or not os.path.exists(_LIB)
            or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)):
        tmp = _LIB + ".tmp"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        L = ctypes.CDLL(compile_library())
        f32, i32, i64, u32, u64 = (ctypes.c_float, ctypes.c_int32, ctypes.c_int64,
                                   ctypes.c_uint32, ctypes.c_uint64)
        vp = ctypes.c_void_p
        sig = {
            "oracle_wrap": (f32, [f32, f32]),
            "oracle_quantize": (u32, [f32, f32]),
            "oracle_quant_scale": (f32, [f32]),
            "oracle_hilbert_key": (u64, [u32, u32, u32, ctypes.c_int]),
            "oracle_hilbert_axes": (None, [u64, ctypes.c_int, vp]),
            "oracle_morton_key": (u64, [u32, u32, u32, ctypes.c_int]),
            "oracle_keys": (None, [i64, vp, vp, ctypes.c_int, vp]),
            "oracle_sort": (ctypes.c_int, [i64, vp, vp, ctypes.c_int, vp, vp]),
            "oracle_min_image": (f32, [f32, f32]),
            "oracle_r2": (f32, [vp, vp, vp]),
            "oracle_bruteforce": (ctypes.c_int, [i64, vp, vp, f32, f32, i32, vp, vp]),
            "oracle_rows": (ctypes.c_int, [i64, vp, vp, f32, f32, i32, i64, vp, vp, vp]),
            "oracle_build": (ctypes.c_int, [i64, vp, vp, f32, f32, i32, vp, vp]),
            "oracle_skin_check": (f32, [i64, vp, vp, vp, f32, vp]),
            "oracle_close_pairs": (ctypes.c_int, [i64, vp, vp, f32, f32, f32, vp, vp]),
            "oracle_edge_features": (None, [i64, vp, vp, ctypes.c_int32, vp, vp, vp]),
            "oracle_displacement": (f32, [u64, i64, i64, ctypes.c_int, f32]),
            "oracle_displace": (None, [i64, vp, u64, i64, f32]),
            "oracle_md_decisions": (i64, [i64, vp, vp, vp, f32, u64, f32, i64, vp]),
            "oracle_set_threads": (ctypes.c_int, [ctypes.c_int]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _pos4(pos) -> np.ndarray:
    pos = np.ascontiguousarray(pos, dtype=np.float32)
    if pos.ndim != 2 or pos.shape[1] not in (3, 4):
        raise ValueError("positions must be (n, 3) or (n, 4)")
    if pos.shape[1] == 3:
        pos = np.concatenate([pos, np.zeros((pos.shape[0], 1), np.float32)], axis=1)
    return np.ascontiguousarray(pos)


def _box(box) -> np.ndarray:
    b = np.ascontiguousarray(np.asarray(box, dtype=np.float32).reshape(3))
    return b


def set_threads(n: int) -> int:
    """Threads the oracle's per-atom and per-row loops may use (1 = plain
    single-threaded).  Returns the previous setting."""
    return int(lib().oracle_set_threads(int(n)))


# ----------------------------------------------------------------- scalars
def wrap(x: float, L: float) -> float:
    return lib().oracle_wrap(np.float32(x), np.float32(L))


def quant_scale(L: float) -> float:
    return lib().oracle_quant_scale(np.float32(L))


def quantize(w: float, S: float) -> int:
    return lib().oracle_quantize(np.float32(w), np.float32(S))


def hilbert_key(qx: int, qy: int, qz: int, bits: int = 21) -> int:
    return lib().oracle_hilbert_key(qx, qy, qz, bits)


def hilbert_axes(key: int, bits: int = 21) -> tuple[int, int, int]:
    out = np.zeros(3, np.uint32)
    lib().oracle_hilbert_axes(key, bits, _p(out))
    return int(out[0]), int(out[1]), int(out[2])


def morton_key(qx: int, qy: int, qz: int, bits: int = 21) -> int:
    return lib().oracle_morton_key(qx, qy, qz, bits)


def min_image(d: float, L: float) -> float:
    return lib().oracle_min_image(np.float32(d), np.float32(L))


def r2(a, b, box) -> float:
    a = np.ascontiguousarray(np.asarray(a, np.float32).reshape(3))
    b = np.ascontiguousarray(np.asarray(b, np.float32).reshape(3))
    bx = _box(box)
    return lib().oracle_r2(_p(a), _p(b), _p(bx))


def displacement(seed: int, step: int, atom: int, axis: int, sigma: float) -> float:
    return lib().oracle_displacement(seed, step, atom, axis, np.float32(sigma))


# ------------------------------------------------------------------ arrays
def keys(pos, box, curve: str = "hilbert") -> np.ndarray:
    p = _pos4(pos)
    bx = _box(box)
    out = np.zeros(p.shape[0], np.uint64)
    lib().oracle_keys(p.shape[0], _p(p), _p(bx), 1 if curve == "morton" else 0, _p(out))
    return out


def sort(pos, box, curve: str = "hilbert"):
    """Returns (perm int32[n], sorted keys uint64[n])."""
    p = _pos4(pos)
    bx = _box(box)
    n = p.shape[0]
    perm = np.zeros(n, np.int32)
    ks = np.zeros(n, np.uint64)
    rc = lib().oracle_sort(n, _p(p), _p(bx), 1 if curve == "morton" else 0, _p(perm), _p(ks))
    if rc != 0:
        raise MemoryError("oracle_sort failed")
    return perm, ks


def build(pos, box, cutoff: float, skin: float, capacity: int):
    """Full neighbor list: (nbr int32[n, K], counts int32[n], overflow bool)."""
    p = _pos4(pos)
    bx = _box(box)
    n = p.shape[0]
    nbr = np.zeros((n, capacity), np.int32)
    cnt = np.zeros(n, np.int32)
    rc = lib().oracle_build(n, _p(p), _p(bx), np.float32(cutoff), np.float32(skin),
                            capacity, _p(nbr), _p(cnt))
    if rc < 0:
        raise MemoryError("oracle_build failed")
    return nbr, cnt, bool(rc)


def rows(pos, box, cutoff: float, skin: float, capacity: int, which):
    """Rows for the atoms in `which` only: (nbr [len, K], counts [len], overflow)."""
    p = _pos4(pos)
    bx = _box(box)
    w = np.ascontiguousarray(np.asarray(which, np.int64))
    nbr = np.zeros((w.shape[0], capacity), np.int32)
    cnt = np.zeros(w.shape[0], np.int32)
    rc = lib().oracle_rows(p.shape[0], _p(p), _p(bx), np.float32(cutoff), np.float32(skin),
                           capacity, w.shape[0], _p(w), _p(nbr), _p(cnt))
    if rc < 0:
        raise MemoryError("oracle_rows failed")
    return nbr, cnt, bool(rc)


def bruteforce(pos, box, cutoff: float, skin: float, capacity: int):
    p = _pos4(pos)
    bx = _box(box)
    n = p.shape[0]
    nbr = np.zeros((n, capacity), np.int32)
    cnt = np.zeros(n, np.int32)
    rc = lib().oracle_bruteforce(n, _p(p), _p(bx), np.float32(cutoff), np.float32(skin),
                                 capacity, _p(nbr), _p(cnt))
    if rc < 0:
        raise MemoryError("oracle_bruteforce failed")
    return nbr, cnt, bool(rc)


def close_pairs(pos, box, cutoff: float, skin: float, close_d2: float):
    """Smallest r2 over all directed neighbor pairs (inf if none) and the
    number of directed neighbor pairs with r2 < close_d2."""
    p = _pos4(pos)
    bx = _box(box)
    mn = np.zeros(1, np.float32)
    nc = np.zeros(1, np.int64)
    rc = lib().oracle_close_pairs(p.shape[0], _p(p), _p(bx), np.float32(cutoff),
                                  np.float32(skin), np.float32(close_d2), _p(mn), _p(nc))
    if rc < 0:
        raise MemoryError("oracle_close_pairs failed")
    return float(mn[0]), int(nc[0])


def edge_features(pos, box, nbr, counts) -> np.ndarray:
    """Per-slot (dx, dy, dz, r) of padded rows: n x K x 4 float32, the
    minimum-image displacement from atom i to nbr[i][s] and its length for
    s < min(counts[i], K), zeros elsewhere."""
    p = _pos4(pos)
    bx = _box(box)
    nb = np.ascontiguousarray(nbr, dtype=np.int32)
    ct = np.ascontiguousarray(counts, dtype=np.int32)
    n, K = nb.shape
    assert p.shape[0] == n and ct.shape == (n,)
    out = np.zeros((n, K, 4), np.float32)
    lib().oracle_edge_features(n, _p(p), _p(bx), K, _p(nb), _p(ct), _p(out))
    return out


def csr(nbr, counts):
    """Compressed-sparse-row form of padded rows: row_ptr (int64 [n + 1]) =
    0 and the running sum of v_i = min(max(counts[i], 0), K); col = the first
    v_i entries of each row, row after row."""
    nb = np.ascontiguousarray(nbr, dtype=np.int32)
    n, K = nb.shape
    v = np.clip(np.asarray(counts, np.int64), 0, K)
    row_ptr = np.zeros(n + 1, np.int64)
    np.cumsum(v, out=row_ptr[1:])
    keep = np.arange(K)[None, :] < v[:, None]
    return row_ptr, nb[keep]


def skin_check(pos, ref, box, skin: float):
    """Returns (max squared displacement, rebuild flag)."""
    p = _pos4(pos)
    r = _pos4(ref)
    bx = _box(box)
    rb = np.zeros(1, np.int32)
    m = lib().oracle_skin_check(p.shape[0], _p(p), _p(r), _p(bx), np.float32(skin), _p(rb))
    return float(np.float32(m)), bool(rb[0])


def displace(pos, seed: int, step: int, sigma: float) -> np.ndarray:
    """Copy of `pos` (n x 4 float32) moved by the stand-in displacement of `step`."""
    p = _pos4(pos).copy()
    lib().oracle_displace(p.shape[0], _p(p), seed, step, np.float32(sigma))
    return p


def md_decisions(pos, box, skin: float, seed: int, sigma: float, steps: int):
    """Skin-check loop from `pos` (the step-0 build positions).

    Returns (decisions int32[steps], final positions, reference positions at
    the last rebuild)."""
    p = _pos4(pos).copy()
    ref = np.zeros_like(p)
    bx = _box(box)
    dec = np.zeros(steps, np.int32)
    lib().oracle_md_decisions(p.shape[0], _p(p), _p(ref), _p(bx), np.float32(skin),
                              seed, np.float32(sigma), steps, _p(dec))
    return dec, p, ref


def canonical_rows(nbr: np.ndarray, counts: np.ndarray) -> np.ndarray:
    """Sort the valid entries of each row ascending; keep -1 padding at the end."""
    K = nbr.shape[1]
    out = np.where(nbr < 0, np.iinfo(np.int32).max, nbr)
    out = np.sort(out, axis=1)
    out = np.where(out == np.iinfo(np.int32).max, -1, out).astype(np.int32)
    del K
    return out

"""Python binding of libnl.so (C ABI in include/nl.h): argument marshalling only.

Every function here mirrors one C entry point of the same name and forwards
torch CUDA tensors as raw device pointers; all work runs in libnl's kernels.
Importing this module loads the library and raises ImportError if it has not
been built (``python -m neighbor_list_construction_b200.build_lib``): there is
no fallback path.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnl.so")

NL_OK, NL_OVERFLOW = 0, 1
NL_ERR_ARG, NL_ERR_BOX, NL_ERR_CUDA, NL_ERR_TIMEOUT, NL_ERR_CAPACITY = -1, -2, -3, -4, -5
NL_ERR_HALO = -6

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libnl.so not built at {LIB_PATH}; run "
                      "`python -m neighbor_list_construction_b200.build_lib`")

_lib = ctypes.CDLL(LIB_PATH)
_vp, _i32, _i64, _f32, _u64 = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                              ctypes.c_uint64)
_SIGS = {
    "nl_create": (_i32, [ctypes.POINTER(_vp), _i64, _i32]),
    "nl_destroy": (None, [_vp]),
    "nl_sort_hilbert": (_i32, [_vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp]),
    "nl_sort_morton": (_i32, [_vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp]),
    "nl_build": (_i32, [_vp, _i64, _vp, _vp, _f32, _f32, _i32, _vp, _vp, _vp]),
    "nl_build_rows": (_i32, [_vp, _i64, _i64, _vp, _vp, _f32, _f32, _i32, _vp, _vp, _vp]),
    "nl_build_rows_dev": (_i32, [_vp, _i64, _vp, _i64, _vp, _vp, _f32, _f32, _i32, _vp, _vp,
                                 _vp]),
    "nl_build_close": (_i32, [_vp, _i64, _vp, _vp, _f32, _f32, _i32, _vp, _vp, _f32, _vp, _vp,
                              _vp]),
    "nl_skin_check": (_i32, [_vp, _i64, _vp, _vp, _f32, _vp, _vp, _vp]),
    "nl_csr_offsets": (_i32, [_vp, _i64, _vp, _i32, _vp, _vp]),
    "nl_csr_fill": (_i32, [_vp, _i64, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp]),
    "nl_edge_features": (_i32, [_vp, _i64, _vp, _vp, _vp, _vp, _i32, _vp, _vp]),
    "nl_replay": (_i32, [_vp, _vp, _i32, _i64, _vp, _vp, _f32, _f32, _i32, _vp, _vp, _vp, _vp]),
    "nl_replay_resort": (_i32, [_vp, _vp, _i32, _i64, _vp, _vp, _vp, _vp, _f32, _f32, _i32, _vp,
                                _vp, _vp, _vp]),
    "nl_step_counter": (_vp, [_vp]),
    "nl_sync_status": (_i32, [_vp, _vp]),
    "nl_wait_selftest": (_i32, [_vp, _i32, _vp]),
    "nl_status_string": (ctypes.c_char_p, [_i32]),
    "nl_last_build_info": (_i32, [_vp, _vp]),
    "nl_profile_enable": (_i32, [_vp, ctypes.c_int]),
    "nl_profile_read": (_i32, [_vp, _vp, _vp, _i32]),
    "nl_profile_phase_name": (ctypes.c_char_p, [_i32]),
    "nl_sort_hilbert_noalloc": (_i32, [_i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "nl_halo_grid": (_i32, [_vp, _f32, _f32, _vp]),
    "nl_halo_mark": (_i32, [_vp, _i64, _vp, _vp, _vp, _i32, _vp, _vp]),
    "nl_halo_needed": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp]),
    "nl_halo_count": (_i32, [_vp, _i64, _vp, _vp, _vp, _vp, _i32, _i32, _vp, _vp]),
    "nl_halo_fill": (_i32, [_vp, _i64, _vp, _vp, _vp, _vp, _i32, _i32, _vp, _vp, _vp, _vp, _vp]),
    "nl_halo_fill_blocks": (_i32, [_vp, _i64, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _vp, _vp,
                                   _vp, _vp]),
    "nl_halo_pack": (_i32, [_vp, _i32, _i32, _vp, _vp, _i64, _i64, _vp, _vp, _vp]),
    "nl_map_ids": (_i32, [_vp, _i64, _i32, _vp, _vp, _i64, _vp, _vp]),
    "nls_displace": (_i32, [_i64, _vp, _u64, _i64, _vp, _f32, _vp]),
    "nls_step_graph": (_i32, [ctypes.POINTER(_vp), _i64, _vp, _u64, _vp, _f32]),
    "nls_step_graph_ids": (_i32, [ctypes.POINTER(_vp), _i64, _vp, _vp, _u64, _vp, _f32]),
    "nls_graph_destroy": (None, [_vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

EXPORTS = tuple(_SIGS)


class NLError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {nl_status_string(status)}")
        self.status = status


def nl_status_string(status: int) -> str:
    return _lib.nl_status_string(status).decode()


def _check(status: int, where: str) -> int:
    if status < 0:
        raise NLError(status, where)
    return status


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


_I32, _I64, _F32 = (torch.int32,), (torch.int64,), (torch.float32,)
_U64 = (torch.int64, torch.uint64)   # 64-bit keys: either view of the bits


def _buf(t: torch.Tensor | None, name: str, dtypes, numel: int | None = None):
    """Pointer of a buffer the library reads or writes through a raw pointer:
    a contiguous CUDA tensor of one of `dtypes` holding at least `numel`
    elements, so that no launch can run past its end.  None stays None."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or t.dtype not in dtypes:
        raise ValueError(f"{name} must be a CUDA tensor of dtype {' or '.join(map(str, dtypes))}")
    if numel is not None and t.numel() < numel:
        raise ValueError(f"{name} holds {t.numel()} elements; at least {numel} are needed")
    return _ptr(t)


def _box(box) -> ctypes.Array:
    b = [float(v) for v in (box.tolist() if hasattr(box, "tolist") else box)]
    if len(b) != 3:
        raise ValueError("box must have 3 entries")
    return (ctypes.c_float * 3)(*b)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _pos(pos: torch.Tensor) -> torch.Tensor:
    if pos.dtype != torch.float32 or pos.dim() != 2 or pos.shape[1] != 4:
        raise ValueError("positions must be a float32 [n, 4] CUDA tensor")
    return pos


# --------------------------------------------------------------- C mirrors
def nl_create(max_atoms: int, max_capacity: int) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    _check(_lib.nl_create(ctypes.byref(h), int(max_atoms), int(max_capacity)), "nl_create")
    return h


def nl_destroy(ctx) -> None:
    _lib.nl_destroy(ctx)


def _sort_outs(n, perm_out, pos_sorted_out, keys_out):
    return (_buf(perm_out, "perm_out", _I32, n), _buf(pos_sorted_out, "pos_sorted_out", _F32, 4 * n),
            _buf(keys_out, "keys_out", _U64, n))


def _rows_outs(n_rows, capacity, nbr_out, counts_out):
    return (_buf(nbr_out, "nbr_out", _I32, int(n_rows) * max(int(capacity), 0)),
            _buf(counts_out, "counts_out", _I32, int(n_rows)))


def nl_sort_hilbert(ctx, pos, box, perm_out, pos_sorted_out, keys_out=None, stream=None) -> int:
    _pos(pos)
    n = pos.shape[0]
    return _check(_lib.nl_sort_hilbert(ctx, n, _ptr(pos), _box(box),
                                       *_sort_outs(n, perm_out, pos_sorted_out, keys_out),
                                       _stream(stream)), "nl_sort_hilbert")


def nl_sort_morton(ctx, pos, box, perm_out, pos_sorted_out, keys_out=None, stream=None) -> int:
    _pos(pos)
    n = pos.shape[0]
    return _check(_lib.nl_sort_morton(ctx, n, _ptr(pos), _box(box),
                                      *_sort_outs(n, perm_out, pos_sorted_out, keys_out),
                                      _stream(stream)), "nl_sort_morton")


def nl_sort_hilbert_noalloc(pos, box, perm_out, pos_sorted_out, keys_out=None, status_out=None,
                            stream=None) -> int:
    _pos(pos)
    n = pos.shape[0]
    return _check(_lib.nl_sort_hilbert_noalloc(n, _ptr(pos), _box(box),
                                               *_sort_outs(n, perm_out, pos_sorted_out, keys_out),
                                               _buf(status_out, "status_out", _I32, 1),
                                               _stream(stream)), "nl_sort_hilbert_noalloc")


def nl_build(ctx, pos, box, cutoff, skin, capacity, nbr_out, counts_out, stream=None) -> int:
    _pos(pos)
    n = pos.shape[0]
    return _check(_lib.nl_build(ctx, n, _ptr(pos), _box(box), float(cutoff), float(skin),
                                int(capacity), *_rows_outs(n, capacity, nbr_out, counts_out),
                                _stream(stream)), "nl_build")


def nl_build_rows(ctx, pos, n_rows, box, cutoff, skin, capacity, nbr_out, counts_out,
                  stream=None) -> int:
    _pos(pos)
    rows = min(max(int(n_rows), 0), pos.shape[0])
    return _check(_lib.nl_build_rows(ctx, pos.shape[0], int(n_rows), _ptr(pos), _box(box),
                                     float(cutoff), float(skin), int(capacity),
                                     *_rows_outs(rows, capacity, nbr_out, counts_out),
                                     _stream(stream)), "nl_build_rows")


def nl_build_close(ctx, pos, box, cutoff, skin, capacity, nbr_out, counts_out, close_d2,
                   min_d2_out, n_close_out, stream=None) -> int:
    _pos(pos)
    n = pos.shape[0]
    return _check(_lib.nl_build_close(ctx, n, _ptr(pos), _box(box), float(cutoff), float(skin),
                                      int(capacity), *_rows_outs(n, capacity, nbr_out, counts_out),
                                      float(close_d2), _buf(min_d2_out, "min_d2_out", _F32, 1),
                                      _buf(n_close_out, "n_close_out", _I64, 1),
                                      _stream(stream)), "nl_build_close")


def nl_skin_check(ctx, pos, box, skin, rebuild_out, max_d2_out=None, stream=None) -> int:
    _pos(pos)
    return _check(_lib.nl_skin_check(ctx, pos.shape[0], _ptr(pos), _box(box), float(skin),
                                     _buf(rebuild_out, "rebuild_out", _I32, 1),
                                     _buf(max_d2_out, "max_d2_out", _F32, 1), _stream(stream)),
                  "nl_skin_check")


def nl_csr_offsets(ctx, counts, capacity, row_ptr_out, stream=None) -> int:
    if counts.dtype != torch.int32 or counts.dim() != 1:
        raise ValueError("counts must be an int32 [n] CUDA tensor")
    n = counts.shape[0]
    if row_ptr_out.dtype != torch.int64 or tuple(row_ptr_out.shape) != (n + 1,):
        raise ValueError("row_ptr_out must be an int64 [n + 1] CUDA tensor")
    return _check(_lib.nl_csr_offsets(ctx, n, _ptr(counts), int(capacity), _ptr(row_ptr_out),
                                      _stream(stream)), "nl_csr_offsets")


def nl_csr_fill(ctx, nbr, counts, row_ptr, col_out, pos=None, box=None, edges_out=None,
                stream=None) -> int:
    n, K = nbr.shape
    if nbr.dtype != torch.int32 or counts.dtype != torch.int32 or tuple(counts.shape) != (n,):
        raise ValueError("nbr must be int32 [n, K] and counts int32 [n]")
    if col_out.dtype != torch.int32 or row_ptr.dtype != torch.int64:
        raise ValueError("col_out must be int32 and row_ptr int64")
    if edges_out is not None:
        _pos(pos)
        if edges_out.dtype != torch.float32 or edges_out.dim() != 2 or edges_out.shape[1] != 4:
            raise ValueError("edges_out must be a float32 [E, 4] CUDA tensor")
    bx = _box(box) if box is not None else None
    return _check(_lib.nl_csr_fill(ctx, n, _ptr(nbr), _ptr(counts), int(K),
                                   _buf(row_ptr, "row_ptr", _I64, n + 1),
                                   _ptr(col_out), _ptr(pos), bx, _ptr(edges_out),
                                   _stream(stream)), "nl_csr_fill")


def nl_edge_features(ctx, pos, box, nbr, counts, edges_out, stream=None) -> int:
    _pos(pos)
    n = pos.shape[0]
    if nbr.dtype != torch.int32 or nbr.dim() != 2 or nbr.shape[0] != n:
        raise ValueError("nbr must be an int32 [n, K] CUDA tensor")
    if counts.dtype != torch.int32 or tuple(counts.shape) != (n,):
        raise ValueError("counts must be an int32 [n] CUDA tensor")
    if edges_out.dtype != torch.float32 or tuple(edges_out.shape) != (n, nbr.shape[1], 4):
        raise ValueError("edges_out must be a float32 [n, K, 4] CUDA tensor")
    return _check(_lib.nl_edge_features(ctx, pos.shape[0], _ptr(pos), _box(box), _ptr(nbr),
                                        _ptr(counts), int(nbr.shape[1]), _ptr(edges_out),
                                        _stream(stream)), "nl_edge_features")


def nl_replay(ctx, step_graph, n_steps, pos, box, cutoff, skin, capacity, nbr, counts,
              decisions_out, stream=None) -> int:
    _pos(pos)
    n = pos.shape[0]
    return _check(_lib.nl_replay(ctx, step_graph, int(n_steps), n, _ptr(pos), _box(box),
                                 float(cutoff), float(skin), int(capacity),
                                 *_rows_outs(n, capacity, nbr, counts),
                                 _buf(decisions_out, "decisions_out", _I32, max(int(n_steps), 0)),
                                 _stream(stream)), "nl_replay")


def nl_replay_resort(ctx, step_graph, n_steps, pos, ids, aux, box, cutoff, skin, capacity, nbr,
                     counts, decisions_out, stream=None) -> int:
    _pos(pos)
    n = pos.shape[0]
    if ids is not None and (ids.dtype != torch.int32 or tuple(ids.shape) != (n,)):
        raise ValueError("ids must be an int32 [n] CUDA tensor")
    if aux is not None and (aux.dtype != torch.float32 or tuple(aux.shape) != (n, 4)):
        raise ValueError("aux must be a float32 [n, 4] CUDA tensor")
    return _check(_lib.nl_replay_resort(ctx, step_graph, int(n_steps), n, _ptr(pos), _ptr(ids),
                                        _ptr(aux), _box(box), float(cutoff), float(skin),
                                        int(capacity), *_rows_outs(n, capacity, nbr, counts),
                                        _buf(decisions_out, "decisions_out", _I32,
                                             max(int(n_steps), 0)),
                                        _stream(stream)), "nl_replay_resort")


def _cells(dims) -> int:
    return math.prod(max(int(x), 0) for x in dims) if len(dims) == 3 else 0


def _dims(dims):
    d = (ctypes.c_int32 * 3)(*[int(x) for x in dims])
    return d


def nl_halo_grid(box, cutoff, skin):
    """Coarse grid of the halo selection: a tuple of 3 ints."""
    out = (ctypes.c_int32 * 3)()
    _check(_lib.nl_halo_grid(_box(box), float(cutoff), float(skin), out), "nl_halo_grid")
    return tuple(out)


def nl_halo_mark(ctx, pos, box, dims, rank, occ_out, stream=None) -> int:
    _pos(pos)
    return _check(_lib.nl_halo_mark(ctx, pos.shape[0], _ptr(pos), _box(box), _dims(dims),
                                    int(rank), _buf(occ_out, "occ_out", _I32, _cells(dims)),
                                    _stream(stream)), "nl_halo_mark")


def nl_halo_needed(ctx, box, dims, occ_all, need_out, stream=None) -> int:
    c = _cells(dims)
    return _check(_lib.nl_halo_needed(ctx, _box(box), _dims(dims),
                                      _buf(occ_all, "occ_all", _I32, c),
                                      _buf(need_out, "need_out", _I32, c), _stream(stream)),
                  "nl_halo_needed")


def nl_build_rows_dev(ctx, pos, n_dev, n_rows, box, cutoff, skin, capacity, nbr_out, counts_out,
                      stream=None) -> int:
    """pos holds room for n_max = pos.shape[0] atoms; n_dev (int64 [1], device)
    says how many take part."""
    _pos(pos)
    rows = min(max(int(n_rows), 0), pos.shape[0])
    return _check(_lib.nl_build_rows_dev(ctx, pos.shape[0], _buf(n_dev, "n_dev", _I64, 1),
                                         int(n_rows), _ptr(pos), _box(box), float(cutoff),
                                         float(skin), int(capacity),
                                         *_rows_outs(rows, capacity, nbr_out, counts_out),
                                         _stream(stream)), "nl_build_rows_dev")


def nl_halo_count(ctx, pos, box, dims, need, rank, nranks, counts_out, stream=None) -> int:
    _pos(pos)
    return _check(_lib.nl_halo_count(ctx, pos.shape[0], _ptr(pos), _box(box), _dims(dims),
                                     _buf(need, "need", _I32, _cells(dims)), int(rank),
                                     int(nranks), _buf(counts_out, "counts_out", _I32, int(nranks)),
                                     _stream(stream)), "nl_halo_count")


def nl_halo_fill(ctx, pos, box, dims, need, rank, nranks, offsets, counts, cursor, send_out,
                 stream=None) -> int:
    _pos(pos)
    q = int(nranks)
    # send_out must hold sum(counts) x 4 floats; the counts live on the device
    return _check(_lib.nl_halo_fill(ctx, pos.shape[0], _ptr(pos), _box(box), _dims(dims),
                                    _buf(need, "need", _I32, _cells(dims)), int(rank), q,
                                    _buf(offsets, "offsets", _I32, q), _buf(counts, "counts", _I32, q),
                                    _buf(cursor, "cursor", _I32, q), _buf(send_out, "send_out", _F32),
                                    _stream(stream)), "nl_halo_fill")


def nl_halo_fill_blocks(ctx, pos, box, dims, need, rank, nranks, block, counts, cursor, send_out,
                        stream=None) -> int:
    _pos(pos)
    q = int(nranks)
    return _check(_lib.nl_halo_fill_blocks(ctx, pos.shape[0], _ptr(pos), _box(box), _dims(dims),
                                           _buf(need, "need", _I32, _cells(dims)), int(rank), q,
                                           int(block), _buf(counts, "counts", _I32, q),
                                           _buf(cursor, "cursor", _I32, q),
                                           _buf(send_out, "send_out", _F32, q * int(block) * 4),
                                           _stream(stream)), "nl_halo_fill_blocks")


def nl_halo_pack(ctx, nranks, block, recv_counts, recv, n_own, pos_all, n_all_out,
                 stream=None) -> int:
    """pos_all holds room for n_max = pos_all.shape[0] atoms, its first n_own
    the own ones."""
    _pos(pos_all)
    q, blk = int(nranks), int(block)
    return _check(_lib.nl_halo_pack(ctx, q, blk, _buf(recv_counts, "recv_counts", _I32, q),
                                    _buf(recv, "recv", _F32, q * blk * 4), int(n_own),
                                    pos_all.shape[0], _ptr(pos_all),
                                    _buf(n_all_out, "n_all_out", _I64, 1), _stream(stream)),
                  "nl_halo_pack")


def nl_map_ids(ctx, nbr, pos_all, counts=None, stream=None) -> int:
    _pos(pos_all)
    if nbr.dtype != torch.int32 or nbr.dim() != 2:
        raise ValueError("nbr must be an int32 [n_rows, K] CUDA tensor")
    return _check(_lib.nl_map_ids(ctx, nbr.shape[0], int(nbr.shape[1]), _ptr(nbr),
                                  _buf(counts, "counts", _I32, nbr.shape[0]),
                                  pos_all.shape[0], _ptr(pos_all), _stream(stream)), "nl_map_ids")


def nl_step_counter(ctx) -> int:
    return _lib.nl_step_counter(ctx)


def nl_wait_selftest(ctx, max_polls: int, stream=None) -> int:
    return _check(_lib.nl_wait_selftest(ctx, int(max_polls), _stream(stream)), "nl_wait_selftest")


def nl_sync_status(ctx, stream=None) -> int:
    return _check(_lib.nl_sync_status(ctx, _stream(stream)), "nl_sync_status")


def nl_last_build_info(ctx) -> list[int]:
    out = (ctypes.c_int64 * 8)()
    _check(_lib.nl_last_build_info(ctx, out), "nl_last_build_info")
    return list(out)


def nl_profile_enable(ctx, on: bool = True) -> None:
    _check(_lib.nl_profile_enable(ctx, 1 if on else 0), "nl_profile_enable")


def nl_profile_read(ctx) -> dict[str, tuple[float, int]]:
    ms = (ctypes.c_double * 32)()
    ln = (ctypes.c_int64 * 32)()
    n = _lib.nl_profile_read(ctx, ms, ln, 32)
    if n < 0:
        raise NLError(NL_ERR_CUDA, "nl_profile_read")
    return {_lib.nl_profile_phase_name(p).decode(): (ms[p], ln[p]) for p in range(n)}


def nl_profile_phase_name(phase: int) -> str:
    return _lib.nl_profile_phase_name(int(phase)).decode()


def nls_displace(pos, seed: int, step: int, sigma: float, step_dev: int | None = None,
                 stream=None) -> None:
    _pos(pos)
    _check(_lib.nls_displace(pos.shape[0], _ptr(pos), int(seed) & (2 ** 64 - 1), int(step),
                             ctypes.c_void_p(step_dev) if step_dev else None, float(sigma),
                             _stream(stream)), "nls_displace")


def nls_step_graph(pos, seed: int, step_dev: int, sigma: float) -> ctypes.c_void_p:
    _pos(pos)
    g = ctypes.c_void_p()
    _check(_lib.nls_step_graph(ctypes.byref(g), pos.shape[0], _ptr(pos), int(seed) & (2 ** 64 - 1),
                               ctypes.c_void_p(step_dev), float(sigma)), "nls_step_graph")
    return g


def nls_step_graph_ids(pos, ids, seed: int, step_dev: int, sigma: float) -> ctypes.c_void_p:
    _pos(pos)
    g = ctypes.c_void_p()
    _check(_lib.nls_step_graph_ids(ctypes.byref(g), pos.shape[0], _ptr(pos), _ptr(ids),
                                   int(seed) & (2 ** 64 - 1), ctypes.c_void_p(step_dev),
                                   float(sigma)), "nls_step_graph_ids")
    return g


def nls_graph_destroy(graph) -> None:
    _lib.nls_graph_destroy(graph)


# ------------------------------------------------------------ convenience
class Context:
    """Owns an nl_ctx and allocates output tensors for the common calls."""

    def __init__(self, max_atoms: int, max_capacity: int):
        self.handle = nl_create(max_atoms, max_capacity)

    def close(self) -> None:
        if self.handle:
            nl_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def sort(self, pos, box, curve: str = "hilbert", keys: bool = False, stream=None):
        n = pos.shape[0]
        perm = torch.empty(n, dtype=torch.int32, device=pos.device)
        ps = torch.empty(n, 4, dtype=torch.float32, device=pos.device)
        ks = torch.empty(n, dtype=torch.int64, device=pos.device) if keys else None
        fn = nl_sort_hilbert if curve == "hilbert" else nl_sort_morton
        fn(self.handle, pos, box, perm, ps, ks, stream)
        return perm, ps, ks

    def build(self, pos, box, cutoff, skin, capacity, nbr=None, counts=None, stream=None):
        n = pos.shape[0]
        if nbr is None:
            nbr = torch.empty(n, capacity, dtype=torch.int32, device=pos.device)
        if counts is None:
            counts = torch.empty(n, dtype=torch.int32, device=pos.device)
        nl_build(self.handle, pos, box, cutoff, skin, capacity, nbr, counts, stream)
        return nbr, counts

    def build_rows(self, pos, n_rows, box, cutoff, skin, capacity, stream=None):
        """Rows for the first n_rows atoms of pos, neighbors among all."""
        nbr = torch.empty(n_rows, capacity, dtype=torch.int32, device=pos.device)
        counts = torch.empty(n_rows, dtype=torch.int32, device=pos.device)
        nl_build_rows(self.handle, pos, n_rows, box, cutoff, skin, capacity,
                      nbr if n_rows else None, counts if n_rows else None, stream)
        return nbr, counts

    def build_close(self, pos, box, cutoff, skin, capacity, close_d2, stream=None):
        """nl_build plus the close-pair detector: (nbr, counts, min_d2[1], n_close[1])."""
        n = pos.shape[0]
        nbr = torch.empty(n, capacity, dtype=torch.int32, device=pos.device)
        counts = torch.empty(n, dtype=torch.int32, device=pos.device)
        mn = torch.empty(1, dtype=torch.float32, device=pos.device)
        nc = torch.empty(1, dtype=torch.int64, device=pos.device)
        nl_build_close(self.handle, pos, box, cutoff, skin, capacity, nbr, counts, close_d2, mn,
                       nc, stream)
        return nbr, counts, mn, nc

    def to_csr(self, nbr, counts, pos=None, box=None, stream=None):
        """CSR form of the rows: (row_ptr int64 [n + 1], col int32 [E]) and,
        with pos and box, the entries' edge features float32 [E, 4]."""
        n, K = nbr.shape
        row_ptr = torch.empty(n + 1, dtype=torch.int64, device=nbr.device)
        nl_csr_offsets(self.handle, counts, K, row_ptr, stream)
        E = int(row_ptr[n].item())
        # at least one element, so the buffers have an address when E = 0
        col = torch.empty(max(E, 1), dtype=torch.int32, device=nbr.device)
        edges = None
        if pos is not None:
            edges = torch.empty(max(E, 1), 4, dtype=torch.float32, device=nbr.device)
        nl_csr_fill(self.handle, nbr, counts, row_ptr, col, pos, box, edges, stream)
        col = col[:E]
        return (row_ptr, col) if edges is None else (row_ptr, col, edges[:E])

    def edge_features(self, pos, box, nbr, counts, stream=None):
        """Per-slot (dx, dy, dz, r) of the rows: float32 [n, K, 4]."""
        n, K = nbr.shape
        out = torch.empty(n, K, 4, dtype=torch.float32, device=pos.device)
        nl_edge_features(self.handle, pos, box, nbr, counts, out, stream)
        return out

    def skin_check(self, pos, box, skin, stream=None):
        rb = torch.zeros(1, dtype=torch.int32, device=pos.device)
        md = torch.zeros(1, dtype=torch.float32, device=pos.device)
        nl_skin_check(self.handle, pos, box, skin, rb, md, stream)
        return rb, md

    def sync_status(self, stream=None) -> int:
        return nl_sync_status(self.handle, stream)

"""The Python binding's marshalling, on the CPU with a stand-in for libnl:
every mirror function hands its C entry point exactly the arguments the
declared signature lists (each convertible to its ctypes type), and a buffer
that is too small or of the wrong dtype is refused before any call, so no
launch can write past the end of a caller's tensor."""
import ctypes

import pytest
import torch

from neighbor_list_construction_b200 import nl

N, K, STEPS = 10, 8, 4
BOX = [9.0, 9.0, 9.0]
DIMS = (2, 3, 2)


class FakeLib:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        res, argtypes = nl._SIGS[name]

        def call(*args):
            assert len(args) == len(argtypes), (name, len(args), len(argtypes))
            for v, t in zip(args, argtypes):
                if v is not None:
                    t.from_param(v)          # raises on a value of the wrong kind
            self.calls.append(name)
            return 0
        return call


@pytest.fixture
def fake(monkeypatch):
    f = FakeLib()
    monkeypatch.setattr(nl, "_lib", f)
    # CPU tensors stand in for device memory: only the pointer is forwarded
    monkeypatch.setattr(nl, "_ptr", lambda t: None if t is None else ctypes.c_void_p(t.data_ptr()))
    monkeypatch.setattr(nl, "_stream", lambda s: ctypes.c_void_p(0))
    return f


def bufs():
    i32 = lambda *s: torch.zeros(*s, dtype=torch.int32)
    b = dict(pos=torch.zeros(N, 4), perm=i32(N), ps=torch.zeros(N, 4),
             keys=torch.zeros(N, dtype=torch.int64), status=i32(1), nbr=i32(N, K), cnt=i32(N),
             nbr5=i32(5, K), cnt5=i32(5), mn=torch.zeros(1), nc=torch.zeros(1, dtype=torch.int64),
             rb=i32(1), md=torch.zeros(1), row_ptr=torch.zeros(N + 1, dtype=torch.int64),
             col=i32(N * K), edges=torch.zeros(N * K, 4), edges3=torch.zeros(N, K, 4),
             dec=i32(STEPS), ids=i32(N), aux=torch.zeros(N, 4), occ=i32(12), need=i32(12),
             cnt2=i32(2), offs=i32(2), cursor=i32(2), send=torch.zeros(N, 4),
             ndev=torch.zeros(1, dtype=torch.int64), blocks=torch.zeros(2 * 3, 4))
    return b


def calls(b):
    ctx = ctypes.c_void_p(0)
    return {
        "nl_sort_hilbert": lambda: nl.nl_sort_hilbert(ctx, b["pos"], BOX, b["perm"], b["ps"], b["keys"]),
        "nl_sort_morton": lambda: nl.nl_sort_morton(ctx, b["pos"], BOX, b["perm"], b["ps"]),
        "nl_sort_hilbert_noalloc": lambda: nl.nl_sort_hilbert_noalloc(
            b["pos"], BOX, b["perm"], b["ps"], b["keys"], b["status"]),
        "nl_build": lambda: nl.nl_build(ctx, b["pos"], BOX, 2.0, 0.5, K, b["nbr"], b["cnt"]),
        "nl_build_rows": lambda: nl.nl_build_rows(ctx, b["pos"], 5, BOX, 2.0, 0.5, K, b["nbr5"],
                                                  b["cnt5"]),
        "nl_build_close": lambda: nl.nl_build_close(ctx, b["pos"], BOX, 2.0, 0.5, K, b["nbr"],
                                                    b["cnt"], 1.0, b["mn"], b["nc"]),
        "nl_skin_check": lambda: nl.nl_skin_check(ctx, b["pos"], BOX, 0.5, b["rb"], b["md"]),
        "nl_csr_offsets": lambda: nl.nl_csr_offsets(ctx, b["cnt"], K, b["row_ptr"]),
        "nl_csr_fill": lambda: nl.nl_csr_fill(ctx, b["nbr"], b["cnt"], b["row_ptr"], b["col"],
                                              b["pos"], BOX, b["edges"]),
        "nl_edge_features": lambda: nl.nl_edge_features(ctx, b["pos"], BOX, b["nbr"], b["cnt"],
                                                        b["edges3"]),
        "nl_replay": lambda: nl.nl_replay(ctx, None, STEPS, b["pos"], BOX, 2.0, 0.5, K, b["nbr"],
                                          b["cnt"], b["dec"]),
        "nl_replay_resort": lambda: nl.nl_replay_resort(ctx, None, STEPS, b["pos"], b["ids"],
                                                        b["aux"], BOX, 2.0, 0.5, K, b["nbr"],
                                                        b["cnt"], b["dec"]),
        "nl_halo_mark": lambda: nl.nl_halo_mark(ctx, b["pos"], BOX, DIMS, 0, b["occ"]),
        "nl_halo_needed": lambda: nl.nl_halo_needed(ctx, BOX, DIMS, b["occ"], b["need"]),
        "nl_halo_count": lambda: nl.nl_halo_count(ctx, b["pos"], BOX, DIMS, b["need"], 0, 2,
                                                  b["cnt2"]),
        "nl_halo_fill": lambda: nl.nl_halo_fill(ctx, b["pos"], BOX, DIMS, b["need"], 0, 2,
                                                b["offs"], b["cnt2"], b["cursor"], b["send"]),
        "nl_halo_fill_blocks": lambda: nl.nl_halo_fill_blocks(ctx, b["pos"], BOX, DIMS, b["need"],
                                                              0, 2, 3, b["cnt2"], b["cursor"],
                                                              b["blocks"]),
        "nl_halo_pack": lambda: nl.nl_halo_pack(ctx, 2, 3, b["cnt2"], b["blocks"], 4, b["pos"],
                                                b["ndev"]),
        "nl_build_rows_dev": lambda: nl.nl_build_rows_dev(ctx, b["pos"], b["ndev"], 5, BOX, 2.0,
                                                          0.5, K, b["nbr5"], b["cnt5"]),
        "nl_map_ids": lambda: nl.nl_map_ids(ctx, b["nbr"], b["pos"], b["cnt"]),
        "nl_wait_selftest": lambda: nl.nl_wait_selftest(ctx, 1000),
    }


def test_every_mirror_passes_its_signature(fake):
    cs = calls(bufs())
    for name, fn in cs.items():
        assert fn() == 0
    assert fake.calls == list(cs)


# (function, buffer, replacement): one buffer made too small or of another dtype
BAD = [
    ("nl_sort_hilbert", "perm", torch.zeros(N - 1, dtype=torch.int32)),
    ("nl_sort_hilbert", "ps", torch.zeros(N - 1, 4)),
    ("nl_sort_hilbert", "keys", torch.zeros(N, dtype=torch.int32)),
    ("nl_sort_hilbert_noalloc", "status", torch.zeros(0, dtype=torch.int32)),
    ("nl_build", "nbr", torch.zeros(N, K - 1, dtype=torch.int32)),
    ("nl_build", "nbr", torch.zeros(N, K, dtype=torch.int64)),
    ("nl_build", "cnt", torch.zeros(N - 1, dtype=torch.int32)),
    ("nl_build_rows", "nbr5", torch.zeros(4, K, dtype=torch.int32)),
    ("nl_build_rows", "cnt5", torch.zeros(4, dtype=torch.int32)),
    ("nl_build_close", "nc", torch.zeros(1, dtype=torch.float32)),
    ("nl_build_close", "mn", torch.zeros(0)),
    ("nl_skin_check", "rb", torch.zeros(0, dtype=torch.int32)),
    ("nl_skin_check", "md", torch.zeros(1, dtype=torch.float64)),
    ("nl_csr_fill", "row_ptr", torch.zeros(N, dtype=torch.int64)),
    ("nl_replay", "dec", torch.zeros(STEPS - 1, dtype=torch.int32)),
    ("nl_replay", "cnt", torch.zeros(N - 1, dtype=torch.int32)),
    ("nl_replay_resort", "nbr", torch.zeros(N - 1, K, dtype=torch.int32)),
    ("nl_halo_mark", "occ", torch.zeros(11, dtype=torch.int32)),
    ("nl_halo_needed", "need", torch.zeros(11, dtype=torch.int32)),
    ("nl_halo_count", "cnt2", torch.zeros(1, dtype=torch.int32)),
    ("nl_halo_fill", "cursor", torch.zeros(1, dtype=torch.int32)),
    ("nl_map_ids", "cnt", torch.zeros(N - 1, dtype=torch.int32)),
    ("nl_halo_fill_blocks", "blocks", torch.zeros(5, 4)),
    ("nl_halo_pack", "ndev", torch.zeros(1, dtype=torch.int32)),
    ("nl_halo_pack", "cnt2", torch.zeros(1, dtype=torch.int32)),
    ("nl_build_rows_dev", "ndev", torch.zeros(0, dtype=torch.int64)),
    ("nl_build_rows_dev", "nbr5", torch.zeros(4, K, dtype=torch.int32)),
]


@pytest.mark.parametrize("fn,key,bad", BAD, ids=[f"{f}-{k}-{i}" for i, (f, k, _) in enumerate(BAD)])
def test_small_or_mistyped_buffer_is_refused(fake, fn, key, bad):
    b = bufs()
    b[key] = bad
    with pytest.raises(ValueError):
        calls(b)[fn]()
    assert fake.calls == []


def test_buffer_check_on_real_tensors():
    """Without the stand-ins: size and dtype are checked first, and a CPU
    tensor that passes them is still refused as not on the device."""
    with pytest.raises(ValueError, match="at least 4"):
        nl._buf(torch.zeros(3, dtype=torch.int32), "x", nl._I32, 4)
    with pytest.raises(ValueError, match="dtype"):
        nl._buf(torch.zeros(4, dtype=torch.int64), "x", nl._I32, 4)
    with pytest.raises(ValueError, match="CUDA"):
        nl._buf(torch.zeros(4, dtype=torch.int32), "x", nl._I32, 4)
    assert nl._buf(None, "x", nl._I32, 4) is None


def test_context_methods_allocate_what_the_calls_need(fake):
    """The Context helpers allocate buffers that pass the checks, including
    the empty row range (no buffers at all)."""
    ctx = nl.Context(N, K)
    b = bufs()
    perm, ps, ks = ctx.sort(b["pos"], BOX, keys=True)
    assert perm.shape == (N,) and ps.shape == (N, 4) and ks.shape == (N,)
    ctx.sort(b["pos"], BOX, curve="morton")
    nbr, cnt = ctx.build(b["pos"], BOX, 2.0, 0.5, K)
    assert nbr.shape == (N, K) and cnt.shape == (N,)
    for rows in (0, 5, N):
        nbr_r, cnt_r = ctx.build_rows(b["pos"], rows, BOX, 2.0, 0.5, K)
        assert nbr_r.shape == (rows, K)
    ctx.build_close(b["pos"], BOX, 2.0, 0.5, K, 1.0)
    assert ctx.edge_features(b["pos"], BOX, nbr, cnt).shape == (N, K, 4)
    ctx.skin_check(b["pos"], BOX, 0.5)
    assert fake.calls == ["nl_create", "nl_sort_hilbert", "nl_sort_morton", "nl_build",
                          "nl_build_rows", "nl_build_rows", "nl_build_rows", "nl_build_close",
                          "nl_edge_features", "nl_skin_check"]

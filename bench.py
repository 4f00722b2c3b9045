"""Benchmark of the neighbor-list hot path on B200.

One step = nl_sort_hilbert + nl_build + nl_skin_check on the 10.29M-atom
salt-solution workload (rigid water + 0.15 M NaCl on 151^3 sites, cutoff
5.75 A, skin 1.0 A, capacity 256), inputs resident in HBM.  Prints one JSON
line (rank 0).  `--impl reference` times the CPU oracle instead, on a
bounded sample of the same workload recipe.

Multi-GPU: the path does not shard across GPUs in this build (one problem per
GPU), so `--gpus N` under torchrun runs N independent replicas; `value` is
the atoms of all replicas over the slowest replica's time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "neighbor-list build atoms/s and pairs/s at 1 B200; % of HBM roofline"
NOMINAL_HBM_GBS = 8000.0

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one
# pair-search launch on the saltwater10m workload, from one ncu capture.  It
# belongs to the kernel source it was taken on (nl_pairs.cu and the device
# header it includes): with any other source the bench reports null.
PAIR_TRAFFIC = {"workload": "saltwater10m",
                "sha256": "8398376fd4c3185f8fde92f93c2db1636f1864cd7bbb4912c8fb704c611995a4",
                "bytes": 724856832 + 10774896128}


def pair_traffic(workload: str):
    import hashlib
    h = hashlib.sha256()
    for f in ("nl_pairs.cu", "nl_device.cuh"):
        with open(os.path.join(ROOT, "neighbor_list_construction_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    if workload == PAIR_TRAFFIC["workload"] and h.hexdigest() == PAIR_TRAFFIC["sha256"]:
        return PAIR_TRAFFIC["bytes"]
    return None


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock/throttle samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        # nvidia-smi numbers GPUs physically; map through CUDA_VISIBLE_DEVICES
        vis = [v.strip() for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
        self.gpu = vis[gpu_index] if gpu_index < len(vis) else str(gpu_index)
        self.proc = None
        self.lines: list[str] = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def window(self, t0: float, t1: float) -> dict:
        """Median clocks and active throttle reasons of the samples taken
        between host times t0 and t1 (the sampler keeps running)."""
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        deadline = time.monotonic() + 1.0
        while time.monotonic() < deadline and (not self.lines or self.lines[-1][0] < t1):
            time.sleep(0.05)
        return self._summary([ln for (t, ln) in list(self.lines) if t0 <= t <= t1 + 0.15])

    def stop(self) -> None:
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)

    def _summary(self, lines) -> dict:
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_step(w, threads: int, steps: int = 1) -> dict:
    """The CPU oracle, as it stands, on workload `w`: curve sort + neighbor
    list + skin check per step, its per-atom and per-row loops on `threads`
    OpenMP threads (1 = the plain single-threaded oracle)."""
    import oracle
    oracle.lib()
    old = oracle.set_threads(threads)
    try:
        t0 = time.perf_counter()
        pairs = 0
        for _ in range(steps):
            perm, _ = oracle.sort(w.pos, w.box)
            ps = w.pos[perm]
            nbr, cnt, _ = oracle.build(ps, w.box, w.cutoff, w.skin, w.capacity)
            oracle.skin_check(ps, ps, w.box, w.skin)
            pairs += int(cnt.sum())
            del nbr
        dt = time.perf_counter() - t0
    finally:
        oracle.set_threads(old)
    return {"value": steps * w.n / dt, "unit": "atoms/s", "cores": threads, "kind": "oracle",
            "pairs_per_s": pairs / dt, "seconds": dt, "steps": steps}


def sample_workload(nside: int = 66):
    """A smaller instance of the salt-solution recipe (nside^3 sites; 66 ->
    859,376 atoms, 1/12 of saltwater10m): same density, cutoff 5.75, skin 1.0,
    capacity 256."""
    from neighbor_list_construction_b200 import workloads
    return workloads.make(f"saltwater_n{nside}", seed=4)


def cpu_baseline(workload: str, w) -> dict:
    """The oracle on the benchmark workload itself, all host cores (one step),
    and single-threaded on the 66^3-site instance of the same recipe."""
    cores = cpu_cores()
    full = oracle_step(w, cores)
    small = sample_workload()
    one = oracle_step(small, 1)
    return {"value": full["value"], "unit": "atoms/s", "cores": cores, "kind": "oracle",
            "sample": f"{workload} itself ({w.n} atoms): sort+build+skin x1 on {cores} host "
                      f"cores ({cpu_model()}), {full['seconds']:.1f} s",
            "pairs_per_s": full["pairs_per_s"],
            "single_core": {"value": one["value"], "unit": "atoms/s", "cores": 1,
                            "sample": f"{small.n} atoms, salt-solution recipe on 66^3 sites, "
                                      f"sort+build+skin x1, {one['seconds']:.1f} s"}}


def arm_config(workload: str, world: int) -> dict:
    """The config of the GPU arm's line, from the workload table."""
    from neighbor_list_construction_b200 import workloads
    n, cutoff, skin, K, desc = workloads.INFO[workload]
    return {"workload": f"{workload}: {desc}", "atoms": n, "cutoff": cutoff, "skin": skin,
            "capacity": K, "step": "nl_sort_hilbert + nl_build + nl_skin_check",
            "parallelism": "replicas" if world > 1 else "single"}


def run_reference(args, rank: int, world: int) -> None:
    """The oracle, as it stands, on all host cores: K timed steps (after up to
    3 warm-up steps), each one curve sort + neighbor list + skin check of the
    66^3-site instance of the benchmark's salt-solution recipe (859,376 atoms,
    a twelfth of saltwater10m), so a 20-step run takes about a minute."""
    if rank != 0:
        return
    cores = cpu_cores()
    small = sample_workload()
    warm = max(0, min(args.warmup, 3))
    if warm:
        oracle_step(small, cores, warm)
    r = oracle_step(small, cores, args.steps)
    cfg = arm_config(args.workload, world)
    sample = (f"{small.n} atoms, salt-solution recipe on 66^3 sites (same density, cutoff "
              f"5.75, skin 1.0, capacity 256), sort+build+skin x{args.steps} on {cores} host "
              f"cores ({cpu_model()}), {r['seconds']:.1f} s")
    cfg["sample"] = sample
    line = {
        "impl": "reference", "metric": METRIC, "value": r["value"], "unit": "atoms/s",
        "n_gpus": world, "steps": args.steps, "warmup": warm,
        "ms_per_step": 1000.0 * r["seconds"] / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": cfg,
        "cpu_baseline": {"value": r["value"], "unit": "atoms/s", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": r["value"], "unit": "atoms/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "pairs_per_s": r["pairs_per_s"],
    }
    print(json.dumps(line), flush=True)


def interval_timing(nl, torch, h, ps_src, w, K, steps: int, seed: int = 2024) -> dict:
    """The skin-check interval: `steps` iterations of [stand-in MD step ->
    skin check -> rebuild if needed], once as one replayed CUDA graph
    (nl_replay) and once eagerly from the host (launch, read the decision,
    rebuild).  Device time per step for each."""
    n = ps_src.shape[0]
    stream = torch.cuda.current_stream()
    nbr = torch.empty(n, K, dtype=torch.int32, device="cuda")
    cnt = torch.empty(n, dtype=torch.int32, device="cuda")
    dec = torch.zeros(steps, dtype=torch.int32, device="cuda")
    rb = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = {}
    # graph
    p = ps_src.clone()
    nl.nl_build(h, p, w.box, w.cutoff, w.skin, K, nbr, cnt, stream)
    g = nl.nls_step_graph(p, seed, nl.nl_step_counter(h), w.sigma_step)
    try:
        nl.nl_replay(h, g, steps, p, w.box, w.cutoff, w.skin, K, nbr, cnt, dec, stream)  # warm
        p.copy_(ps_src)
        nl.nl_build(h, p, w.box, w.cutoff, w.skin, K, nbr, cnt, stream)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        nl.nl_replay(h, g, steps, p, w.box, w.cutoff, w.skin, K, nbr, cnt, dec, stream)
        e1.record(stream)
        torch.cuda.synchronize()
        out["graph_ms_per_step"] = e0.elapsed_time(e1) / steps
        out["rebuilds"] = int(dec.sum().item())
    finally:
        nl.nls_graph_destroy(g)
    # graph, re-sorting at each rebuild (ids follow the atoms)
    p = ps_src.clone()
    ids = torch.arange(n, dtype=torch.int32, device="cuda")
    nl.nl_build(h, p, w.box, w.cutoff, w.skin, K, nbr, cnt, stream)
    g = nl.nls_step_graph_ids(p, ids, seed, nl.nl_step_counter(h), w.sigma_step)
    try:
        nl.nl_replay_resort(h, g, steps, p, ids, None, w.box, w.cutoff, w.skin, K, nbr, cnt, dec,
                            stream)  # warm
        p.copy_(ps_src)
        ids.copy_(torch.arange(n, dtype=torch.int32, device="cuda"))
        nl.nl_build(h, p, w.box, w.cutoff, w.skin, K, nbr, cnt, stream)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        nl.nl_replay_resort(h, g, steps, p, ids, None, w.box, w.cutoff, w.skin, K, nbr, cnt, dec,
                            stream)
        e1.record(stream)
        torch.cuda.synchronize()
        out["graph_resort_ms_per_step"] = e0.elapsed_time(e1) / steps
        out["resort_rebuilds"] = int(dec.sum().item())
    finally:
        nl.nls_graph_destroy(g)
    # eager
    p.copy_(ps_src)
    nl.nl_build(h, p, w.box, w.cutoff, w.skin, K, nbr, cnt, stream)
    torch.cuda.synchronize()
    rbh = torch.zeros(1, dtype=torch.int32).pin_memory()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    rebuilds = 0
    for t in range(1, steps + 1):
        nl.nls_displace(p, seed, t, w.sigma_step, None, stream)
        nl.nl_skin_check(h, p, w.box, w.skin, rb, None, stream)
        rbh.copy_(rb, non_blocking=True)
        stream.synchronize()
        if rbh.item():
            rebuilds += 1
            nl.nl_build(h, p, w.box, w.cutoff, w.skin, K, nbr, cnt, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    out["eager_ms_per_step"] = e0.elapsed_time(e1) / steps
    out["eager_rebuilds"] = rebuilds
    out["steps"] = steps
    out["graph_speedup"] = out["eager_ms_per_step"] / out["graph_ms_per_step"]
    return out


def curve_comparison(nl, torch, h, pos, w, K, reps: int = 5) -> dict:
    """nl_build time after a Hilbert sort vs after a Morton sort (same atoms)."""
    n = pos.shape[0]
    stream = torch.cuda.current_stream()
    perm = torch.empty(n, dtype=torch.int32, device="cuda")
    ps = torch.empty(n, 4, dtype=torch.float32, device="cuda")
    nbr = torch.empty(n, K, dtype=torch.int32, device="cuda")
    cnt = torch.empty(n, dtype=torch.int32, device="cuda")
    res = {}
    for curve, fn in (("hilbert", nl.nl_sort_hilbert), ("morton", nl.nl_sort_morton)):
        fn(h, pos, w.box, perm, ps, None, stream)
        nl.nl_build(h, ps, w.box, w.cutoff, w.skin, K, nbr, cnt, stream)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            nl.nl_build(h, ps, w.box, w.cutoff, w.skin, K, nbr, cnt, stream)
        e1.record(stream)
        torch.cuda.synchronize()
        res[f"{curve}_build_ms"] = e0.elapsed_time(e1) / reps
    return res


def close_pair_timing(nl, torch, h, ps, w, K, close_d2: float = 1.0, reps: int = 5) -> dict:
    """nl_build_close (the list plus the close-pair detector) against
    nl_build on the same sorted positions: device time per call, and the
    detector's results (smallest pair r2, directed pairs with r2 < close_d2)."""
    n = ps.shape[0]
    stream = torch.cuda.current_stream()
    nbr = torch.empty(n, K, dtype=torch.int32, device="cuda")
    cnt = torch.empty(n, dtype=torch.int32, device="cuda")
    mn = torch.empty(1, dtype=torch.float32, device="cuda")
    nc = torch.empty(1, dtype=torch.int64, device="cuda")
    res = {"close_d2": close_d2}
    for name in ("build", "build_close"):
        def call():
            if name == "build":
                nl.nl_build(h, ps, w.box, w.cutoff, w.skin, K, nbr, cnt, stream)
            else:
                nl.nl_build_close(h, ps, w.box, w.cutoff, w.skin, K, nbr, cnt, close_d2, mn, nc,
                                  stream)
        call()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            call()
        e1.record(stream)
        torch.cuda.synchronize()
        res[f"{name}_ms"] = e0.elapsed_time(e1) / reps
    res["min_d2"] = float(mn.item())
    res["n_close"] = int(nc.item())
    return res


def edge_feature_timing(nl, torch, h, ps, w, K, reps: int = 5) -> dict:
    """nl_edge_features on the rows of one nl_build: device time per call and
    its HBM roofline.  Algorithmic bytes: counts and positions of every row
    (4 + 16 per atom), the index of every valid slot (4 per pair), and the
    K float4 features of every row (16 K per atom); the gathered neighbor
    positions are counted once, with the rows' own."""
    n = ps.shape[0]
    stream = torch.cuda.current_stream()
    nbr = torch.empty(n, K, dtype=torch.int32, device="cuda")
    cnt = torch.empty(n, dtype=torch.int32, device="cuda")
    nl.nl_build(h, ps, w.box, w.cutoff, w.skin, K, nbr, cnt, stream)
    out = torch.empty(n, K, 4, dtype=torch.float32, device="cuda")
    nl.nl_edge_features(h, ps, w.box, nbr, cnt, out, stream)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        nl.nl_edge_features(h, ps, w.box, nbr, cnt, out, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    slots = int(cnt.clamp(max=K).to(torch.int64).sum().item())
    alg = n * (4 + 16 + 16 * K) + 4 * slots
    peak = measured_peaks()
    gbs = alg / (ms * 1e-3) / 1e9
    del out
    # the CSR form with features: offsets, entries and (dx, dy, dz, r) per
    # entry, no padding.  Algorithmic bytes: counts, positions and offsets
    # (4 + 16 + 8 per atom), index in and index + feature out (4 + 20 per entry)
    row_ptr = torch.empty(n + 1, dtype=torch.int64, device="cuda")
    nl.nl_csr_offsets(h, cnt, K, row_ptr, stream)
    E = int(row_ptr[n].item())
    col = torch.empty(E, dtype=torch.int32, device="cuda")
    feat = torch.empty(E, 4, dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(reps):
        nl.nl_csr_offsets(h, cnt, K, row_ptr, stream)
        nl.nl_csr_fill(h, nbr, cnt, row_ptr, col, ps, w.box, feat, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    csr_ms = e0.elapsed_time(e1) / reps
    csr_alg = n * (4 + 16 + 8) + E * (4 + 4 + 16)
    csr_gbs = csr_alg / (csr_ms * 1e-3) / 1e9
    del col, feat, row_ptr
    return {"ms": ms, "bytes": alg, "achieved_gbs": gbs, "peak_gbs": peak["hbm_gbs"],
            "peak_source": peak["source"], "frac": gbs / peak["hbm_gbs"],
            "layout": f"float32 [{n}, {K}, 4] (dx, dy, dz, r), zero padding",
            "csr": {"ms": csr_ms, "entries": E, "bytes": csr_alg, "achieved_gbs": csr_gbs,
                    "frac": csr_gbs / peak["hbm_gbs"],
                    "layout": f"int64 row_ptr [{n + 1}], int32 col [{E}], float32 [{E}, 4]"}}


def sharded_timing(torch, ctx, ps, w, K, nranks: int = 8, reps: int = 2) -> dict:
    """The curve-sharded build of the whole system with nranks equal-count
    shards, all in this process on this GPU (collectives routed in memory):
    halo sizes, and the time of the whole sharded build (all shards, their
    no host reads once the halo block is agreed) against one nl_build of the
    whole system."""
    from neighbor_list_construction_b200 import shard
    n = ps.shape[0]
    p = shard.with_ids(ps, 0)
    bounds = shard.shard_bounds(n, nranks)
    shards = [p[s:e] for s, e in bounds]
    res = shard.build_sharded_local(ctx, shards, w.box, w.cutoff, w.skin, K)
    halos = [int(r[2].item()) for r in res]
    block = res[0][3]
    del res
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        res = shard.build_sharded_local(ctx, shards, w.box, w.cutoff, w.skin, K, block)
        del res
    e1.record()
    torch.cuda.synchronize()
    return {"shards": nranks, "atoms_per_shard": [e - s for s, e in bounds],
            "halo_atoms": halos, "halo_fraction": sum(halos) / n, "halo_block": block,
            "ms_all_shards_one_gpu": e0.elapsed_time(e1) / reps}


def run_extras(nl, torch, ctx, ps, pos, w, K, workload: str) -> dict:
    """The rows of the scope table beyond the timed step, each timed on the
    device after the step (outside its timed region): the replayed skin-check
    interval against host-driven steps, nl_build after Hilbert vs Morton
    order (this workload and shell10m, the non-uniform one), the close-pair
    detector, edge features and their CSR form, and the curve-sharded build
    (8 shards on this GPU)."""
    h = ctx.handle
    out = {"interval": interval_timing(nl, torch, h, ps, w, K, w.steps or 200),
           "curves": curve_comparison(nl, torch, h, pos, w, K),
           "close_pairs": close_pair_timing(nl, torch, h, ps, w, K),
           "edge_features": edge_feature_timing(nl, torch, h, ps, w, K),
           "sharded": sharded_timing(torch, ctx, ps, w, K)}
    torch.cuda.empty_cache()
    if workload != "shell10m":
        from neighbor_list_construction_b200 import workloads
        sw = workloads.make("shell10m")
        sctx = nl.Context(sw.n, sw.capacity)
        try:
            spos = torch.from_numpy(sw.pos).cuda()
            c = curve_comparison(nl, torch, sctx.handle, spos, sw, sw.capacity)
            c["workload"] = "shell10m"
            out["curves_shell10m"] = c
            del spos
        finally:
            sctx.close()
            torch.cuda.empty_cache()
    return out


def run_gpu(args, rank: int, world: int, local_rank: int) -> None:
    import torch
    import torch.distributed as dist
    from neighbor_list_construction_b200 import nl, workloads

    # nvidia-smi starts before this process touches the GPU, so its start-up
    # never overlaps a timed region; samples are matched to regions by time.
    clocks = ClockSampler(local_rank)
    clocks.start()
    torch.cuda.set_device(local_rank)
    w = workloads.make(args.workload)
    n, K = w.n, (args.capacity or w.capacity)
    box = w.box
    pos_host = torch.from_numpy(w.pos).pin_memory()
    pos = pos_host.cuda()
    ctx = nl.Context(n, K)
    h = ctx.handle
    perm = torch.empty(n, dtype=torch.int32, device="cuda")
    ps = torch.empty(n, 4, dtype=torch.float32, device="cuda")
    nbr = torch.empty(n, K, dtype=torch.int32, device="cuda")
    cnt = torch.empty(n, dtype=torch.int32, device="cuda")
    rb = torch.zeros(1, dtype=torch.int32, device="cuda")
    cnt_host = torch.empty(n, dtype=torch.int32).pin_memory()
    stream = torch.cuda.current_stream()

    sort_fn = nl.nl_sort_morton if args.curve == "morton" else nl.nl_sort_hilbert

    def step(src):
        sort_fn(h, src, box, perm, ps, None, stream)
        nl.nl_build(h, ps, box, w.cutoff, w.skin, K, nbr, cnt, stream)
        nl.nl_skin_check(h, ps, box, w.skin, rb, None, stream)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def max_over_ranks(x: float) -> float:
        if world == 1:
            return x
        t = torch.tensor([x], dtype=torch.float64, device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    for _ in range(args.warmup):
        step(pos)
    st = ctx.sync_status()
    if st < 0:
        raise RuntimeError(nl.nl_status_string(st))
    info = nl.nl_last_build_info(h)
    pairs = int(cnt.to(torch.int64).sum().item())
    nl.nl_profile_read(h)

    # ---- device-resident timed region
    nl.nl_profile_enable(h, True)
    barrier()
    t_host0 = time.monotonic()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step(pos)
    e1.record(stream)
    barrier()
    clk = clocks.window(t_host0, time.monotonic())
    ms = e0.elapsed_time(e1) / args.steps
    phases = nl.nl_profile_read(h)
    nl.nl_profile_enable(h, False)
    ms_max = max_over_ranks(ms)

    # ---- end to end through the public API with host buffers.  Every step
    # copies its positions in from pinned host memory and its result back to
    # pinned host memory: the padded rows and counts (the reported e2e), or,
    # for comparison, the counts alone.  Pipelined: positions and results
    # double-buffered on the device, one copy stream per direction, so step
    # i's kernels overlap the upload for step i+1 and the download of step
    # i-1.  Serial: copy in, step, copy out on one stream.
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    nbr_host = torch.empty(n, K, dtype=torch.int32).pin_memory()
    pos_buf = [pos, torch.empty_like(pos)]
    cnt_buf = [cnt, torch.empty_like(cnt)]
    nbr_buf = [nbr, torch.empty_like(nbr)]

    def step_into(src, counts, rows):
        sort_fn(h, src, box, perm, ps, None, stream)
        nl.nl_build(h, ps, box, w.cutoff, w.skin, K, rows, counts, stream)
        nl.nl_skin_check(h, ps, box, w.skin, rb, None, stream)

    def e2e_serial(rows: bool) -> float:
        barrier()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.steps):
            pos.copy_(pos_host, non_blocking=True)
            step_into(pos, cnt, nbr)
            cnt_host.copy_(cnt, non_blocking=True)
            if rows:
                nbr_host.copy_(nbr, non_blocking=True)
        f1.record(stream)
        barrier()
        return max_over_ranks(f0.elapsed_time(f1) / args.steps)

    def e2e_pipelined(rows: bool) -> float:
        computed = [torch.cuda.Event(), torch.cuda.Event()]   # step done with buffers b
        uploaded = [torch.cuda.Event(), torch.cuda.Event()]
        downloaded = [torch.cuda.Event(), torch.cuda.Event()]
        barrier()
        g0 = torch.cuda.Event(enable_timing=True)
        g1 = torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        up.wait_event(g0)
        down.wait_event(g0)
        for i in range(args.steps):
            b = i & 1
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(computed[b])
                pos_buf[b].copy_(pos_host, non_blocking=True)
                uploaded[b].record(up)
            stream.wait_event(uploaded[b])
            if i >= 2:
                stream.wait_event(downloaded[b])
            step_into(pos_buf[b], cnt_buf[b], nbr_buf[b])
            computed[b].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(computed[b])
                cnt_host.copy_(cnt_buf[b], non_blocking=True)
                if rows:
                    nbr_host.copy_(nbr_buf[b], non_blocking=True)
                downloaded[b].record(down)
        stream.wait_stream(up)
        stream.wait_stream(down)
        g1.record(stream)
        barrier()
        return max_over_ranks(g0.elapsed_time(g1) / args.steps)

    e2e_ms = e2e_pipelined(True)
    e2e_serial_ms = e2e_serial(True)
    # the host rows are a bit-for-bit copy of the last step's device rows
    rows_ok = bool(torch.equal(nbr_host[:4096], nbr[:4096].cpu()))
    e2e_counts_ms = e2e_pipelined(False)
    e2e_counts_serial_ms = e2e_serial(False)
    del nbr_buf[1], cnt_buf[1], pos_buf[1]
    st = ctx.sync_status()

    if rank == 0:
        peaks = measured_peaks()
        # the pair search of one build: the persistent launch, plus the
        # launches that take the tiles listed by it (no work on saltwater10m)
        pair_ms, pair_launches = phases.get("pair_search", (0.0, 0))
        listed_ms, _ = phases.get("pair_search_listed", (0.0, 0))
        dom = "pair_search"
        dom_ms = (pair_ms + listed_ms) / max(pair_launches, 1)
        bytes_per_atom = 16 + 4 * K + 4
        alg_bytes = n * bytes_per_atom
        achieved = alg_bytes / (dom_ms * 1e-3) / 1e9
        traffic = pair_traffic(args.workload) if K == w.capacity else None
        build_ms = sum(phases.get(p, (0.0, 0))[0] for p in
                       ("bin_count", "cell_scan", "bin_scatter", "cell_sort", "pair_search",
                        "pair_search_listed")) / args.steps
        sort_ms = sum(phases.get(p, (0.0, 0))[0] for p in
                      ("keys", "key_scan", "radix_sort", "gather")) / args.steps
        # launches per profiled phase: the sort phase holds 3 digit passes, the
        # run finish and the gated full sort (keys, scan, 8 passes, gather)
        kernels_per_phase = {"radix_sort": 15}
        launches_per_step = sum(v[1] * kernels_per_phase.get(k, 1)
                                for k, v in phases.items()) / args.steps
        line = {
            "metric": METRIC,
            "value": world * n / (ms_max * 1e-3),
            "unit": "atoms/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_max,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic",
            "config": {"workload": f"{args.workload}: {w.description}", "atoms": n,
                       "cutoff": w.cutoff, "skin": w.skin, "capacity": K,
                       "step": f"nl_sort_{args.curve} + nl_build + nl_skin_check",
                       "cells": info[:3], "staged_pair_kernel": bool(info[3]),
                       "l2": "inputs larger than L2 (positions 165 MB, rows "
                             f"{n * K * 4 / 1e9:.1f} GB per step)",
                       "parallelism": "replicas" if world > 1 else "single"},
            "pairs_per_s": world * pairs / (ms_max * 1e-3),
            "directed_pairs": pairs,
            "build": {"ms": build_ms, "atoms_per_s": n / (build_ms * 1e-3),
                      "pairs_per_s": pairs / (build_ms * 1e-3),
                      "bytes": alg_bytes,
                      "frac_of_8TBs": alg_bytes / (build_ms * 1e-3) / 1e9 / NOMINAL_HBM_GBS,
                      "frac_of_measured": alg_bytes / (build_ms * 1e-3) / 1e9 / peaks["hbm_gbs"]},
            "sort_ms": sort_ms,
            "roofline": {"kernel": dom, "bound": "hbm", "achieved": achieved,
                         "peak": peaks["hbm_gbs"], "peak_source": peaks["source"],
                         "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                         "traffic": traffic,
                         "traffic_over_algorithmic": (traffic / alg_bytes) if traffic else None,
                         "bytes_per_atom": bytes_per_atom, "launch_ms": dom_ms},
            "phases_ms": {k: v[0] / args.steps for k, v in phases.items() if v[1]},
            "e2e": {"value": world * n / (e2e_ms * 1e-3), "unit": "atoms/s",
                    "h2d_bytes_per_step": n * 16, "d2h_bytes_per_step": n * 4 * (K + 1),
                    "result": "padded rows int32[n, K] and counts int32[n] to pinned host "
                              "memory every step",
                    "ms_per_step": e2e_ms, "pipelined": True,
                    "serial_value": world * n / (e2e_serial_ms * 1e-3),
                    "serial_ms_per_step": e2e_serial_ms, "rows_copied_ok": rows_ok,
                    "counts_only": {"value": world * n / (e2e_counts_ms * 1e-3),
                                    "unit": "atoms/s", "h2d_bytes_per_step": n * 16,
                                    "d2h_bytes_per_step": n * 4, "ms_per_step": e2e_counts_ms,
                                    "serial_ms_per_step": e2e_counts_serial_ms,
                                    "result": "counts int32[n] only; the rows stay on the "
                                              "device"}},
            "clocks": clk,
            "gpu_launches": int(round(launches_per_step * args.steps)),
            "status": nl.nl_status_string(st),
        }
        if not args.no_extras and world == 1:
            del nbr_host
            line["extras"] = run_extras(nl, torch, ctx, ps, pos, w, K, args.workload)
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(args.workload, w)
        print(json.dumps(line), flush=True)
    clocks.stop()
    ctx.close()


def run_sharded(args, rank: int, world: int, local_rank: int) -> None:
    """The pages' multi-GPU design (opt-in, --sharded): the whole workload is
    sorted along the curve and cut into `world` equal-count shards, one per
    rank; a timed step is every rank's halo build (coarse-cell marks, an
    all-reduce, counts and atoms by all-to-all, nl_build_rows over own + halo
    atoms, global ids).  Total work is fixed: "scaling": "strong"."""
    import torch
    import torch.distributed as dist
    from neighbor_list_construction_b200 import nl, shard, workloads

    clocks = ClockSampler(local_rank)
    clocks.start()
    torch.cuda.set_device(local_rank)
    w = workloads.make(args.workload)
    n, K = w.n, w.capacity
    bounds = shard.shard_bounds(n, world)
    s0, s1 = bounds[rank]
    ctx = nl.Context(n, K)
    pos = torch.from_numpy(w.pos).cuda()
    perm, ps, _ = ctx.sort(pos, w.box)
    own = shard.with_ids(ps[s0:s1].contiguous(), s0)
    del perm, ps, pos
    comm = shard.DistExchange() if world > 1 else None
    block = [None]   # agreed by the first (warm-up) build, reused after

    def step():
        if comm is not None:
            r = shard.build_sharded(ctx, own, w.box, w.cutoff, w.skin, K, comm, block[0])
        else:
            r = shard.build_sharded_local(ctx, [own], w.box, w.cutoff, w.skin, K, block[0])[0]
        block[0] = r[3]
        return r

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        res = step()
    halo = int(res[2].item())
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_host0 = time.monotonic()
    e0.record()
    for _ in range(args.steps):
        res = step()
    e1.record()
    barrier()
    clk = clocks.window(t_host0, time.monotonic())
    ms = e0.elapsed_time(e1) / args.steps
    if world > 1:
        t = torch.tensor([ms], dtype=torch.float64, device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
        h = torch.tensor([halo], dtype=torch.int64, device="cuda")
        dist.all_reduce(h, op=dist.ReduceOp.SUM)
        halo_total = int(h.item())
    else:
        halo_total = halo
    st = ctx.sync_status()
    if rank == 0:
        line = {
            "metric": METRIC, "value": n / (ms * 1e-3), "unit": "atoms/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": dict(arm_config(args.workload, world),
                           parallelism=f"curve shards x{world}, halo exchange",
                           step="halo build: marks, all-reduce, all-to-all, nl_build_rows"),
            "halo_atoms_total": halo_total, "halo_fraction": halo_total / n,
            "clocks": clk, "status": nl.nl_status_string(st),
        }
        print(json.dumps(line), flush=True)
    clocks.stop()
    del own
    ctx.close()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="saltwater10m")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--curve", default="hilbert", choices=["hilbert", "morton"],
                    help="curve of the sort in the timed step (Morton: the pages' baseline order)")
    ap.add_argument("--sharded", action="store_true",
                    help="time the pages' multi-GPU design instead of replicas: equal-count "
                         "curve shards of the one workload, halo exchange over NCCL")
    ap.add_argument("--capacity", type=int, default=0,
                    help="row capacity K instead of the workload's (for profiling captures that "
                         "must stay small on the device; rows past K only count)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the rows timed after the step (replayed interval vs eager, "
                         "Hilbert vs Morton, close pairs, edge features and CSR, 8 shards)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        if args.sharded:
            run_sharded(args, rank, world, local_rank)
        else:
            run_gpu(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

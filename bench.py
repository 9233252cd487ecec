#!/usr/bin/env python3
"""Benchmark of the multipole-attention decode step on B200.

Workload (default): batch 16, 8 KV / 32 query heads, head_dim 128, 32768 cached
tokens per sequence, token budget 1638 (5% of the context, "95% sparsity"),
seeded Gaussian-mixture keys (1 centroid per 16 tokens, 8K-token clustering
blocks), bf16.  One step = one decode step of one attention layer for the
whole batch: one kernel launch on the bf16 path (centroid scores, selection,
centroid terms, exact rows, combine), four on the multi-kernel path (fp32 and
two-level indexes: centroid pass, selection, token pass, combine).

Reports algorithmic HBM GB/s (the bytes the method must read: all key and value
centroids, the run offsets, the selected clusters' keys and values, the
unclustered tail, Q and O) per device-timed step, with the L2 flushed between
steps.  `--impl reference` times the CPU oracle instead (a bounded sample per
step on the host cores).  N > 1: one process per GPU (torchrun), each decoding
its own batch (weak scaling); time = max over ranks.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode attention µs/step & HBM GB/s (% roofline), B=16, 32K ctx, 95% sparsity"
UNIT = "GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- helpers
def peaks():
    """Measured roofline denominators, else the pool's earlier measurement."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        d["source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["source"] = "fallback"
    return d


def aggregate(local_value_sum, local_time, dist=None):
    """(sum over ranks of the work, max over ranks of the time)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return local_value_sum, local_time
    import torch
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    w = torch.tensor([float(local_value_sum)], dtype=torch.float64, device=dev)
    t = torch.tensor([float(local_time)], dtype=torch.float64, device=dev)
    dist.all_reduce(w, op=dist.ReduceOp.SUM)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return w.item(), t.item()


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms in the background."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def algorithmic_bytes_unit(w, C, n_sel_tokens, n_tail):
    """Bytes one (batch, KV head) step must read or write (bf16 elements of 2 bytes):
    all key and value centroids, the run offsets, the selected tokens' keys and
    values, the tail's keys and values, the group's queries and outputs."""
    e = 2 if w["dtype"] == "bf16" else 4
    d, G = w["d"], w["Hq"] // w["Hkv"]
    return 2 * C * d * e + (C + 1) * 4 + 2 * (n_sel_tokens + n_tail) * d * e + 2 * G * d * e


# ----------------------------------------------------------------------------- CPU oracle arm
def oracle_units(w, k, seed):
    """k (batch, KV head) units of the workload with oracle indices.

    Clusters are the mixture components of each 8K block (a stand-in for the
    k-means result: the decode cost does not depend on how clusters were found).
    """
    from clustered_sparse_decode_b200 import synth
    from oracle import multipole as mp
    rng = np.random.default_rng(seed)
    n, d, G = w["n"], w["d"], w["Hq"] // w["Hkv"]
    o = dict(B=1, Hkv=1, Hq=G, d=d, n_max=n, T=w["T"], L_blk=w["L_blk"], levels=1, Tc=w.get("Tc", 128),
             iters=w["iters"], update_interval=w.get("update_interval", 1024), dtype=w["dtype"], seed=0)
    units = []
    for _ in range(k):
        K, V, lab = synth.make_cache(1, 1, n, d, w["comps"], w["sigma"], radius=w["radius"],
                                     outliers=w["outliers"], dtype=w["dtype"], seed=int(rng.integers(1 << 30)))
        a = synth.component_assignment(lab, n, w["L_blk"], w["T"])
        idx = mp.index_from_assignment(K, V, n, o, a)
        units.append((idx, int(np.count_nonzero(np.diff(idx["off"][0, 0])))))
    return units


def time_oracle(w, units, seconds, seed):
    """Time the oracle's decode over the units, fresh queries each, until `seconds` of decode time.

    Returns (algorithmic bytes, decode seconds, unit-steps)."""
    from clustered_sparse_decode_b200 import synth
    from oracle import multipole as mp
    rng = np.random.default_rng(seed)
    d, G = w["d"], w["Hq"] // w["Hkv"]
    tot_bytes, tot_time, pairs = 0, 0.0, 0
    while tot_time < seconds:
        idx, C = units[pairs % len(units)]
        Q = synth.make_queries(1, 1, G, d, w["dtype"], seed=int(rng.integers(1 << 30)))[0]
        info = {}
        t0 = time.perf_counter()
        mp.decode(idx, Q, w["budget"], info=info)
        tot_time += time.perf_counter() - t0
        nsel = int(np.sum(np.diff(idx["off"][0, 0])[info[(0, 0)]["sel"]]))
        tot_bytes += algorithmic_bytes_unit(w, C, nsel, 0)
        pairs += 1
    return tot_bytes, tot_time, pairs


# One oracle worker process per host core: each builds its own (batch, KV head)
# units once and then times the oracle's decode over them, numpy limited to one
# thread per process so that the workers do not oversubscribe the cores.
_WORKER_UNITS = None


def _oracle_worker_init(w, seed):
    global _WORKER_UNITS
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except ImportError:
        pass
    _WORKER_UNITS = oracle_units(w, 2, seed=seed)


def _oracle_worker_step(job):
    w, seconds, seed = job
    return time_oracle(w, _WORKER_UNITS, seconds, seed)


class OraclePool:
    """The oracle's decode timed on the host cores: one spawned process per core
    (at most `max_workers`), all timing the same workload in parallel."""

    def __init__(self, w, max_workers=32):
        import multiprocessing as mpr
        from concurrent.futures import ProcessPoolExecutor
        self.w = w
        self.host_cores = len(os.sched_getaffinity(0))
        self.workers = max(1, min(self.host_cores, max_workers))
        # spawn: no forked copy of a process that may hold a CUDA context
        self.pool = ProcessPoolExecutor(self.workers, mp_context=mpr.get_context("spawn"),
                                        initializer=_oracle_worker_init, initargs=(w, 1))

    def step(self, seconds, seed):
        """All workers time `seconds` of decodes in parallel.  Returns (bytes, wall seconds, unit-steps)."""
        jobs = [(self.w, seconds, seed + 7919 * i) for i in range(self.workers)]
        list(self.pool.map(_oracle_worker_step, [(self.w, 0.0, 0)] * self.workers))   # workers ready
        t0 = time.perf_counter()
        res = list(self.pool.map(_oracle_worker_step, jobs))
        wall = time.perf_counter() - t0
        return sum(r[0] for r in res), wall, sum(r[2] for r in res)

    def close(self):
        self.pool.shutdown()


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    units = w["B"] * w["Hkv"]
    pool = OraclePool(w)
    per_step = []
    tot_b = tot_t = 0.0
    pairs = 0
    for s in range(args.warmup + args.steps):
        b, t, p = pool.step(args.ref_seconds_per_step, seed=1000 + s)
        if s >= args.warmup:
            tot_b, tot_t, pairs = tot_b + b, tot_t + t, pairs + p
            per_step.append(t / p * units)          # seconds for all units of one step
    pool.close()
    gbs = tot_b / tot_t / 1e9
    ms = 1e3 * statistics.mean(per_step)
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(w, args),
        "cpu_baseline": {"kind": "oracle", "cores": pool.workers, "host_cores": pool.host_cores, "value": gbs,
                         "unit": UNIT,
                         "sample": f"{pairs} (batch, KV head) decode steps of the workload over {pool.workers} "
                                   f"processes, ~{args.ref_seconds_per_step:.0f} s per step, extrapolated to "
                                   f"{units} heads x batch per step"},
        "e2e": {"value": gbs, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_dict(w, args):
    return {"workload": args.workload, "batch": w["B"], "kv_heads": w["Hkv"], "q_heads": w["Hq"],
            "head_dim": w["d"], "context": w["n"], "budget": w["budget"], "tokens_per_centroid": w["T"],
            "block_tokens": w["L_blk"], "levels": w.get("levels", 1), "kmeans_iters": w["iters"],
            "l2": "flushed between timed steps (2x L2 written, then 2x L2 read: cold and clean)", "parallelism": f"dp{args.gpus} (independent batches)"}


# ----------------------------------------------------------------------------- GPU arm
def run_ours(args, w):
    import torch
    import torch.distributed as dist

    from clustered_sparse_decode_b200 import Config, MultipoleIndex, synth
    from clustered_sparse_decode_b200 import build as libbuild

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    libbuild.build()
    dev = torch.device("cuda", local)
    B, Hkv, Hq, d, n = w["B"], w["Hkv"], w["Hq"], w["d"], w["n"]
    tdt = torch.bfloat16 if w["dtype"] == "bf16" else torch.float32

    # inputs: seeded synthetic caches (distinct per rank), clustered on the GPU
    K, V, _ = synth.make_cache(B, Hkv, n, d, w["comps"], w["sigma"], radius=w["radius"], outliers=w["outliers"],
                               dtype=w["dtype"], seed=w["seed"] + 100 * rank)
    Kd = torch.from_numpy(K).to(dev).to(tdt)
    Vd = torch.from_numpy(V).to(dev).to(tdt)
    del K, V
    cfg = Config(batch=B, kv_heads=Hkv, q_heads=Hq, head_dim=d, max_tokens=n, tokens_per_centroid=w["T"],
                 block_tokens=w["L_blk"], levels=w.get("levels", 1), coarse_tokens_per_centroid=w.get("Tc", 128),
                 kmeans_iters=w["iters"], dtype=w["dtype"], seed=w["seed"])
    idx = MultipoleIndex(cfg, device=dev)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    idx.build(Kd, Vd)
    torch.cuda.synchronize()
    build_s = time.perf_counter() - t0
    if idx.check_device_error() != 0:
        raise RuntimeError("device error after build")
    kassign = time_assign(idx, Kd, w, args) if not args.no_assign else None
    if args.no_extras or world > 1:
        del Kd, Vd
        Kd = Vd = None
    nq = args.warmup + args.steps
    Qh = synth.make_queries(nq, B, Hq, d, w["dtype"], seed=w["seed"] + 7 + 100 * rank)
    Q = torch.from_numpy(Qh).to(dev).to(tdt)
    O = torch.empty((B, Hq, d), dtype=tdt, device=dev)
    budget = w["budget"]
    cb = w.get("coarse_budget", 0)

    # algorithmic bytes of each timed step, from its actual selection (untimed pass)
    off = idx.arrays()["off"]
    cnt = (off[:, :, 1:] - off[:, :, :-1]).to(torch.int64)
    C_unit = (cnt > 0).sum(dim=2)                                     # [B, Hkv]
    mask = torch.zeros((B, Hkv, idx.slots), dtype=torch.uint8, device=dev)
    step_bytes = []
    for s in range(args.warmup, nq):
        idx.decode(Q[s], budget, coarse_budget=cb, out=O, sel_mask=mask)
        nsel = (cnt * mask.to(torch.int64)).sum(dim=2)                # [B, Hkv]
        tot = 0
        for b in range(B):
            for h in range(Hkv):
                tot += algorithmic_bytes_unit(w, int(C_unit[b, h]), int(nsel[b, h]), 0)
        step_bytes.append(tot)
    sel_tokens_mean = float(nsel.float().mean())

    # L2 flush buffer and per-step / per-phase events
    l2 = getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 126 << 20) or (126 << 20)
    flush_w = torch.empty(2 * l2, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(2 * l2, dtype=torch.uint8, device=dev)

    def flush_l2():
        # write 2x L2 (evicts the index), then read another 2x L2 so that the
        # written lines are back in HBM before the step starts: the step sees
        # a cold L2 and no write-back of the flush inside its timed region
        flush_w.zero_()
        flush_r.amax()
    names = idx.decode_phases()
    n_ph = len(names) + 1
    stream = torch.cuda.current_stream()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ph)] for _ in range(args.steps)]
    for row in ev:
        for e in row:
            e.record(stream)
    for s in range(args.warmup):
        flush_l2()
        idx.decode(Q[s], budget, coarse_budget=cb, out=O)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    for i in range(args.steps):
        flush_l2()
        idx.decode(Q[args.warmup + i], budget, coarse_budget=cb, out=O, phase_events=ev[i])
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop()
    step_ms = [ev[i][0].elapsed_time(ev[i][-1]) for i in range(args.steps)]
    phase_ms = [statistics.mean(ev[i][p].elapsed_time(ev[i][p + 1]) for i in range(args.steps))
                for p in range(n_ph - 1)]
    local_time = sum(step_ms) / 1e3
    local_bytes = sum(step_bytes)
    tot_bytes, tot_time = aggregate(local_bytes, local_time, dist)
    gbs = tot_bytes / tot_time / 1e9
    ms_per_step = 1e3 * tot_time / args.steps

    # end to end through the C ABI with host buffers: each step's Q is read from
    # pinned host memory (by the library's staging kernel) and O is written back
    # to pinned host memory (by the decode's combine), and the host waits for it
    Qpin = torch.from_numpy(Qh).to(tdt).pin_memory() if w["dtype"] == "bf16" else torch.from_numpy(Qh).pin_memory()
    Opin = torch.empty((B, Hq, d), dtype=tdt).pin_memory()
    e2e_ms = []
    for i in range(args.warmup + args.steps):
        flush_l2()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        idx.decode(Qpin[i], budget, coarse_budget=cb, out=Opin)
        b_.record(stream)
        b_.synchronize()
        if i >= args.warmup:
            e2e_ms.append(a.elapsed_time(b_))
    e2e_bytes, e2e_time = aggregate(local_bytes, sum(e2e_ms) / 1e3, dist)
    qbytes = B * Hq * d * (2 if w["dtype"] == "bf16" else 4)

    # roofline of the dominant kernel
    pk = peaks()
    dom = int(np.argmax(phase_ms))
    e = 2 if w["dtype"] == "bf16" else 4
    C_tot = int(C_unit.sum())
    sel_tot = sum(step_bytes) / len(step_bytes)
    phase_alg = {
        "decode": sel_tot,
        "centroid pass": 2 * C_tot * d * e + (idx.slots + 1) * 4 * B * Hkv,
        "token pass": sel_tot - (2 * C_tot * d * e + (idx.slots + 1) * 4 * B * Hkv) - 2 * B * Hq * d * e,
    }
    dom_name = names[dom]
    dom_bytes = phase_alg.get(dom_name)
    roof = None
    if dom_bytes is not None:
        ach = dom_bytes / (phase_ms[dom] / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": ach / pk["hbm_gbs"], "traffic": traffic_for(dom_name, args.workload),
                "kernel": dom_name, "peak_source": pk["source"]}

    extras = None
    if rank == 0 and world == 1 and not args.no_extras:
        extras = run_extras(args, w, dev, cfg, Kd, Vd, Qh, 1e3 * ms_per_step)
        del Kd, Vd

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        pool = OraclePool(w)
        b_, t_, p_ = pool.step(args.cpu_seconds, seed=99)
        pool.close()
        cpu = {"value": b_ / t_ / 1e9, "unit": UNIT, "cores": pool.workers, "host_cores": pool.host_cores,
               "kind": "oracle",
               "sample": f"{p_} (batch, KV head) decode steps of the workload, {pool.workers} processes in "
                         f"parallel for ~{args.cpu_seconds:.0f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": gbs, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w["dtype"], "data": "synthetic",
            "config": config_dict(w, args),
            "us_per_step": 1e3 * ms_per_step, "tokens_per_s": w["B"] * world * args.steps / tot_time,
            "pct_hbm_roofline": gbs / world / pk["hbm_gbs"],
            "roofline": roof,
            "phases_ms": dict(zip(names, phase_ms)),
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_bytes / e2e_time / 1e9, "unit": UNIT, "h2d_bytes_per_step": qbytes,
                    "d2h_bytes_per_step": qbytes},
            "gpu_launches": args.steps * len(names),
            "clocks": clk,
            "build_s": build_s,
            "kmeans_assign": kassign,
            "selected_tokens_per_head": sel_tokens_mean,
            "extra_configs": extras,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ----------------------------------------------------------------------------- other configurations
def make_flusher(dev):
    """write 2x L2, then read another 2x L2: the next step starts from a cold, clean L2"""
    import torch
    l2 = getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 126 << 20) or (126 << 20)
    fw = torch.empty(2 * l2, dtype=torch.uint8, device=dev)
    fr = torch.ones(2 * l2, dtype=torch.uint8, device=dev)

    def flush():
        fw.zero_()
        fr.amax()
    return flush


def time_steps(fn, steps, warmup, flush):
    """Device time (ms) of `steps` calls fn(i) after `warmup` untimed ones, L2 flushed before each
    (outside the events), CUDA events on the launching stream."""
    import torch
    stream = torch.cuda.current_stream()
    for i in range(warmup):
        flush()
        fn(i)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush()
        ev[i][0].record(stream)
        fn(warmup + i)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def hier_bytes_unit(w, cc_nonempty, n_cand, n_sel_tokens):
    """Bytes one two-level (batch, KV head) step must read or write: every coarse key and value
    centroid and coarse range, the key and value centroids and offsets of the fine clusters inside
    the selected coarse clusters, the selected tokens' keys and values, Q and O."""
    e = 2 if w["dtype"] == "bf16" else 4
    d, G = w["d"], w["Hq"] // w["Hkv"]
    return (2 * cc_nonempty * d * e + (cc_nonempty + 1) * 4 + 2 * n_cand * d * e + (n_cand + 1) * 4
            + 2 * n_sel_tokens * d * e + 2 * G * d * e)


def run_extra_decode(name, args, dev, pk, flush):
    """Decode µs/step of another configuration (its own cache, build and queries)."""
    import torch
    from clustered_sparse_decode_b200 import Config, MultipoleIndex, synth
    w = synth.workload(name)
    B, Hkv, Hq, d, n = w["B"], w["Hkv"], w["Hq"], w["d"], w["n"]
    tdt = torch.bfloat16 if w["dtype"] == "bf16" else torch.float32
    K, V, _ = synth.make_cache(B, Hkv, n, d, w["comps"], w["sigma"], radius=w["radius"], outliers=w["outliers"],
                               dtype=w["dtype"], seed=w["seed"])
    Kd, Vd = torch.from_numpy(K).to(dev).to(tdt), torch.from_numpy(V).to(dev).to(tdt)
    del K, V
    levels = w.get("levels", 1)
    cfg = Config(batch=B, kv_heads=Hkv, q_heads=Hq, head_dim=d, max_tokens=n, tokens_per_centroid=w["T"],
                 block_tokens=w["L_blk"], levels=levels, coarse_tokens_per_centroid=w.get("Tc", 128),
                 kmeans_iters=w["iters"], dtype=w["dtype"], seed=w["seed"])
    idx = MultipoleIndex(cfg, device=dev)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    idx.build(Kd, Vd)
    torch.cuda.synchronize()
    build_s = time.perf_counter() - t0
    del Kd, Vd
    if idx.check_device_error() != 0:
        raise RuntimeError(f"device error after the {name} build")
    steps = min(args.steps, 20)
    Qh = synth.make_queries(args.warmup + steps, B, Hq, d, w["dtype"], seed=w["seed"] + 7)
    Q = torch.from_numpy(Qh).to(dev).to(tdt)
    O = torch.empty((B, Hq, d), dtype=tdt, device=dev)
    budget, cb = w["budget"], w.get("coarse_budget", 0)
    # algorithmic bytes of every timed step, from its own selection (untimed pass)
    arr = idx.arrays()
    off = arr["off"].to(torch.int64)
    cnt = off[:, :, 1:] - off[:, :, :-1]
    mask = torch.zeros((B, Hkv, idx.slots), dtype=torch.uint8, device=dev)
    cmask = torch.zeros((B, Hkv, max(idx.coarse_slots, 1)), dtype=torch.uint8, device=dev) if levels == 2 else None
    step_bytes = []
    for i in range(args.warmup, args.warmup + steps):
        idx.decode(Q[i], budget, coarse_budget=cb, out=O, sel_mask=mask, coarse_sel_mask=cmask)
        nsel = (cnt * mask.to(torch.int64)).sum(dim=2)
        tot = 0
        if levels == 1:
            C_unit = (cnt > 0).sum(dim=2)
            for b in range(B):
                for h in range(Hkv):
                    tot += algorithmic_bytes_unit(w, int(C_unit[b, h]), int(nsel[b, h]), 0)
        else:
            coff = arr["coff"].to(torch.int64)
            ccnt = off.gather(2, coff[:, :, 1:]) - off.gather(2, coff[:, :, :-1])
            cc_ne = (ccnt > 0).sum(dim=2)
            for b in range(B):
                for h in range(Hkv):
                    cand = 0
                    for c in torch.nonzero(cmask[b, h]).flatten().tolist():
                        r0, r1 = int(coff[b, h, c]), int(coff[b, h, c + 1])
                        cand += int((cnt[b, h, r0:r1] > 0).sum())
                    tot += hier_bytes_unit(w, int(cc_ne[b, h]), cand, int(nsel[b, h]))
        step_bytes.append(tot)
    clocks = ClockSampler(dev.index or 0)
    clocks.start()
    time.sleep(0.3)
    ms = time_steps(lambda i: idx.decode(Q[i], budget, coarse_budget=cb, out=O), steps, args.warmup, flush)
    clk = clocks.stop()
    if idx.check_device_error() != 0:
        raise RuntimeError(f"device error in the {name} decode")
    us = 1e3 * statistics.mean(ms)
    gbs = sum(step_bytes) / (sum(ms) / 1e3) / 1e9
    return {"us_per_step": us, "gb_s": gbs, "frac_hbm": gbs / pk["hbm_gbs"], "tokens_per_s": B * 1e6 / us,
            "bytes_per_step": statistics.mean(step_bytes), "build_s": build_s, "steps": steps,
            "budget": budget, "coarse_budget": cb if levels == 2 else None, "clocks": clk,
            "config": {"batch": B, "kv_heads": Hkv, "q_heads": Hq, "head_dim": d, "context": n, "levels": levels}}


def run_extras(args, w, dev, cfg, Kd, Vd, Qh, us_headline):
    """The other configurations, each with its own clock record: the dense decode baseline on the
    headline's cache, single-sequence 32K, two-level 64K, and the online workload."""
    import torch
    from clustered_sparse_decode_b200 import dense_decode
    pk = peaks()
    flush = make_flusher(dev)
    out = {}
    # dense baseline: every key of the same cache, exact (a FlashDecoding-style split-KV decode)
    tdt = torch.bfloat16 if w["dtype"] == "bf16" else torch.float32
    Q = torch.from_numpy(Qh).to(dev).to(tdt)
    O = torch.empty_like(Q[0])
    steps = min(args.steps, 20)
    clocks = ClockSampler(dev.index or 0)
    clocks.start()
    time.sleep(0.3)
    ms = time_steps(lambda i: dense_decode(cfg, Kd, Vd, w["n"], Q[i % Q.shape[0]], out=O), steps, args.warmup, flush)
    clk = clocks.stop()
    e = 2 if w["dtype"] == "bf16" else 4
    dense_bytes = w["B"] * w["Hkv"] * w["n"] * w["d"] * 2 * e + 2 * w["B"] * w["Hq"] * w["d"] * e
    us = 1e3 * statistics.mean(ms)
    gbs = dense_bytes / (us / 1e6) / 1e9
    out["dense_baseline"] = {"us_per_step": us, "gb_s": gbs, "frac_hbm": gbs / pk["hbm_gbs"],
                             "bytes_per_step": dense_bytes, "multipole_speedup": us / us_headline, "clocks": clk,
                             "what": "exact attention over all keys of the same cache (mp_dense_decode)"}
    del Q, O
    for name in ("single_bf16", "hier_64k"):
        out[name] = run_extra_decode(name, args, dev, pk, flush)
    ow = synth_workload("online_16k_plus_16k")
    out["online_16k_plus_16k"] = online_measure(args, ow, dev, 0, 1, None)
    return out


def synth_workload(name):
    from clustered_sparse_decode_b200 import synth
    return synth.workload(name)


def run_online(args, w):
    """Online workload: build on the prompt, then per generated token append it
    (mp_cluster_update: re-clusters the open block every update_interval tokens or
    at a block end) and decode one step.  Reports decode plus amortised update
    time per generated token, device-timed (CUDA events around each call, L2
    flushed between tokens outside the events)."""
    import torch
    import torch.distributed as dist

    from clustered_sparse_decode_b200 import build as libbuild

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local))
    libbuild.build()
    dev = torch.device("cuda", local)
    r = online_measure(args, w, dev, rank, world, dist if world > 1 else None)
    if rank == 0:
        line = {
            "metric": "online decode + amortised cluster update, us per generated token", "value": r["us_per_token"],
            "unit": "us/token", "n_gpus": world, "steps": r["generated"], "warmup": args.warmup,
            "ms_per_step": r["us_per_token"] / 1e3, "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": w["dtype"], "data": "synthetic",
            "config": {"workload": args.workload, "batch": w["B"], "kv_heads": w["Hkv"], "q_heads": w["Hq"],
                       "head_dim": w["d"], "prompt": w["n"], "generated": r["generated"], "budget": w["budget"],
                       "block_tokens": w["L_blk"], "update_interval": w["update_interval"],
                       "kmeans_iters": w["iters"],
                       "l2": "flushed before every generated token (2x L2 written, then 2x L2 read)",
                       "parallelism": f"dp{world} (independent batches)"},
        }
        line.update({k: v for k, v in r.items() if k not in ("generated",)})
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def online_measure(args, w, dev, rank, world, dist):
    """Per generated token: mp_cluster_update (append; re-cluster the open block on a
    trigger) and one decode step, each bracketed by CUDA events, L2 flushed before each
    token outside the events.  Returns the per-token times (max over ranks)."""
    import torch

    from clustered_sparse_decode_b200 import Config, MultipoleIndex, synth
    B, Hkv, Hq, d, n0, ng = w["B"], w["Hkv"], w["Hq"], w["d"], w["n"], w["n_gen"]
    if args.gen_tokens > 0:
        ng = min(ng, args.gen_tokens)
    tdt = torch.bfloat16 if w["dtype"] == "bf16" else torch.float32
    K, V, _ = synth.make_cache(B, Hkv, n0 + ng, d, w["comps"], w["sigma"], radius=w["radius"], outliers=w["outliers"],
                               dtype=w["dtype"], seed=w["seed"] + 100 * rank, drift=w.get("drift"))
    Kd = torch.from_numpy(K).to(dev).to(tdt)
    Vd = torch.from_numpy(V).to(dev).to(tdt)
    del K, V
    Kgen = Kd[:, :, n0:].permute(2, 0, 1, 3).contiguous()   # [ng, B, Hkv, d]: token t's rows contiguous
    Vgen = Vd[:, :, n0:].permute(2, 0, 1, 3).contiguous()
    cfg = Config(batch=B, kv_heads=Hkv, q_heads=Hq, head_dim=d, max_tokens=n0 + ng, tokens_per_centroid=w["T"],
                 block_tokens=w["L_blk"], kmeans_iters=w["iters"], update_interval=w["update_interval"],
                 dtype=w["dtype"], seed=w["seed"])
    idx = MultipoleIndex(cfg, device=dev)
    idx.build(Kd[:, :, :n0].contiguous(), Vd[:, :, :n0].contiguous())
    del Kd, Vd
    torch.cuda.synchronize()
    Qh = synth.make_queries(args.warmup + ng, B, Hq, d, w["dtype"], seed=w["seed"] + 7 + 100 * rank)
    Q = torch.from_numpy(Qh).to(dev).to(tdt)
    O = torch.empty((B, Hq, d), dtype=tdt, device=dev)
    flush = make_flusher(dev)
    stream = torch.cuda.current_stream()
    for s in range(args.warmup):
        flush()
        idx.decode(Q[s], w["budget"], out=O)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(dev.index or 0)
    clocks.start()
    time.sleep(0.3)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(ng)]
    fired = []
    for t in range(ng):
        flush()
        e = ev[t]
        e[0].record(stream)
        fired.append(idx.update(Kgen[t].unsqueeze(2), Vgen[t].unsqueeze(2)))
        e[1].record(stream)
        idx.decode(Q[args.warmup + t], w["budget"], out=O)
        e[2].record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop()
    if idx.check_device_error() != 0:
        raise RuntimeError("device error in the online run")
    upd = [ev[t][0].elapsed_time(ev[t][1]) for t in range(ng)]
    upd_ms = sum(upd)
    n_fired = sum(fired)
    fired_ms = sum(u for u, f in zip(upd, fired) if f)
    dec_ms = sum(ev[t][1].elapsed_time(ev[t][2]) for t in range(ng))
    tot_tokens, tot_s = aggregate(B * ng, (upd_ms + dec_ms) / 1e3, dist)
    return {"us_per_token": 1e6 * tot_s / ng, "generated": ng,
            "decode_us_per_token": 1e3 * dec_ms / ng, "update_us_per_token": 1e3 * upd_ms / ng,
            "reclusterings": n_fired, "recluster_ms_each": fired_ms / max(n_fired, 1),
            "append_us_each": 1e3 * (upd_ms - fired_ms) / max(ng - n_fired, 1), "tokens_per_s": tot_tokens / tot_s,
            "clocks": clk}


def assign_flops(w):
    """Algorithmic flops of one assignment step: 2 L_j C_j d per (unit, block), C_j = ceil(L_j / T)."""
    n, Lb, T, d = w["n"], w["L_blk"], w["T"], w["d"]
    f = 0
    for j in range(-(-n // Lb)):
        L = min(n, (j + 1) * Lb) - j * Lb
        f += 2 * L * (-(-L // T)) * d
    return f * w["B"] * w["Hkv"]


def time_assign(idx, Kd, w, args, reps=5, warm=3):
    """One k-means assignment step over the whole index (one launch), CUDA events on the launching stream.

    The keys (B x Hkv x n x d) are far larger than L2, so each step streams them from HBM.
    """
    import torch
    out = torch.empty((w["B"], w["Hkv"], idx.n_clustered), dtype=torch.int32, device=Kd.device)
    stream = torch.cuda.current_stream()
    for _ in range(warm):
        idx.assign(Kd, out=out)
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
    ev[0].record(stream)
    for i in range(reps):
        idx.assign(Kd, out=out)
        ev[i + 1].record(stream)
    torch.cuda.synchronize()
    ms = statistics.median(ev[i].elapsed_time(ev[i + 1]) for i in range(reps))
    if idx.check_device_error() != 0:
        raise RuntimeError("device error after assignment")
    flops = assign_flops(w)
    pk = peaks()
    tf = flops / (ms / 1e3) / 1e12
    return {"ms": ms, "flops_per_launch": flops, "tflops": tf, "bound": "tensor",
            "peak": pk["bf16_tflops"], "frac": tf / pk["bf16_tflops"],
            "frac_sustained": tf / pk.get("bf16_tflops_sustained", pk["bf16_tflops"]),
            "peak_source": pk["source"], "dtype": w["dtype"]}


def traffic_for(kernel, workload):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if current."""
    p = os.path.join(ROOT, "profiles", "traffic.md")
    if not os.path.exists(p):
        return None
    for line in open(p):
        parts = [x.strip() for x in line.strip().strip("|").split("|")]
        if len(parts) >= 4 and parts[0] == kernel and parts[1] == workload:
            try:
                if parts[3] != source_digest(kernel):
                    return None
                return float(parts[2])
            except ValueError:
                return None
    return None


# the sources of each kernel whose traffic profiles/traffic.md records
KERNEL_SOURCES = {"decode": ("decode_unit.cu", "stream_common.cuh", "mp_internal.cuh")}


def source_digest(kernel=None):
    """sha256 prefix of the kernel's source files (all of csrc/ for an unlisted kernel)."""
    import hashlib
    csrc = os.path.join(ROOT, "clustered_sparse_decode_b200", "csrc")
    files = KERNEL_SOURCES.get(kernel) or sorted(os.listdir(csrc))
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:12]


SWEEP_T = (8, 16, 32, 64, 128)
SWEEP_BLOCK = (2048, 4096, 8192, 16384)


def run_sweep(args):
    """The ablation knobs of the pages as a speed sweep (NEXT-2): tokens per centroid T x
    clustering block size, on one seeded batch-4 (or, with --sweep-batch 16, the bench's batch-16)
    32K-token cache (the bench's key and value distribution) with the bench's 5% budget.  Each configuration builds its own index (timed)
    and decodes `steps` queries with the L2 flushed before each (CUDA events).  Prints one JSON
    line; with --sweep-out also writes the table as markdown."""
    import torch
    from clustered_sparse_decode_b200 import Config, MultipoleIndex, synth
    from clustered_sparse_decode_b200 import build as libbuild
    libbuild.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(0)
    base = synth.workload("batch4_32k_sparse95" if args.sweep_batch == 4 else "batch16_32k_sparse95")
    B, Hkv, Hq, d, n = base["B"], base["Hkv"], base["Hq"], base["d"], base["n"]
    K, V, _ = synth.make_cache(B, Hkv, n, d, base["comps"], base["sigma"], radius=base["radius"],
                               outliers=base["outliers"], dtype="bf16", seed=base["seed"])
    Kd = torch.from_numpy(K).to(dev).to(torch.bfloat16)
    Vd = torch.from_numpy(V).to(dev).to(torch.bfloat16)
    del K, V
    steps = min(args.steps, 20)
    Q = torch.from_numpy(synth.make_queries(args.warmup + steps, B, Hq, d, "bf16", seed=base["seed"] + 7)) \
        .to(dev).to(torch.bfloat16)
    O = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=dev)
    pk = peaks()
    flush = make_flusher(dev)
    budget = base["budget"]
    clocks = ClockSampler(0)
    clocks.start()
    rows = []
    for T in SWEEP_T:
        for L in SWEEP_BLOCK:
            w = dict(base, T=T, L_blk=L)
            cfg = Config(batch=B, kv_heads=Hkv, q_heads=Hq, head_dim=d, max_tokens=n, tokens_per_centroid=T,
                         block_tokens=L, kmeans_iters=base["iters"], dtype="bf16", seed=base["seed"])
            idx = MultipoleIndex(cfg, device=dev)
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            idx.build(Kd, Vd)
            torch.cuda.synchronize()
            build_s = time.perf_counter() - t0
            if idx.check_device_error() != 0:
                raise RuntimeError(f"device error after the T={T}, block={L} build")
            # algorithmic bytes from each timed step's own selection (untimed pass)
            off = idx.arrays()["off"].to(torch.int64)
            cnt = off[:, :, 1:] - off[:, :, :-1]
            C_unit = (cnt > 0).sum(dim=2)
            mask = torch.zeros((B, Hkv, idx.slots), dtype=torch.uint8, device=dev)
            step_bytes, sel_tokens = [], []
            for i in range(args.warmup, args.warmup + steps):
                idx.decode(Q[i], budget, out=O, sel_mask=mask)
                nsel = (cnt * mask.to(torch.int64)).sum(dim=2)
                sel_tokens.append(float(nsel.to(torch.float64).mean()))
                step_bytes.append(sum(algorithmic_bytes_unit(w, int(C_unit[b, h]), int(nsel[b, h]), 0)
                                      for b in range(B) for h in range(Hkv)))
            ms = time_steps(lambda i: idx.decode(Q[i], budget, out=O), steps, args.warmup, flush)
            if idx.check_device_error() != 0:
                raise RuntimeError(f"device error in the T={T}, block={L} decode")
            us = 1e3 * statistics.mean(ms)
            gbs = sum(step_bytes) / (sum(ms) / 1e3) / 1e9
            rows.append({"T": T, "block_tokens": L, "slots_per_head": idx.slots, "us_per_step": us, "gb_s": gbs,
                         "frac_hbm": gbs / pk["hbm_gbs"], "bytes_per_step": statistics.mean(step_bytes),
                         "selected_tokens_per_head": statistics.mean(sel_tokens), "build_s": build_s})
            del idx
            torch.cuda.empty_cache()
    clk = clocks.stop()
    head = next(r for r in rows if r["T"] == 16 and r["block_tokens"] == 8192)
    line = {"metric": f"decode µs/step and build s per (tokens per centroid, block size), B={B}, 32K ctx, 5% budget",
            "value": head["gb_s"], "unit": "GB/s", "n_gpus": 1, "steps": steps, "warmup": args.warmup,
            "ms_per_step": head["us_per_step"] / 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"sweep (batch{B}_32k_sparse95 cache; T x block)", "batch": B, "kv_heads": Hkv,
                       "q_heads": Hq, "head_dim": d, "context": n, "budget": budget,
                       "l2": "flushed between timed steps (2x L2 written, then 2x L2 read: cold and clean)"},
            "clocks": clk, "sweep": rows}
    print(json.dumps(line), flush=True)
    if args.sweep_out:
        with open(args.sweep_out, "w") as f:
            f.write("| T (tokens per centroid) | block tokens | slots per head | µs/step | GB/s | % of HBM | "
                    "selected tokens per head | build s |\n|---|---|---|---|---|---|---|---|\n")
            for r in rows:
                f.write(f"| {r['T']} | {r['block_tokens']} | {r['slots_per_head']} | {r['us_per_step']:.1f} | "
                        f"{r['gb_s']:.0f} | {100 * r['frac_hbm']:.1f}% | {r['selected_tokens_per_head']:.0f} | "
                        f"{r['build_s']:.3f} |\n")
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="batch16_32k_sparse95")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-seconds-per-step", type=float, default=1.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-assign", action="store_true", help="skip the timed k-means assignment step")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the other configurations (dense baseline, single sequence, two-level, online)")
    ap.add_argument("--gen-tokens", type=int, default=0,
                    help="online workloads: generated tokens to time (0 = all of the workload's)")
    ap.add_argument("--sweep-out", default=None, help="--workload sweep: also write the table as markdown here")
    ap.add_argument("--sweep-batch", type=int, choices=[4, 16], default=4,
                    help="--workload sweep: the cache's batch (4, or 16 = the bench geometry)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.workload == "sweep":
        if args.impl == "reference" or args.gpus != 1:
            ap.error("--workload sweep runs our implementation on one GPU")
        return run_sweep(args)
    from clustered_sparse_decode_b200 import synth
    w = synth.workload(args.workload)
    if args.impl == "reference":
        return run_reference(args, w)
    if "n_gen" in w:
        return run_online(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())

"""Benchmark of the streaming top-k indexer step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload long] [--no-e2e] [--no-cpu-baseline]
    python bench.py --sweep k|s [--workload v4flash] [--sweep-values ...]

A step is one si_indexer_topk call over one batch of synthetic inputs: the
fused scoring, selection and row-sort kernel, with q, w, kc already resident
in HBM.  Every rank runs its own
problem of the named workload (seeds differ by rank), so per-GPU work is
fixed as N grows ("scaling": "weak"); no data moves between ranks.

Rank 0 prints one JSON line.  `value` is the indexer TFLOP/s of the whole
job (2*H_I*d_I FLOPs per causally visible query-key pair, all ranks) over
the device-timed region (max over ranks).  `--impl reference` times the CPU
oracle (fp64, OpenMP) on bounded row samples of the same workload instead.
`--sweep k|s` prints one line per design-space cell instead (see run_sweep).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = ("indexer TFLOP/s & query rows/s at S=262,144 (H_I=64,d_I=128,m=4,k=512); peak HBM")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def visible_pairs(B: int, S: int, T: int, m: int) -> int:
    """Sum over query rows of min(T, floor((t+1)/m)) (closed form)."""
    # rows with (t+1)//m < T contribute (t+1)//m; the rest contribute T
    total = 0
    full_from = m * T - 1  # first t with (t+1)//m >= T
    n_part = min(S, max(full_from, 0))
    # sum_{t=0}^{n_part-1} floor((t+1)/m) = sum_{x=1}^{n_part} floor(x/m)
    x = n_part
    q, r = divmod(x, m)
    part = m * q * (q - 1) // 2 + q * (r + 1)
    total = part + max(S - n_part, 0) * T
    return B * total


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


SELECT_SOURCES = ("si_select.cuh", "si_ptx.cuh", "si_keys.cuh")


def csrc_hash() -> str:
    """Hash of the sources the select kernel is built from."""
    d = os.path.join(ROOT, "streaming_top_indexer_b200", "csrc")
    h = hashlib.sha256()
    for name in SELECT_SOURCES:
        with open(os.path.join(d, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str):
    """DRAM bytes per launch of the select kernel from a committed ncu summary,
    or None if absent or taken on different kernel sources."""
    path = os.path.join(ROOT, "profiles", "select_kernel_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("csrc_hash") != csrc_hash():
        return None
    return d.get("per_launch_bytes", {}).get(workload)


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        # raw samples go to $SI_BENCH_OUT (default: the system temporary directory)
        out_dir = os.environ.get("SI_BENCH_OUT") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"clocks_gpu{gpu_index}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sms, maxs, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sms.append(float(parts[1]))
                    maxs.append(float(parts[2]))
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(nm)
        if not sms:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": max(maxs), "reasons": sorted(reasons),
                "samples": len(sms)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if args.impl == "ours" else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def all_max(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def sample_rows_uniform(S: int, n: int, seed: int):
    rng = np.random.default_rng(seed + 4242)
    return np.sort(rng.choice(S, size=min(n, S), replace=False)).astype(np.int64)


def oracle_sample(q, w, kc, wl, rows_t, b=0):
    """Time the CPU oracle on the given rows of batch b; returns (seconds, flops)."""
    from oracle import oracle as orc
    from streaming_top_indexer_b200 import synth
    tt = torch.from_numpy(rows_t).to(q.device)
    q_rows = synth.bf16_bits(q[b, tt])
    w_rows = w[b, tt].cpu().numpy()
    kc_bits = synth.bf16_bits(kc[b:b + 1])
    rb = np.zeros_like(rows_t)
    t0 = time.perf_counter()
    orc.topk_rows(q_rows, w_rows, rb, rows_t, kc_bits, wl.m, wl.k)
    dt = time.perf_counter() - t0
    vis = np.minimum(wl.T, (rows_t + 1) // wl.m)
    flops = float(2 * wl.H * wl.D * vis.sum())
    return dt, flops


def cpu_baseline(q, w, kc, wl, budget_s: float, seed: int):
    """Oracle on a bounded, seeded sample of the workload's rows (host cores)."""
    from oracle import oracle as orc
    cores = orc.max_threads()
    # calibrate on a small sample, then size the main sample to the budget
    probe = sample_rows_uniform(wl.S, max(cores, 8), seed)
    dt, fl = oracle_sample(q, w, kc, wl, probe)
    per_row = dt / len(probe)
    n = int(max(len(probe), min(4096, budget_s / max(per_row, 1e-9))))
    rows = sample_rows_uniform(wl.S, n, seed + 1)
    dt, fl = oracle_sample(q, w, kc, wl, rows)
    # the same oracle on one host thread, on a sample of about a quarter of the budget
    n1 = int(max(4, min(len(rows), (budget_s / 4) / max(dt / len(rows) * cores, 1e-9))))
    rows1 = sample_rows_uniform(wl.S, n1, seed + 2)
    orc.set_threads(1)
    try:
        dt1, fl1 = oracle_sample(q, w, kc, wl, rows1)
    finally:
        orc.set_threads(cores)
    return {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "rows_per_s": len(rows) / dt,
            "value_1thread": fl1 / dt1 / 1e12, "rows_per_s_1thread": len(rows1) / dt1,
            "sample": f"{len(rows)} uniformly sampled query rows of batch 0 of the {wl.name} workload "
                      f"(fp64 C oracle, OpenMP, {dt:.1f} s); one-thread figure on {len(rows1)} rows "
                      f"({dt1:.1f} s)"}


def run_reference(args, world, rank, local):
    """Reference arm: the CPU oracle as it stands on bounded row samples."""
    from streaming_top_indexer_b200 import synth
    if rank != 0:
        return
    wl = synth.WORKLOADS[args.workload]
    dev = f"cuda:{local}" if torch.cuda.is_available() else "cpu"
    q, w, kc = synth.generate(wl, seed=args.seed, device=dev)
    from oracle import oracle as orc
    cores = orc.max_threads()
    probe = sample_rows_uniform(wl.S, max(cores, 8), args.seed)
    dt, _ = oracle_sample(q, w, kc, wl, probe)
    per_row = dt / len(probe)
    steps_total = args.steps + args.warmup
    n = int(max(8, min(1024, (args.ref_budget / steps_total) / max(per_row, 1e-9))))
    for i in range(args.warmup):
        oracle_sample(q, w, kc, wl, sample_rows_uniform(wl.S, n, args.seed + 100 + i))
    tot_t, tot_f = 0.0, 0.0
    for i in range(args.steps):
        dt, fl = oracle_sample(q, w, kc, wl, sample_rows_uniform(wl.S, n, args.seed + 200 + i))
        tot_t += dt
        tot_f += fl
    value = tot_f / tot_t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(wl, args),
        "rows_per_s": n * args.steps / tot_t,
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"{n} uniformly sampled query rows per step of the {wl.name} workload"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_of(wl, args):
    return {"workload": wl.name, "B": wl.B, "S": wl.S, "T": wl.T, "H_I": wl.H, "d_I": wl.D, "m": wl.m,
            "k": wl.k, "global_batch": wl.B * args.gpus, "seq_len": wl.S,
            "parallelism": f"replicas{args.gpus}" if args.gpus > 1 else "single",
            "l2": "inputs larger than L2 (q alone exceeds 126 MB); no flush between steps"}


def run_ours(args, world, rank, local):
    import streaming_top_indexer_b200 as si
    from streaming_top_indexer_b200 import build as sbuild
    from streaming_top_indexer_b200 import synth

    if rank == 0 and sbuild.needs_build():
        sbuild.build()
    barrier(world)
    dev = torch.device(f"cuda:{local}")
    wl = synth.WORKLOADS[args.workload]
    B, S, T, H, D, m, k = wl.B, wl.S, wl.T, wl.H, wl.D, wl.m, wl.k
    # The per-head materialise baseline needs 4*B*S*H_I*(S/m) bytes for its fp32
    # score tensor (Abstract): the largest S that fits this device's free memory.
    free_start = torch.cuda.mem_get_info(dev)[0]
    materialise = {"bytes_at_workload": 4 * B * S * H * T, "free_bytes": int(free_start),
                   "s_max_fitting": int((free_start / (4 * B * H / m)) ** 0.5),
                   "fits_at_workload": 4 * B * S * H * T <= free_start}
    q, w, kc = synth.generate(wl, seed=args.seed + rank, device=dev)
    # Peak HBM of the indexer step: counted from here, with the inputs resident
    # (generation's own temporaries are freed and not counted).
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    torch.cuda.reset_peak_memory_stats(dev)
    free0 = torch.cuda.mem_get_info(dev)[0]
    input_bytes = q.numel() * 2 + w.numel() * 4 + kc.numel() * 2
    idx = torch.empty((B, S, k), dtype=torch.int32, device=dev)
    sc = torch.empty((B, S, k), dtype=torch.float32, device=dev)
    ws_bytes = si.workspace_bytes(B, S, T, H, D, m, k)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    if args.sort_kernel:
        si.set_sort_in_select(False)  # the earlier design: unordered rows + the row-sort kernel
    sorted_in_select = si.select_sorts_rows(H, D, k)
    launches_per_step = 1 if sorted_in_select else 2

    # One step is the product call, si_indexer_topk: a 256-byte reset of the
    # workspace header, then the select kernel (which also sorts the rows),
    # plus the row-sort kernel only where the select kernel cannot sort.
    def step():
        si.indexer_topk(q, w, kc, m, k, idx, sc, ws, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    assert si.check_device_status(ws) == 0, "device error during warm-up"

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    sampler = ClockSampler(local)
    with sampler:
        barrier(world)
        torch.cuda.synchronize(dev)
        for i in range(args.steps):
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        barrier(world)
    assert si.check_device_status(ws) == 0, "device error during the timed region"
    total_ms = ev[0][0].elapsed_time(ev[-1][1])
    call_ms = [e[0].elapsed_time(e[1]) for e in ev]
    peak_bytes = torch.cuda.max_memory_allocated(dev)
    # cross-check: device memory taken by the outputs and workspace, as the
    # driver sees it (the caching allocator's rounding included)
    mem_get_info_bytes = free0 - torch.cuda.mem_get_info(dev)[0]
    output_bytes = 2 * B * S * k * 4
    total_ms_max = all_max(total_ms, world, dev)

    pairs = visible_pairs(B, S, T, m)
    flops_rank = 2.0 * H * D * pairs
    ms_per_step = total_ms_max / args.steps
    value = world * flops_rank * args.steps / (total_ms_max * 1e-3) / 1e12
    rows_per_s = world * B * S * args.steps / (total_ms_max * 1e-3)

    peaks, peak_src = load_peaks()
    # The dominant kernel's duration: each call's events bracket the 256-byte
    # header reset (a few microseconds) and the select kernel, and also the
    # row sort where the select kernel leaves rows unordered.  So this slightly
    # understates the kernel's own rate.
    call_avg_ms = statistics.mean(call_ms)
    achieved = flops_rank / (call_avg_ms * 1e-3) / 1e12
    traffic = ncu_traffic(wl.name)
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"], "traffic": traffic,
                "peak_source": f"{peak_src} bf16 burst",
                "frac_of_sustained": achieved / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]),
                "kernel": f"select_kernel<{H},{D}>",
                "kernel_ms": call_avg_ms, "kernel_ms_scope": "whole si_indexer_topk call",
                "rows_sorted_in_select": sorted_in_select}

    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config_of(wl, args),
            "rows_per_s": rows_per_s,
            # rows/s at the measured tensor peak: every row costs the step's average FLOPs
            "rows_per_s_roofline": {"achieved": rows_per_s,
                                    "peak": world * B * S * peaks["bf16_tflops"] * 1e12 / flops_rank,
                                    "frac": value / (world * peaks["bf16_tflops"]),
                                    "peak_source": f"{peak_src} bf16 burst"},
            "peak_hbm_bytes": int(peak_bytes), "peak_hbm_gb": peak_bytes / 1e9,
            "hbm_breakdown_bytes": {"inputs": int(input_bytes), "outputs": int(output_bytes),
                                    "workspace": int(ws_bytes),
                                    "outputs_workspace_mem_get_info": int(mem_get_info_bytes)},
            "peak_hbm_scope": "allocator peak during the indexer calls, inputs resident, input generation excluded",
            "materialise_baseline": materialise,
            "workspace_bytes": ws_bytes, "gpu_launches": launches_per_step * args.steps, "roofline": roofline,
            "clocks": sampler.summary()}

    if args.csa:
        att = attention_measure(si, idx, wl, args, dev, stream, peaks, peak_src)
        att["indexer_plus_attention_ms"] = ms_per_step + att["ms"]
        line["csa_attention"] = att
        prod = producers_measure(si, wl, args, dev, stream, peaks, peak_src)
        line["csa_producers"] = prod
        line["csa_step_ms"] = {"producers": prod["ms"], "indexer": ms_per_step, "attention": att["ms"],
                               "total": prod["ms"] + ms_per_step + att["ms"]}
    # end to end through the public API with host buffers
    if not args.no_e2e:
        line["e2e"] = e2e_measure(si, q, w, kc, wl, args, world, dev, stream, flops_rank)
    del idx, sc
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(q, w, kc, wl, args.cpu_budget, args.seed)
    if rank == 0:
        print(json.dumps(line), flush=True)


def materialised_topk_rows(dense, rows, m, k):
    """Top-k of the given query rows from dense [S,T] scores (NaN where not
    visible): score descending, index ascending (stable sort), visible only."""
    T = dense.shape[-1]
    sub = dense[rows]
    sub = torch.where(torch.isnan(sub), torch.full_like(sub, float("-inf")), sub)
    order = torch.sort(-sub, dim=-1, stable=True).indices[:, :min(k, T)]
    vis = torch.clamp((rows + 1) // m, max=T)
    return order, vis


def run_sweep(args):
    """Design-space sweep (one GPU): indexer TFLOP/s of select + sort per cell,
    and recall of each cell's top-k against the materialised baseline (dense
    scores of the same pipeline, stable-sorted by torch) on sampled rows.  One
    JSON line per cell.  The cells vary k (--sweep k) or S with T = S/m
    (--sweep s); queries per unit (256/H_I) and keys per tile (128) are fixed
    by the tcgen05 tile shape."""
    import streaming_top_indexer_b200 as si
    from streaming_top_indexer_b200 import build as sbuild
    from streaming_top_indexer_b200 import synth

    if sbuild.needs_build():
        sbuild.build()
    dev = torch.device("cuda:0")
    base = synth.WORKLOADS[args.workload]
    # cells: (S, k, tuning); tuning = si_set_tuning's design parameters (the
    # counterparts of the pages' chunk and key-tile sizes), defaults elsewhere
    vals = [int(v) for v in args.sweep_values.split(",")] if args.sweep_values else None
    if args.sweep == "k":
        cells = [(base.S, v, {}) for v in (vals or (64, 128, 256, 512, 1024, 2048))]
    elif args.sweep == "s":
        cells = [(v, base.k, {}) for v in (vals or (16384, 32768, 65536, 131072, 262144))]
    else:
        key = {"pool": "pool_entries", "check": "check_tiles", "slack": "cut_slack"}[args.sweep]
        default = {"pool": (800, 1056, 1344, 1600, 1856), "check": (1, 2, 3, 4, 6),
                   "slack": (32, 64, 128, 256, 512)}[args.sweep]
        cells = [(base.S, base.k, {key: v}) for v in (vals or default)]
    stream = torch.cuda.current_stream(dev)
    dense_cache = {}
    for S, k, tuning in cells:
        si.set_tuning(**tuning)
        wl = synth.Workload(f"{base.name}-sweep", base.B, S, base.m, base.H, base.D, k, base.kind)
        B, T, H, D, m = wl.B, wl.T, wl.H, wl.D, wl.m
        if S not in dense_cache:
            dense_cache.clear()
            q, w, kc = synth.generate(wl, seed=args.seed, device=dev)
            dense = si.indexer_scores(q, w, kc, m)[0] if S * T * 4 <= args.sweep_dense_bytes else None
            dense_cache[S] = (q, w, kc, dense)
        q, w, kc, dense = dense_cache[S]
        torch.cuda.synchronize(dev)
        torch.cuda.reset_peak_memory_stats(dev)
        base_bytes = torch.cuda.memory_allocated(dev)  # inputs (and the cached dense scores)
        idx = torch.empty((B, S, k), dtype=torch.int32, device=dev)
        sc = torch.empty((B, S, k), dtype=torch.float32, device=dev)
        ws = torch.zeros(si.workspace_bytes(B, S, T, H, D, m, k), dtype=torch.uint8, device=dev)
        for _ in range(args.warmup):
            si.indexer_topk(q, w, kc, m, k, idx, sc, ws, stream)
        torch.cuda.synchronize(dev)
        e0, e1 = (torch.cuda.Event(enable_timing=True) for _ in range(2))
        times = []
        for _ in range(args.steps):
            e0.record(stream)
            si.indexer_topk(q, w, kc, m, k, idx, sc, ws, stream)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            times.append(e0.elapsed_time(e1))
        assert si.check_device_status(ws) == 0, "device error in the sweep"
        flops = 2.0 * H * D * visible_pairs(B, S, T, m)
        ms = statistics.median(times)
        inputs = q.numel() * 2 + w.numel() * 4 + kc.numel() * 2
        # indexer footprint: inputs + outputs + workspace (the dense scores of the recall check excluded)
        peak_idx = inputs + torch.cuda.max_memory_allocated(dev) - base_bytes
        cell = {"sweep": args.sweep, "workload": base.name, "B": B, "S": S, "T": T, "H_I": H, "d_I": D, "m": m,
                "k": k, "value": flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms": ms,
                "tuning": tuning, "steps": args.steps, "warmup": args.warmup, "peak_hbm_bytes": int(peak_idx),
                "recall_vs_materialised": None}
        if dense is not None:
            g = torch.Generator().manual_seed(args.seed + 1)
            rows = torch.randperm(S, generator=g)[:args.sweep_rows].to(dev)
            order, vis = materialised_topk_rows(dense, rows, m, k)
            got = idx[0, rows].long()
            rec, exact = [], 0
            for r in range(rows.numel()):
                n = int(min(k, int(vis[r])))
                if n == 0:
                    continue
                a = set(order[r, :n].tolist())
                b = set(got[r, :n].tolist())
                rec.append(len(a & b) / n)
                exact += int(torch.equal(order[r, :n], got[r, :n]))
            cell["recall_vs_materialised"] = {"rows": len(rec), "mean": float(np.mean(rec)) if rec else None,
                                              "min": float(np.min(rec)) if rec else None,
                                              "rows_identical": exact}
        print(json.dumps(cell), flush=True)
        del idx, sc, ws
    si.set_tuning()


def attention_pairs(S: int, T: int, m: int, k: int) -> int:
    """Number of (query row, selected key) pairs: sum_t min(k, V_t)."""
    t = np.arange(S, dtype=np.int64)
    return int(np.minimum(k, np.minimum(T, (t + 1) // m)).sum())


def attention_measure(si, idx, wl, args, dev, stream, peaks, peak_src):
    """The CSA step's third stage on the indexer's output: sparse attention of
    128 heads (d = d_v = 128, bf16) over the selected keys, CUDA-event timed
    on the same stream.  FLOPs: 2*128*(d + d_v) per (row, selected key)."""
    from streaming_top_indexer_b200 import synth
    D = DV = 128
    q, kc, vc = synth.generate_attention(wl.B, wl.S, wl.T, D, DV, seed=args.seed, device=dev)
    out = torch.empty((wl.B, wl.S, 128, DV), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((wl.B, wl.S, 128), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    scale = 1.0 / math.sqrt(D)
    for _ in range(args.warmup):
        si.sparse_attention(q, kc, vc, idx, scale, out, lse, status, stream)
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for e0, e1 in ev:
        e0.record(stream)
        si.sparse_attention(q, kc, vc, idx, scale, out, lse, status, stream)
        e1.record(stream)
    torch.cuda.synchronize(dev)
    assert int(status.item()) == 0, "device error in the attention stage"
    ms = statistics.mean(e0.elapsed_time(e1) for e0, e1 in ev)
    pairs = wl.B * attention_pairs(wl.S, wl.T, wl.m, wl.k)
    flops = 2.0 * 128 * (D + DV) * pairs
    tflops = flops / (ms * 1e-3) / 1e12
    # bytes: q and out once, the gathered K and V rows (from L2 when they fit)
    hbm = q.numel() * 2 + out.numel() * 2 + lse.numel() * 4 + idx.numel() * 4
    gathered = pairs * (D + DV) * 2
    del q, kc, vc, out, lse
    return {"kernel": "sparse_attn_kernel<128,128>", "heads": 128, "d": D, "d_v": DV, "ms": ms,
            "value": tflops, "unit": "TFLOP/s",
            "roofline": {"bound": "tensor", "achieved": tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": tflops / peaks["bf16_tflops"], "peak_source": f"{peak_src} bf16 burst"},
            "hbm_bytes_per_call": int(hbm), "hbm_gbs": hbm / (ms * 1e-3) / 1e9,
            "gathered_kv_bytes_per_call": int(gathered),
            "indexer_plus_attention_ms": None}


def producers_measure(si, wl, args, dev, stream, peaks, peak_src, d_model=4096):
    """The indexer's inputs from hidden states (si_indexer_inputs): q, w and
    the m:1 compressed keys by tcgen05 GEMMs, random weights, CUDA-event timed.
    FLOPs: 2*B*S*d_model*(H_I*d_I + H_I) + 2*B*T*m*d_model*d_I."""
    from streaming_top_indexer_b200 import synth
    B, S, H, D, m = wl.B, wl.S, wl.H, wl.D, wl.m
    x, w_q, w_w, w_k = synth.generate_hidden(B, S, d_model, H, D, m, seed=args.seed, device=dev)
    q = torch.empty((B, S, H, D), dtype=torch.bfloat16, device=dev)
    w = torch.empty((B, S, H), dtype=torch.float32, device=dev)
    kc = torch.empty((B, S // m, D), dtype=torch.bfloat16, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    for _ in range(args.warmup):
        si.indexer_inputs(x, w_q, w_w, w_k, H, D, m, q, w, kc, st, stream)
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for e0, e1 in ev:
        e0.record(stream)
        si.indexer_inputs(x, w_q, w_w, w_k, H, D, m, q, w, kc, st, stream)
        e1.record(stream)
    torch.cuda.synchronize(dev)
    assert int(st.item()) == 0, "device error in the producers"
    ms = statistics.mean(e0.elapsed_time(e1) for e0, e1 in ev)
    flops = 2.0 * B * S * d_model * (H * D + H) + 2.0 * B * (S // m) * m * d_model * D
    tflops = flops / (ms * 1e-3) / 1e12
    del x, w_q, w_w, w_k, q, w, kc
    return {"kernel": "gemm_kernel (q: BN=256, w: BN=64, kc: BN=128)", "d_model": d_model, "ms": ms,
            "value": tflops, "unit": "TFLOP/s",
            "roofline": {"bound": "tensor", "achieved": tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": tflops / peaks["bf16_tflops"], "peak_source": f"{peak_src} bf16 burst"}}


def e2e_measure(si, q, w, kc, wl, args, world, dev, stream, flops_rank):
    """Same metric through the C-ABI host-buffer call si_indexer_topk_host
    (binding indexer_topk_host): pinned host inputs copied in, outputs copied
    out, inside the timed region every step."""
    qh = q.cpu().pin_memory()
    wh = w.cpu().pin_memory()
    kch = kc.cpu().pin_memory()
    bufs = {}
    steps = max(1, min(args.steps, args.e2e_steps))
    for _ in range(2):
        si.indexer_topk_host(qh, wh, kch, wl.m, wl.k, device=dev, buffers=bufs, stream=stream)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    e0.record(stream)
    for _ in range(steps):
        si.indexer_topk_host(qh, wh, kch, wl.m, wl.k, device=dev, buffers=bufs, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = all_max(e0.elapsed_time(e1), world, dev)
    h2d = qh.numel() * 2 + wh.numel() * 4 + kch.numel() * 2
    d2h = bufs["idx_h"].numel() * 4 + bufs["score_h"].numel() * 4
    return {"value": world * flops_rank * steps / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": steps,
            "ms_per_step": ms / steps}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=None, help="long (default), or v4flash for --sweep")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--csa", action="store_true",
                    help="also time the rest of the CSA step: the producers of q, w, kc from hidden states "
                         "(d_model 4096) and the sparse attention (128 heads, d=d_v=128) over the indexer's output")
    ap.add_argument("--sort-kernel", action="store_true",
                    help="sort rows in the separate row-sort kernel instead of inside the select kernel")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work")
    ap.add_argument("--ref-budget", type=float, default=60.0, help="seconds of oracle work, reference arm")
    ap.add_argument("--sweep", choices=["k", "s", "pool", "check", "slack"], default=None,
                    help="design-space sweep over k, S, pool capacity, check interval or cut slack "
                         "(one GPU; one JSON line per cell)")
    ap.add_argument("--sweep-values", default="", help="comma-separated k or S values of the sweep")
    ap.add_argument("--sweep-rows", type=int, default=256, help="rows checked against the materialised top-k")
    ap.add_argument("--sweep-dense-bytes", type=float, default=20e9,
                    help="largest dense score matrix materialised for the recall check")
    args = ap.parse_args()
    if args.workload is None:
        args.workload = "v4flash" if args.sweep else "long"
    if args.sweep:
        run_sweep(args)
        return
    world, rank, local = dist_setup(args)
    args.gpus = world if world > 1 else args.gpus
    try:
        if args.impl == "reference":
            run_reference(args, world, rank, local)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""Benchmark of the Fathom per-query read-depth top-k key scan on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fathom|reference]
                    [--workload qwen3_8b_layer_128k|qwen3_8b_layer_128k_8plane|
                               qwen3_8b_layer_128k_blocked|
                               plan_variants_128k|host_1m|host_256k|fixed_vs_wf_1m|
                               agent_16_sessions|append_layer_128k|
                               attention_layer_128k]

A step is one decode-step scan of a whole layer through the hot path, once
per plan of the workload: plan (reverse water-filling at B bits per key, or
a fixed top-r plan; GQA union) then scan + top-k, for every KV head and
query head.  agent_16_sessions instead plans 16 independent sessions and
scans them in one batched call per step.  Default workload: a Qwen3-8B-shaped
layer resident in HBM (8 KV heads x 4 query heads, head_dim 128, 131072
keys, B in {68, 92, 136}, k = 2048).  Inputs are synthetic (seeded, see
synth/); each step gets fresh queries and the L2 is flushed (256 MiB write)
between timed steps, outside the step's events.

Prints one JSON line (rank 0).  value = Gkeys/s over all ranks (keys per KV
head x KV heads x scans per step x steps / the slowest rank's summed step
time).  For N > 1 each rank scans its own independent layer (weak scaling;
the path needs no collective).  --impl reference times the CPU oracle
instead, on a bounded sample of the same workload.

e2e: every step copies its queries and budgets from pinned host memory,
runs the public API calls (with --graph 1, captured once as a CUDA graph on
the staged input buffers, as a decode loop would, and replayed) and copies
the top-k indices and scores back, timed by the host clock.
"""
from __future__ import annotations

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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "Gkeys/s per decode-step scan; achieved GB/s vs HBM / PCIe roofline"
UNIT = "Gkeys/s"
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20

# plans: ("wf", B) = reverse water-filling at B bits per key; ("mg", B) = the
# marginal-gain variant; ("fixed", r) = the top-r channels by |q_c| at all
# b bits.  "bits": b, the stored code width (4 unless given; 8 = the 8-plane
# variant for an 8-bit K cache).  "block_keys": grouped per-token-block
# scales over blocks of that many tokens (0 unless given).  "device_keys":
# keys drawn on the GPU
# (synth.device_keys) instead of numpy, for sizes numpy would take minutes
# on.  agent_16_sessions scans its sessions in one batched call.
WORKLOADS = {
    "qwen3_8b_layer_128k": dict(H=8, G=4, n=131072, d=128, k=2048, residency="device",
                                plans=(("wf", 68), ("wf", 92), ("wf", 136))),
    # the same layer with an 8-bit K cache (8 planes per channel), same budgets
    "qwen3_8b_layer_128k_8plane": dict(H=8, G=4, n=131072, d=128, k=2048, residency="device",
                                       bits=8, plans=(("wf", 68), ("wf", 92), ("wf", 136))),
    # the same layer with grouped per-token-block scales (blocks of 2048 keys)
    "qwen3_8b_layer_128k_blocked": dict(H=8, G=4, n=131072, d=128, k=2048, residency="device",
                                        block_keys=2048,
                                        plans=(("wf", 68), ("wf", 92), ("wf", 136))),
    # the million-token layer with its planes in pinned host memory (the
    # offloaded setting), followed by the same keys resident in HBM
    "host_1m": dict(H=8, G=4, n=1 << 20, d=128, k=2048, residency="host_mapped",
                    plans=(("wf", 18), ("wf", 68), ("wf", 92), ("wf", 136)), device_keys=True,
                    resident_twin="hbm_1m"),
    "hbm_1m": dict(H=8, G=4, n=1 << 20, d=128, k=2048, residency="device",
                   plans=(("wf", 18), ("wf", 68), ("wf", 92), ("wf", 136)), device_keys=True),
    # the host path at a quarter of the keys: the profiling case of the fetch
    # kernel (its traffic scales with n)
    "host_256k": dict(H=8, G=4, n=1 << 18, d=128, k=2048, residency="host_mapped",
                      plans=(("wf", 18), ("wf", 68), ("wf", 92), ("wf", 136)), device_keys=True),
    # reverse water-filling against its marginal-gain variant, same budgets
    "plan_variants_128k": dict(H=8, G=4, n=131072, d=128, k=2048, residency="device",
                               plans=(("wf", 68), ("mg", 68), ("wf", 92), ("mg", 92),
                                      ("wf", 136), ("mg", 136))),
    "fixed_vs_wf_1m": dict(H=8, G=4, n=1 << 20, d=128, k=2048, residency="host_mapped",
                           plans=(("fixed", 34), ("fixed", 17), ("wf", 68), ("wf", 92)),
                           device_keys=True),
    # the append path: decode-step keys (m = 1 per KV head) and a bulk chunk
    # into a packed Qwen3-8B-shaped layer
    "append_layer_128k": dict(H=8, G=4, n=131072, d=128, k=0, residency="device",
                              append=(1, 8192), plans=None),
    # after the scan: attention over each plan's top-k, with its error
    # against dense attention (and against attention over the exact top-k)
    "attention_layer_128k": dict(H=8, G=4, n=131072, d=128, k=2048, residency="device",
                                 plans=(("wf", 68), ("wf", 92), ("wf", 136), ("fixed", 34),
                                        ("fixed", 17)), attention=True),
    "agent_16_sessions": dict(H=8, G=4, n=None, d=128, k=1024, residency="host_mapped",
                              sessions=16, plans=None, device_keys=True, batched=True),
}


def plan_name(spec):
    return f"{spec[0]}{spec[1]}"


def plan_bits(spec, bits=4):
    """Bits per key a query of this plan reads (bits = the code width b)."""
    return bits * spec[1] if spec[0] == "fixed" else spec[1]


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=("fathom", "reference"), default="fathom")
    p.add_argument("--workload", choices=tuple(WORKLOADS), default="host_1m")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-recall", action="store_true",
                   help="free the float32 keys once packed and skip the recall check (keeps "
                        "profiler runs small on the device)")
    p.add_argument("--graph", type=int, default=1,
                   help="replay the timed steps as one CUDA graph (1) or launch them eagerly (0)")
    p.add_argument("--heat-seconds", type=float, default=1.0,
                   help="minimum warm-up duration (load for the clock sampler); 0 for "
                        "profiler runs, which then see exactly --warmup warm-up steps")
    return p.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def config_of(wl_name, wl, flush_note, sessions=None):
    c = {"workload": wl_name, "kv_heads": wl["H"], "query_heads_per_kv": wl["G"],
         "head_dim": wl["d"], "k": wl["k"],
         "residency": "hbm" if wl["residency"] == "device" else "host_pinned_mapped",
         "code_bits": wl.get("bits", 4), "scale_block_keys": wl.get("block_keys", 0),
         "l2": flush_note}
    if sessions is None:
        c["n_keys"] = wl["n"]
        c["plans"] = [plan_name(p) for p in wl["plans"]]
    else:
        c["sessions"] = len(sessions)
        c["n_keys_per_session"] = [x["n"] for x in sessions]
        c["budget_per_session"] = [x["budget"] for x in sessions]
        c["batched"] = True
    return c


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------ host link
def measure_host_link(fp, torch, nbytes=1 << 30, reps=10):
    """Host->device link peaks measured in this run: a pinned host->device
    copy of `nbytes` and a zero-copy read kernel over the same pinned buffer
    (best of `reps` each, CUDA events)."""
    host = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    dev = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    sink = torch.zeros(1, dtype=torch.int64, device="cuda")
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    best_copy = best_zero = 0.0
    for _ in range(reps):
        a.record()
        dev.copy_(host, non_blocking=True)
        b.record()
        b.synchronize()
        best_copy = max(best_copy, nbytes / (a.elapsed_time(b) / 1e3) / 1e9)
    for _ in range(reps):
        a.record()
        fp.fathom_link_probe(host, nbytes, sink)
        b.record()
        b.synchronize()
        best_zero = max(best_zero, nbytes / (a.elapsed_time(b) / 1e3) / 1e9)
    del host, dev
    return {"h2d_memcpy_gbs": best_copy, "zero_copy_read_gbs": best_zero,
            "how": f"pinned host->device copy and zero-copy read kernel over {nbytes >> 20} MiB, "
                   f"best of {reps}, CUDA events"}


# ------------------------------------------------------------- CPU oracle
def host_cpu():
    """-> (model name from /proc/cpuinfo or None, usable host cores)."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        cores = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        cores = os.cpu_count() or 1
    return model, cores


def _oracle_query_scan(oracle, ref, hi, qrow, spec, k, bits):
    """One query's plan + fp64 score of every key + full-sort top-k."""
    if spec[0] == "wf":
        tq = oracle.plan_greedy(oracle.importance(qrow, ref["sigma2"][hi]), spec[1], bits)
    elif spec[0] == "mg":
        tq = oracle.plan_marginal(oracle.importance(qrow, ref["sigma2"][hi]), spec[1], bits)
    else:
        tq = oracle.fixed_plan(qrow, spec[1], bits)
    s = oracle.score_head(ref, hi, qrow, tq)
    oracle.topk(s, k)


def oracle_sample(keys_heads, q_bf16, G, plans, k, ref=None, min_seconds=0.0, bits=4,
                  block_keys=0, threads=1):
    """Time the oracle (plan + fp64 score + full-sort top-k per query) over
    the given KV heads' keys (float32 [h][n][d]) at every plan spec, cycling
    over (head, plan, query head) until at least min_seconds have passed
    (every (head, plan) once at least).  threads > 1 runs independent queries
    on that many host threads at once (the C oracle runs without the GIL).
    The index build (storage side, off the decode path) is not timed.
    Returns (seconds, query scans, KV-head keys = query scans * n / G)."""
    import oracle
    if ref is None:
        ref = oracle.build_index(keys_heads, bits=bits, block_keys=block_keys)
    oracle._load()
    n = keys_heads.shape[1]
    items = [(hi, spec, g) for hi in range(keys_heads.shape[0]) for spec in plans
             for g in range(G)]

    def one(i):
        hi, spec, g = items[i % len(items)]
        _oracle_query_scan(oracle, ref, hi, q_bf16[hi * G + g], spec, k, bits)

    done = 0
    t0 = time.perf_counter()
    if threads <= 1:
        while done < len(items) or time.perf_counter() - t0 < min_seconds:
            one(done)
            done += 1
    else:
        from concurrent.futures import ThreadPoolExecutor
        wave = len(items) if min_seconds <= 0 else max(len(items), 2 * threads)
        with ThreadPoolExecutor(max_workers=threads) as pool:
            while done < len(items) or time.perf_counter() - t0 < min_seconds:
                list(pool.map(one, range(done, done + wave)))
                done += wave
    secs = time.perf_counter() - t0
    return secs, done, done * n / G


CPU_BASELINE_SECONDS = 12.0


def cpu_baseline(keys_heads, q_bf16, G, plans, k, bits=4, block_keys=0):
    """The oracle on the host cores, on a sample of the workload: about 12 s
    on one thread, then about 12 s with one query scan per host core at a
    time.  value / cores: the all-core run."""
    import oracle
    ref = oracle.build_index(keys_heads, bits=bits, block_keys=block_keys)
    model, cores = host_cpu()
    plan_names = [plan_name(p) for p in plans]
    n = keys_heads.shape[1]
    s1, q1, keys1 = oracle_sample(keys_heads, q_bf16, G, plans, k, ref,
                                  min_seconds=CPU_BASELINE_SECONDS, bits=bits)
    sa, qa, keysa = oracle_sample(keys_heads, q_bf16, G, plans, k, ref,
                                  min_seconds=CPU_BASELINE_SECONDS, bits=bits, threads=cores)
    what = (f"query scans (plan + fp64 score of all {n} keys + full-sort top-k) cycling over "
            f"{keys_heads.shape[0]} KV head(s) x {G} query heads x plans {plan_names}")
    return {"value": keysa / sa / 1e9, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{qa} {what}, {cores} threads, {sa:.1f} s; KV-head keys = query scans "
                      f"x n / {G}",
            "single_thread": {"value": keys1 / s1 / 1e9, "unit": UNIT, "cores": 1,
                              "sample": f"{q1} {what}, one thread, {s1:.1f} s"},
            "host_cpu": model, "nproc": cores}


def reference_plans(wl):
    if wl.get("plans"):
        return wl["plans"]
    return tuple(("wf", B) for B in (68, 92, 136))


def run_reference(args, wl_name, wl):
    """The oracle as the reference arm: every step scans one KV head of the
    workload at its full key count once per plan (each of its G query heads),
    the query scans spread over the host cores."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    n = wl["n"] or (1 << 18)
    plans = reference_plans(wl)
    bits = wl.get("bits", 4)
    ses = synth.make_session(0, 1, wl["G"], n, plan_bits(plans[0], bits), head_dim=wl["d"])
    import oracle
    ref = oracle.build_index(ses.keys[:1], bits=bits, block_keys=wl.get("block_keys", 0))
    model, cores = host_cpu()
    threads = min(cores, len(plans) * wl["G"])
    times, keys = [], 0.0
    for i in range(args.warmup + args.steps):
        secs, _, kk = oracle_sample(ses.keys[:1], ses.q_bf16, wl["G"], plans, wl["k"], ref,
                                    bits=bits, threads=threads)
        if i >= args.warmup:
            times.append(secs)
            keys += kk
    total = sum(times)
    value = keys / total / 1e9
    sample = (f"each step: 1 of {wl['H']} KV heads ({wl['G']} query heads) once per plan "
              f"{[plan_name(p) for p in plans]}, {n} keys, query scans on {threads} threads "
              f"of {cores} cores ({model})")
    cfg = config_of(wl_name, dict(wl, n=n, plans=plans), "n/a (CPU)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": cfg,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": sample, "host_cpu": model, "nproc": cores},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------ traffic
def recorded_traffic(wl_name, wl, kernel):
    """Measured traffic per launch of the dominant kernel, from the ncu
    capture recorded in profiles/traffic.json: DRAM read+write bytes for the
    HBM scan, host-memory read bytes (sysmem sectors x 32 B) for the fetch.
    None unless the kernel's source is unchanged since the capture (sha256)
    and the capture covers this workload's plans; host workloads of other
    sizes scale the capture by their key count (the union planes are
    proportional to it)."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            recs = json.load(f)
        # a capture of this very workload ("kernel@workload") before the
        # kernel's default one
        rec = recs.get(f"{kernel}@{wl_name}") or recs[kernel]
        with open(os.path.join(ROOT, rec["source"]), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest() != rec["sha256"]:
                return None, "kernel changed since the recorded capture"
    except (OSError, KeyError, ValueError):
        return None, "no recorded capture"
    plans = [plan_name(p) for p in (wl.get("plans") or ())]
    if plans != rec["plans"]:
        return None, "no capture of these plans"
    if kernel == "scan_kernel":
        if wl_name != rec["workload"]:
            return None, "no capture of this workload"
        vals = rec["dram_bytes_per_launch"]
        note = f"ncu dram__bytes_read+write, {rec['workload']}, mean over plans"
    else:
        vals = [v * wl["n"] / rec["n_keys"] for v in rec["host_link_read_bytes_per_launch"]]
        note = (f"ncu host-memory read sectors x 32 B, {rec['workload']} scaled to "
                f"{wl['n']} keys, mean over plans")
    return sum(vals) / len(vals), note


# ------------------------------------------------------------ ranks
def max_over_ranks(dist, values, device):
    """Each value's maximum over the ranks (the slowest rank's device-timed
    totals); the values themselves when there is no process group."""
    if dist is None:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_throughput(keys_per_step, steps, world, total_ms, e2e_seconds):
    """Whole-job Gkeys/s: every rank scans keys_per_step keys per step (weak
    scaling), timed by the slowest rank.  -> (device-timed, end to end)."""
    keys = keys_per_step * steps * world
    return keys / (total_ms / 1e3) / 1e9, keys / e2e_seconds / 1e9


# ---------------------------------------------------------------- GPU path
def build_sessions(wl, rank, torch, fp):
    """-> list of dicts {n, budget, keys (device float32 [H][n][d]), index,
    plans}: the workload's sessions packed into their indices."""
    H, G, d = wl["H"], wl["G"], wl["d"]
    if wl.get("sessions"):
        params = synth.agent_session_params(wl["sessions"], base_seed=1000 + 100 * rank,
                                            n_kv_heads=H, head_dim=d)
    else:
        sigma, _ = synth.channel_sigma(rank, H, d)
        params = [dict(seed=rank, n=wl["n"], budget=None, sigma=sigma)]
    out = []
    for p in params:
        if wl.get("device_keys"):
            keys = synth.device_keys(torch, p["sigma"], p["n"], p["seed"])
        else:
            ses = synth.make_session(p["seed"], H, G, p["n"], 64, head_dim=d)
            keys = torch.from_numpy(ses.keys).cuda()
        index = fp.KeyIndex(H, G, p["n"], d, wl["residency"], bits=wl.get("bits", 4),
                            block_keys=wl.get("block_keys", 0))
        index.pack(keys)
        plans = wl["plans"] if wl.get("plans") else (("wf", p["budget"]),)
        out.append(dict(n=p["n"], budget=p["budget"], keys=keys, index=index, plans=plans))
    torch.cuda.synchronize()
    return out


def run_fathom(args, wl_name, wl):
    import torch
    import decode_fathom_plan_b200 as fp

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    fp.load_library()
    sessions = build_sessions(wl, rank, torch, fp)
    assert fp.fathom_last_device_status() == fp.FATHOM_OK
    if args.no_recall:
        for S in sessions:
            S["keys"] = None
        torch.cuda.empty_cache()
    link = measure_host_link(fp, torch) if wl["residency"] != "device" else None
    line = measure_workload(args, wl_name, wl, sessions, link, dist, torch, fp)

    twin_name = wl.get("resident_twin")
    if twin_name and not args.no_recall:   # the twin is packed from the same keys
        # the same keys and queries with the index resident in HBM: the
        # resident mode of the same configuration, as a sub-record
        twin = WORKLOADS[twin_name]
        for S in sessions:
            S["index"] = None
        torch.cuda.empty_cache()
        for S in sessions:
            ix = fp.KeyIndex(twin["H"], twin["G"], S["n"], twin["d"], twin["residency"])
            ix.pack(S["keys"])
            S["index"] = ix
        torch.cuda.synchronize()
        assert fp.fathom_last_device_status() == fp.FATHOM_OK
        sub = measure_workload(args, twin_name, twin, sessions, None, dist, torch, fp)
        line["hbm_resident"] = {key: sub[key] for key in (
            "value", "unit", "ms_per_step", "config", "e2e", "gpu_launches", "roofline",
            "clocks", "per_plan", "step_ms_median")}

    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.no_recall:
        S0 = sessions[0]
        H, G, k = wl["H"], wl["G"], wl["k"]
        nh = max(1, min(H, (8 * 131072) // S0["n"]))
        line["cpu_baseline"] = cpu_baseline(S0["keys"][:nh].cpu().numpy(),
                                            S0["q"][0].cpu().numpy().view(np.uint16), G,
                                            S0["plans"], k, wl.get("bits", 4),
                                            wl.get("block_keys", 0))
        if "hbm_resident" in line:
            line["hbm_resident"]["cpu_baseline"] = dict(
                line["cpu_baseline"], note="the oracle reads host memory either way: "
                                           "the same measurement as the host-resident line")
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def measure_workload(args, wl_name, wl, sessions, link, dist, torch, fp):
    """Time K steps of one workload over its packed sessions (device-timed
    value, roofline of the dominant kernel, end to end through the public
    API) and return its JSON line (without the CPU baseline).  Every rank
    calls it in the same order (one all-reduce)."""
    rank, world, local = dist_env()
    H, G, d, k = wl["H"], wl["G"], wl["d"], wl["k"]
    Q = H * G
    batched = bool(wl.get("batched"))
    W, K = max(3, args.warmup), args.steps
    # scans of one step: (session, plan spec, buffers, budget vector)
    jobs = []
    for si, S in enumerate(sessions):
        S["q"] = torch.from_numpy(synth.draw_queries(10_000 + 100 * rank + si, Q, d,
                                                     count=W + K).view(np.int16)).cuda()
        for spec in S["plans"]:
            B = plan_bits(spec, wl.get("bits", 4))
            jobs.append(dict(s=si, spec=spec, buf=fp.ScanBuffers(S["index"], k),
                             bvec=torch.full((Q,), B, dtype=torch.int32, device="cuda")))
    ws_batch = None
    if batched:
        descs = [S["index"].desc for S in sessions]
        ws_batch = torch.empty(max(16, fp.fathom_scan_batched_workspace_bytes(descs, k)),
                               dtype=torch.uint8, device="cuda")
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    def plan(j, i):
        S = sessions[j["s"]]
        b = j["buf"]
        if j["spec"][0] == "wf":
            fp.fathom_plan(S["index"].desc, S["q"][i], j["bvec"], b.t, b.t_union, b.nbytes)
        elif j["spec"][0] == "mg":
            fp.fathom_plan_marginal(S["index"].desc, S["q"][i], j["bvec"], b.t, b.t_union,
                                    b.nbytes)
        else:
            fp.fathom_fixed_plan(S["index"].desc, S["q"][i], j["spec"][1], b.t, b.t_union,
                                 b.nbytes)

    def step(i, flags=0, qsrc=None):
        if batched:
            for j in jobs:
                plan(j, i)
            fp.fathom_scan_topk_batched(
                [S["index"].desc for S in sessions], [S["q"][i] for S in sessions],
                [j["buf"].t for j in jobs], [j["buf"].t_union for j in jobs], k,
                [j["buf"].idx for j in jobs], [j["buf"].score for j in jobs], ws_batch, flags)
        else:
            for j in jobs:
                S = sessions[j["s"]]
                plan(j, i)
                b = j["buf"]
                fp.fathom_scan_topk(S["index"].desc, S["q"][i], b.t, b.t_union, k, b.idx,
                                    b.score, b.workspace, flags)

    clocks = ClockSampler(local)
    clocks.start()
    t_heat = time.perf_counter()
    i = 0
    while i < W or time.perf_counter() - t_heat < args.heat_seconds:   # warm-up + clock load
        step(i % W)
        flush.fill_(i & 0xFF)
        i += 1
    torch.cuda.synchronize()
    fp.fathom_profile_read()
    status = fp.fathom_last_device_status()
    assert status == fp.FATHOM_OK, fp.status_str(status)

    # external records keep the events timing points inside a captured graph
    ev = [(torch.cuda.Event(enable_timing=True, external=bool(args.graph)),
           torch.cuda.Event(enable_timing=True, external=bool(args.graph))) for _ in range(K)]

    def timed_steps():
        for s in range(K):
            flush.fill_(s & 0xFF)               # L2 flush, outside the step's events
            ev[s][0].record()
            step(W + s, fp.FATHOM_SCAN_PROFILE)
            ev[s][1].record()

    launches0 = fp.fathom_launch_count()
    graph = None
    if args.graph:
        # the K timed steps as one CUDA graph (kernels, flushes and events are
        # all nodes; every step still runs all of its work)
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            with torch.cuda.graph(graph, stream=side, capture_error_mode="relaxed"):
                timed_steps()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
    launches = fp.fathom_launch_count() - launches0
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    if graph is not None:
        graph.replay()
    else:
        timed_steps()
        launches = fp.fathom_launch_count() - launches0
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clk = clocks.stop()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = sum(step_ms)
    scan_ms, scan_launches = fp.fathom_profile_read()
    if graph is not None:
        del graph
    status = fp.fathom_last_device_status()
    assert status == fp.FATHOM_OK, fp.status_str(status)

    # plan byte counts and quality of the last step (same structure every step)
    per_plan = []
    union_bytes_total = 0.0
    with torch.no_grad():
        for j in jobs:
            S = sessions[j["s"]]
            nb = j["buf"].nbytes.cpu().numpy()
            qb, ub = nb[:Q].astype(np.float64), nb[Q:].astype(np.float64)
            union_bytes_total += ub.sum()
            # recall against the exact fp32 top-k (torch, outside the path)
            qf = S["q"][W + K - 1].view(torch.bfloat16).float().reshape(H, G, d)
            got = j["buf"].idx.reshape(H, G, k).long()
            rec = []
            for h in range(H if S["keys"] is not None else 0):
                exact = (S["keys"][h] @ qf[h].T).topk(k, dim=0).indices.T     # [G][k]
                for g in range(G):
                    inter = np.intersect1d(exact[g].cpu().numpy(), got[h, g].cpu().numpy())
                    rec.append(len(inter) / k)
            per_plan.append({"plan": plan_name(j["spec"]), "session": j["s"], "n_keys": S["n"],
                             "bits_per_key": plan_bits(j["spec"], wl.get("bits", 4)),
                             "bytes_per_query": float(qb.mean()),
                             "union_bytes_per_kv_head": float(ub.mean()),
                             "union_factor": float(ub.sum() / (qb.sum() / G)),
                             "recall_vs_exact_fp32": float(np.mean(rec)) if rec else None})

    # end to end through the public API with host buffers
    q_host = [torch.from_numpy(S["q"][W:W + K].cpu().numpy()).pin_memory() for S in sessions]
    b_host = [j["bvec"].cpu().pin_memory() for j in jobs]
    q_stage = [torch.empty((Q, d), dtype=torch.int16, device="cuda") for _ in sessions]
    idx_host = [torch.empty((Q, k), dtype=torch.int32).pin_memory() for _ in jobs]
    sc_host = [torch.empty((Q, k), dtype=torch.float32).pin_memory() for _ in jobs]
    saved_q = [S["q"] for S in sessions]
    for si, S in enumerate(sessions):
        S["q"] = q_stage[si].unsqueeze(0)   # the API calls read the staged queries
    e2e_graph = None
    if args.graph:
        # a decode loop captures its per-step calls once and replays them:
        # the same public calls on the same staged buffers, one graph launch
        for si in range(len(sessions)):
            q_stage[si].copy_(q_host[si][0])
        torch.cuda.synchronize()
        e2e_graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            with torch.cuda.graph(e2e_graph, stream=side, capture_error_mode="relaxed"):
                step(0)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
    e2e_s = []
    for s in range(K):
        flush.fill_(s & 0xFF)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for si, S in enumerate(sessions):
            q_stage[si].copy_(q_host[si][s], non_blocking=True)
        for ji, j in enumerate(jobs):
            j["bvec"].copy_(b_host[ji], non_blocking=True)
        if e2e_graph is not None:
            e2e_graph.replay()
        else:
            step(0)
        for ji, j in enumerate(jobs):
            idx_host[ji].copy_(j["buf"].idx, non_blocking=True)
            sc_host[ji].copy_(j["buf"].score, non_blocking=True)
        torch.cuda.synchronize()
        e2e_s.append(time.perf_counter() - t0)
    if e2e_graph is not None:
        del e2e_graph
    status = fp.fathom_last_device_status()
    assert status == fp.FATHOM_OK, fp.status_str(status)
    for S, q in zip(sessions, saved_q):
        S["q"] = q
    h2d = len(sessions) * Q * d * 2 + len(jobs) * Q * 4
    d2h = len(jobs) * Q * k * 8

    keys_per_step = sum(H * sessions[j["s"]]["n"] for j in jobs)
    total_ms, e2e_total = max_over_ranks(dist, [total_ms, sum(e2e_s)], "cuda")
    value, e2e_value = job_throughput(keys_per_step, K, world, total_ms, e2e_total)

    launches_per_step = 1 if batched else len(jobs)
    bytes_per_launch = union_bytes_total / launches_per_step
    avg_launch_ms = scan_ms / max(1, scan_launches)
    achieved = bytes_per_launch / (avg_launch_ms / 1e3) / 1e9
    if wl["residency"] == "device":
        peak, peak_src = load_peaks()
        bound, peak_note = "hbm", f"{peak_src} hbm_gbs (MEASURED_PEAKS.json)"
        kernel = "scan_kernel (filter pass)"
    else:
        peak = max(link["h2d_memcpy_gbs"], link["zero_copy_read_gbs"])
        bound, peak_note = "host_link", "measured in this run: max(pinned copy, zero-copy read)"
        kernel = ("fetch_kernel, one launch per unit of KV heads (union planes, host -> "
                  "device ring), timed from the first unit's fetch to the last one's end")
    traffic, traffic_note = recorded_traffic(wl_name, wl, "fetch_kernel" if link else "scan_kernel")
    roofline = {"bound": bound, "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": traffic, "traffic_source": traffic_note,
                "kernel": kernel,
                "peak_source": peak_note, "avg_launch_us": avg_launch_ms * 1e3,
                # the whole step against the same peak: every plan's union bytes
                # over the device-timed step (fetch, scoring, selection, plans)
                "step_level_frac": union_bytes_total / (total_ms / K / 1e3) / 1e9 / peak,
                "algorithmic_bytes_per_launch": bytes_per_launch}

    cfg = config_of(wl_name, wl, "flushed between steps (256 MiB write)",
                    sessions=sessions if wl.get("sessions") else None)
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": total_ms / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": cfg,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h,
                    "launch_mode": "cuda_graph" if args.graph else "eager"},
            "gpu_launches": int(launches), "launch_mode": "cuda_graph" if args.graph else "eager",
            "roofline": roofline, "clocks": clk,
            "per_plan": per_plan,
            "step_ms_median": statistics.median(step_ms)}
    if link is not None:
        line["host_link"] = link
    return line


def run_append(args, wl_name, wl):
    """Append path: K timed appends of m keys per KV head for each m of the
    workload (after W warm-up appends), each timed with CUDA events; the
    index is packed with room for all of them.  Roofline: the append reads
    its keys (H*m*d*4 bytes) and read-modify-writes the touched plane words
    (2 * H*d*4 slots * words * 4 bytes), against measured HBM."""
    import torch
    import decode_fathom_plan_b200 as fp
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    fp.load_library()
    H, G, n, d = wl["H"], wl["G"], wl["n"], wl["d"]
    W, K = max(3, args.warmup), args.steps
    results = []
    e2e = None
    for m in wl["append"]:
        total = n + (W + K) * m
        sigma, _ = synth.channel_sigma(rank, H, d)
        keys = synth.device_keys(torch, sigma, total, rank)
        # room for K more appends of the end-to-end leg below
        index = fp.KeyIndex(H, G, n, d, wl["residency"], capacity=total + K * m)
        index.pack(keys[:, :n].contiguous())
        chunks = [keys[:, n + i * m:n + (i + 1) * m].contiguous() for i in range(W + K)]
        clamped = torch.zeros((H, d), dtype=torch.int32, device="cuda")
        torch.cuda.synchronize()
        for i in range(W):
            index.append(chunks[i], clamped)
        # the K timed appends as one CUDA graph (each append's key count is
        # fixed at capture; replaying once performs each exactly once), so the
        # events time the device, not the host's launch path
        ev = [(torch.cuda.Event(enable_timing=True, external=True),
               torch.cuda.Event(enable_timing=True, external=True)) for _ in range(K)]
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            with torch.cuda.graph(graph, stream=side, capture_error_mode="relaxed"):
                for i in range(K):
                    ev[i][0].record()
                    index.append(chunks[W + i], clamped)
                    ev[i][1].record()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        del graph
        assert fp.fathom_last_device_status() == fp.FATHOM_OK
        ms = [a.elapsed_time(b) for a, b in ev]
        med = statistics.median(ms)
        words = m // 32 + 2
        nbytes = H * m * d * 4 + 2 * H * d * 4 * words * 4
        results.append({"m": m, "us_per_append_median": med * 1e3,
                        "keys_per_s": H * m / (med / 1e3),
                        "bytes_per_append": nbytes,
                        "achieved_gbs": nbytes / (med / 1e3) / 1e9,
                        "clamped_keys_total": int(clamped.sum().item())})
        # end to end through the public call: each step copies its m keys per
        # KV head in from pinned host memory, appends, and reads the clamp
        # counters back (host clock)
        host_chunk = chunks[-1].cpu().pin_memory()
        stage = torch.empty_like(chunks[-1])
        cl_host = torch.empty((H, d), dtype=torch.int32).pin_memory()
        e2e_s = []
        for i in range(K):
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            stage.copy_(host_chunk, non_blocking=True)
            index.append(stage, clamped)
            cl_host.copy_(clamped, non_blocking=True)
            torch.cuda.synchronize()
            e2e_s.append(time.perf_counter() - t0)
        assert fp.fathom_last_device_status() == fp.FATHOM_OK
        e2e = {"value": H * m * K / sum(e2e_s) / 1e9, "unit": "Gkeys/s",
               "h2d_bytes_per_step": H * m * d * 4, "d2h_bytes_per_step": H * d * 4,
               "launch_mode": "eager", "m": m}
        del keys, index, chunks
    peak, peak_src = load_peaks()
    bulk = results[-1]
    line = {"metric": "KV-head keys appended per second (append path)",
            "value": bulk["keys_per_s"] / 1e9, "unit": "Gkeys/s", "n_gpus": 1, "steps": K,
            "warmup": W, "ms_per_step": bulk["us_per_append_median"] / 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": {"workload": wl_name, "kv_heads": H, "head_dim": d,
                                            "n_keys_packed": n, "appends": list(wl["append"])},
            "roofline": {"bound": "hbm", "achieved": bulk["achieved_gbs"], "peak": peak,
                         "unit": "GB/s", "frac": bulk["achieved_gbs"] / peak, "traffic": None,
                         "kernel": f"append_kernel (m = {bulk['m']})",
                         "peak_source": f"{peak_src} hbm_gbs (MEASURED_PEAKS.json)"},
            "e2e": e2e, "per_m": results, "launch_mode": "cuda_graph"}
    print(json.dumps(line), flush=True)


def run_attention_bench(args, wl_name, wl):
    """Attention over the selected keys: for each plan, plan + scan once, then
    K timed attention calls over that top-k (one CUDA graph, CUDA events per
    call).  Roofline: the attention reads k K rows and k V rows per query
    (Q*k*2*d*4 bytes).  Quality: relative L2 error of the output against
    dense attention over all n keys (torch, outside the path), beside the
    error of attention over the exact fp32 top-k (the best k keys)."""
    import torch
    import decode_fathom_plan_b200 as fp
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    fp.load_library()
    H, G, n, d, k = wl["H"], wl["G"], wl["n"], wl["d"], wl["k"]
    Q = H * G
    W, K = max(3, args.warmup), args.steps
    ses = synth.make_session(rank, H, G, n, 64, head_dim=d)
    keys = torch.from_numpy(ses.keys).cuda()
    gen = torch.Generator(device="cuda")
    gen.manual_seed(10_000 + rank)
    values = torch.randn((H, n, d), generator=gen, device="cuda", dtype=torch.float32)
    index = fp.KeyIndex(H, G, n, d, "device")
    index.pack(keys)
    q = torch.from_numpy(synth.draw_queries(20_000 + rank, Q, d, count=1)[0].view(np.int16)).cuda()
    scale = 1.0 / float(np.sqrt(d))
    out = torch.empty((Q, d), dtype=torch.float32, device="cuda")
    ws = torch.empty(fp.fathom_sparse_attention_workspace_bytes(Q, d, k), dtype=torch.uint8,
                     device="cuda")
    qf = q.view(torch.bfloat16).float().reshape(H, G, d)

    def attend(idx):
        fp.fathom_sparse_attention(keys, values, H, G, d, n, q, idx, k, scale, out, ws)

    with torch.no_grad():
        logits = torch.einsum("hnd,hgd->hgn", keys, qf) * scale          # [H][G][n]
        dense = torch.einsum("hgn,hnd->hgd", torch.softmax(logits, dim=-1), values)
        exact_idx = logits.topk(k, dim=-1).indices.reshape(Q, k).int().contiguous()
    attend(exact_idx)
    torch.cuda.synchronize()
    o_exactk = out.clone().reshape(H, G, d)

    def rel_err(o):
        return float(((o - dense).norm(dim=-1) / dense.norm(dim=-1)).mean())

    per_plan, times = [], []
    for spec in wl["plans"]:
        buf = fp.ScanBuffers(index, k)
        bvec = torch.full((Q,), plan_bits(spec), dtype=torch.int32, device="cuda")
        fp.plan_and_scan(index, q, bvec, buf, fixed_r=spec[1] if spec[0] == "fixed" else None)
        for _ in range(W):
            attend(buf.idx)
        ev = [(torch.cuda.Event(enable_timing=True, external=True),
               torch.cuda.Event(enable_timing=True, external=True)) for _ in range(K)]
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            with torch.cuda.graph(graph, stream=side, capture_error_mode="relaxed"):
                for i in range(K):
                    ev[i][0].record()
                    attend(buf.idx)
                    ev[i][1].record()
        torch.cuda.current_stream().wait_stream(side)
        graph.replay()
        torch.cuda.synchronize()
        del graph
        assert fp.fathom_last_device_status() == fp.FATHOM_OK
        ms = statistics.median([a.elapsed_time(b) for a, b in ev])
        times.append(ms)
        per_plan.append({"plan": plan_name(spec), "bits_per_key": plan_bits(spec),
                         "attention_us": ms * 1e3,
                         "attention_error_vs_dense": rel_err(out.reshape(H, G, d)),
                         "recall_vs_exact_fp32": float(np.mean([
                             len(np.intersect1d(buf.idx[i].cpu().numpy(),
                                                exact_idx[i].cpu().numpy())) / k
                             for i in range(Q)]))})
    # end to end through the public call: each step copies the queries and the
    # selected indices in from pinned host memory, attends, and copies the
    # outputs back (host clock)
    q_host = q.cpu().pin_memory()
    idx_host = buf.idx.cpu().pin_memory()
    idx_stage = torch.empty_like(buf.idx)
    out_host = torch.empty((Q, d), dtype=torch.float32).pin_memory()
    e2e_s = []
    for i in range(K):
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        q.copy_(q_host, non_blocking=True)
        idx_stage.copy_(idx_host, non_blocking=True)
        attend(idx_stage)
        out_host.copy_(out, non_blocking=True)
        torch.cuda.synchronize()
        e2e_s.append(time.perf_counter() - t0)
    assert fp.fathom_last_device_status() == fp.FATHOM_OK
    nbytes = Q * k * 2 * d * 4
    ms = statistics.median(times)
    peak, peak_src = load_peaks()
    line = {"metric": "sparse attention over the selected keys: KV-head keys attended per second",
            "value": Q * k / (ms / 1e3) / 1e9, "unit": "Gkeys/s", "n_gpus": 1, "steps": K,
            "warmup": W, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": wl_name, "kv_heads": H, "query_heads_per_kv": G,
                       "head_dim": d, "n_keys": n, "k": k,
                       "plans": [plan_name(p) for p in wl["plans"]]},
            "roofline": {"bound": "hbm", "achieved": nbytes / (ms / 1e3) / 1e9, "peak": peak,
                         "unit": "GB/s", "frac": nbytes / (ms / 1e3) / 1e9 / peak,
                         "traffic": None, "kernel": "attention_split_kernel + combine",
                         "peak_source": f"{peak_src} hbm_gbs (MEASURED_PEAKS.json)",
                         "algorithmic_bytes_per_launch": nbytes},
            "attention_error_exact_topk_vs_dense": rel_err(o_exactk),
            "e2e": {"value": Q * k * K / sum(e2e_s) / 1e9, "unit": "Gkeys/s",
                    "h2d_bytes_per_step": Q * d * 2 + Q * k * 4,
                    "d2h_bytes_per_step": Q * d * 4, "launch_mode": "eager"},
            "per_plan": per_plan, "launch_mode": "cuda_graph"}
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    wl = WORKLOADS[args.workload]
    if wl.get("attention"):
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable":
                              "the attention workload has no CPU reference leg"}))
        else:
            run_attention_bench(args, args.workload, wl)
        return
    if wl.get("append"):
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable":
                              "the append workload has no CPU reference leg"}))
        else:
            run_append(args, args.workload, wl)
        return
    if args.impl == "reference":
        run_reference(args, args.workload, wl)
    else:
        run_fathom(args, args.workload, wl)


if __name__ == "__main__":
    main()

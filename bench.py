"""Benchmark of the BeaconKV compression step on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl bkv|reference]

One step = one whole compression step (Continual FPS over the newest window,
tensor-core scoring with max aggregation, top-K, compaction) over every
(layer, KV head) of the workload, through the C ABI (bkv_compress_step), with
the inputs resident in HBM.  For N > 1 (launched with torch.distributed.run)
every rank compresses its own independent cache of the same shape (weak
scaling; the heads are independent, so no collective is on the data path);
the timed region is bracketed by a barrier and a device synchronise on every
rank and the slowest rank's time is reported.

Rank 0 prints one JSON line.  `value` is the number of KV entries (layer, KV
head, position) scored, selected and compacted per second by all ranks.
`e2e` is the same metric when each step also copies its inputs from pinned
host memory and reads the compacted cache back.  `roofline` is the dominant
kernel's achieved rate against the measured B200 peak; `cpu_baseline` is the
float64 oracle timed on a bounded sample on this host.  `--impl reference`
times only that oracle (the baseline arm).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import shutil
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "KV entries scored+selected+compacted/s per compression step"
UNIT = "entries/s"
PHASES = ["fps", "row_stats", "aggregate", "select", "compact"]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=p["hbm_gbs"], bf16_tflops=p["bf16_tflops"],
                    bf16_tflops_sustained=p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                    sm_max_mhz=p.get("sm_max_mhz", 1965.0), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0,
                sm_max_mhz=1965.0, source="fallback")


def load_traffic():
    """DRAM bytes per launch of each phase's kernel from profiles/traffic.json
    (an ncu capture), or None for a kernel whose sources changed since."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return {}
    with open(path) as f:
        rec = json.load(f)
    out = {}
    for phase, r in rec.items():
        m = hashlib.sha256()
        try:
            for src in r["sources"]:
                with open(os.path.join(ROOT, src), "rb") as f:
                    m.update(f.read())
        except OSError:
            continue
        out[phase] = r["bytes_per_launch"] if m.hexdigest() == r["sha256"] else None
    return out


# ----------------------------------------------------------------------------
# algorithmic work per phase (per step, one rank)
# ----------------------------------------------------------------------------
def work_model(wl, aggregate="max"):
    H = wl.n_layers * wl.n_kv_heads
    Hq = wl.n_layers * wl.n_q_heads
    nb = min(wl.M, wl.beacons_in + wl.W) if wl.W else wl.beacons_in
    n_obs = wl.group * (wl.R + nb)
    d, L, K = wl.head_dim, wl.L, min(wl.K, wl.L)
    es = 2 if wl.dtype == "bf16" else 4
    # the words the select streams per key: one (the max form's merged order
    # key, or the CUDA-core path's single partial), else one partial per
    # group of at most 256 observation rows (the tensor-core mean)
    n_parts = (n_obs + 255) // 256 if aggregate == "mean" and wl.dtype == "bf16" else 1
    contraction = 2.0 * n_obs * L * d * H
    fps_fma = float(Hq) * wl.M * (wl.beacons_in + wl.W) * d
    return {
        # each pick's distance to every point of the union, once: the dot
        # products run on the bf16 tensor cores, so they count as 2 FLOP per
        # FMA against the bf16 peak (fps_fma keeps the FMA count itself)
        "fps": {"bound": "tensor", "work": 2.0 * fps_fma, "unit": "FLOP"},
        "fps_fma": fps_fma,
        "row_stats": {"bound": "tensor", "work": contraction, "unit": "FLOP"},
        "aggregate": {"bound": "tensor", "work": contraction, "unit": "FLOP"},
        "select": {"bound": "hbm", "work": float(H) * (n_parts * 4 * L + 4 * K), "unit": "B"},
        "compact": {"bound": "hbm", "work": float(H) * 4 * K * d * es, "unit": "B"},
        # the step: one contraction + the algorithmic bytes of the whole step
        "step_flop": contraction,
        "step_bytes": float(H) * (L * d * es + n_obs * d * es + 2 * 4 * L + 2 * 4 * K
                                  + 4 * K * d * es),
        # the row normalisers need one exp per logit
        "step_exps": float(H) * n_obs * L,
    }


def mufu_bound_s(wm, peaks):
    """The exps of the step on the MUFU units alone (16 ex2 per clock per SM,
    148 SMs, the max SM clock): a third bound beside the tensor and HBM ones,
    which the row statistics beat by taking part of the exps on the FMA pipe."""
    return wm["step_exps"] / (16 * 148 * peaks["sm_max_mhz"] * 1e6)


def peak_for(bound, peaks):
    """The denominator of a phase's fraction.  The step takes a few ms and the
    timed region a fraction of a second, so a kernel's rate is held against
    the burst bf16 peak (the sustained figure is for seconds-long loops)."""
    if bound == "tensor":
        return peaks["bf16_tflops"], "TFLOP/s"
    if bound == "hbm":
        return peaks["hbm_gbs"], "GB/s"
    raise ValueError(bound)


def fp32_fma_peak_tfma(peaks):
    """FP32 FMA pipe, derived from unit counts: 148 SMs x 128 FMA per clock at
    the max SM clock (not a measured figure)."""
    return 148 * 128 * peaks["sm_max_mhz"] * 1e6 / 1e12


def rate(work, unit, seconds):
    if unit == "FLOP":
        return work / seconds / 1e12
    if unit == "B":
        return work / seconds / 1e9
    return work / seconds / 1e12


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.path = None
        self.err = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            self.sel = []

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="bkv_clocks_", suffix=".csv")
        os.close(fd)
        exe = shutil.which("nvidia-smi") or "/usr/bin/nvidia-smi"
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                [exe, *self.sel, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception as e:  # noqa: BLE001
            self.proc = None
            self.err = type(e).__name__ + ": " + str(e)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None,
                    "reasons": ["nvidia-smi unavailable (%s)" % self.err]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        if not rows:
            with open(self.path) as f:
                head = f.read(200).strip().replace("\n", " ")
            os.unlink(self.path)
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples: " + head]}
        os.unlink(self.path)
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ----------------------------------------------------------------------------
# the float64 oracle on a bounded sample (CPU baseline / reference arm)
# ----------------------------------------------------------------------------
def oracle_sample(wl, seed: int, n_heads: int, L_sample: int, aggregate: str = "max"):
    """Run the oracle's whole step on n_heads (layer, KV head)s, one thread
    each, with each head's keys cut to its first L_sample rows.  Returns
    (entries, seconds, threads)."""
    import oracle
    from kv_cache_compression_bkv_b200 import synth

    wls = wl.replace(L=L_sample, capacity=L_sample, K=min(wl.K, L_sample))
    jobs = []
    for i in range(n_heads):
        l, h = divmod(i, wl.n_kv_heads)
        l %= wl.n_layers
        k, v = synth.keys_values(wls, seed, l, h)
        qs = [synth.head_queries(wls, seed, l, h * wl.group + g) for g in range(wl.group)]
        recent = np.stack([q[0].to(wls.torch_dtype).double().numpy() for q in qs])
        beac = np.stack([q[1].to(wls.torch_dtype).double().numpy() for q in qs])
        win = np.stack([q[2].to(wls.torch_dtype).double().numpy() for q in qs]) if wl.W else None
        jobs.append((k.to(wls.torch_dtype).double().numpy(), v.to(wls.torch_dtype).double().numpy(),
                     recent, beac, win))
    oracle.lib()
    done = []

    def run(job):
        k, v, r, b, w = job
        out = oracle.compress_head(k, v, r, b, wls.beacons_in, w, wls.M, wls.K,
                                   aggregate=aggregate)
        done.append(len(out["idx"]))

    threads = [threading.Thread(target=run, args=(j,)) for j in jobs]
    t0 = time.perf_counter()
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    dt = time.perf_counter() - t0
    return n_heads * L_sample, dt, len(threads)


def workload_config(wl, args) -> dict:
    cfg = {"workload": wl.name, "n_layers": wl.n_layers, "n_q_heads": wl.n_q_heads,
           "n_kv_heads": wl.n_kv_heads, "head_dim": wl.head_dim, "L": wl.L, "R": wl.R,
           "M": wl.M, "K": wl.K, "W": wl.W}
    if args.aggregate != "max":
        cfg["aggregate"] = args.aggregate
    if getattr(args, "in_place", False):
        cfg["compaction"] = "in place"
    return cfg


def max_over_ranks(x: float, dist, device) -> float:
    """The largest of every rank's x (the slowest rank's time); x itself
    without a process group.  Every rank must call it at the same point."""
    if dist is None:
        return x
    tt = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt.item())


def weak_scaling_value(entries_per_rank: int, world: int, ms_max: float) -> float:
    """Entries processed by all ranks per second, timed by the slowest rank."""
    return world * entries_per_rank / (ms_max / 1e3)


def cpu_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def run_reference(args, wl, rank, world):
    """The reference arm: the float64 oracle as it stands, on the workload's
    full shape (every head's L keys, window and beacons), one (layer, KV head)
    per host thread.  Each step is a bounded sample of the workload: one
    full-size head per host core, run side by side (about 5 s a step for the
    14B-shaped workload)."""
    if rank != 0:
        return
    n_cores = cpu_threads()
    n_heads = max(1, min(wl.n_layers * wl.n_kv_heads, n_cores))
    for _ in range(args.warmup):
        oracle_sample(wl, args.seed, n_heads, wl.L, args.aggregate)
    tot_e, tot_t = 0, 0.0
    for _ in range(args.steps):
        e, t, _ = oracle_sample(wl, args.seed, n_heads, wl.L, args.aggregate)
        tot_e += e
        tot_t += t
    value = tot_e / tot_t
    sample = (f"per step: {n_heads} (layer, KV head)s of {wl.name} at full size (all L={wl.L} "
              f"keys, FPS over the {wl.W}-query window and the beacons, top-K, compaction), "
              f"one thread per head on {n_cores} host cores")
    n_thr = n_heads
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * tot_t / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(wl, args),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": n_thr, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# Continual FPS against naive FPS over the whole query history (Fig. 7)
# ----------------------------------------------------------------------------
def fps_sweep(args, wl):
    """Time bkv_update_beacons on the workload's query heads for Continual FPS
    (beacons + the window since the last step) and for naive FPS over the
    whole history of each length in --fps-sweep (no beacons).  One JSON line."""
    from kv_cache_compression_bkv_b200 import bkv, synth

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    hist = [int(x) for x in args.fps_sweep.split(",") if x]
    cases = [("continual", wl.beacons_in, wl.W)] + [("naive", 0, h) for h in hist]
    w_max = max(W for _, _, W in cases)
    Ly, Hq, d, M = wl.n_layers, wl.n_q_heads, wl.head_dim, wl.M
    dt = wl.torch_dtype
    # each query head's history, newest last; a window is its last W rows
    history = torch.empty(Ly, Hq, w_max, d, dtype=dt, device=dev)
    beacons = torch.empty(Ly, Hq, M, d, dtype=dt, device=dev)
    for l in range(Ly):
        for qh in range(Hq):
            history[l, qh] = synth.queries(wl, args.seed, l, qh, w_max, 3).to(dt).to(dev)
            b = torch.zeros(M, d)
            if wl.beacons_in:
                b[:wl.beacons_in] = synth.queries(wl, args.seed, l, qh, wl.beacons_in, 5)
            beacons[l, qh] = b.to(dt).to(dev)
    g = bkv.Geometry(Ly, Hq, wl.n_kv_heads, d, 1, dt)
    out = []
    for name, nb, W in cases:
        window = history[:, :, w_max - W:].contiguous()
        bout = torch.empty_like(beacons)
        ws = torch.empty(max(1, bkv.bkv_workspace_size(g, 1, 0, M, W, 1)), dtype=torch.uint8,
                         device=dev)
        stream = torch.cuda.current_stream()

        def call():
            return bkv.bkv_update_beacons(g, beacons if nb else None, nb, M, window, W, bout,
                                          ws, stream)

        for _ in range(max(1, args.warmup)):
            call()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = max(1, min(args.steps, 5))
        e0.record(stream)
        for _ in range(reps):
            call()
        e1.record(stream)
        torch.cuda.synchronize()
        st, where = bkv.bkv_read_device_status()
        if st != 0:
            raise RuntimeError(f"device status {st} at {where}")
        ms = e0.elapsed_time(e1) / reps
        n = nb + W
        out.append({"fps": name, "beacons_in": nb, "W": W, "union": n, "ms": ms,
                    "union_bytes_per_step": Ly * Hq * n * d * dt.itemsize,
                    "query_store_bytes": Ly * Hq * (M + W if name == "continual" else W) * d
                                         * dt.itemsize})
        del window, ws, bout
    line = {"metric": "Continual vs naive FPS (bkv_update_beacons)", "unit": "ms",
            "workload": wl.name, "n_layers": Ly, "n_q_heads": Hq, "M": M,
            "higher_is_better": False, "data": "synthetic", "sweep": out}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# Table 1's (n_recent, n_beacon) trade-off: the step's time per split
# ----------------------------------------------------------------------------
def rm_sweep(args, wl):
    """Time the whole step for each (R, M) split in --rm-sweep ("R:M,..."),
    the beacons full and the budget --budget; the keys and values are shared
    by every split.  One JSON line."""
    from kv_cache_compression_bkv_b200 import bkv, synth

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    pairs = [tuple(int(x) for x in p.split(":")) for p in args.rm_sweep.split(",") if p]
    base = wl.replace(K=args.budget, n_beacons_in=-1)
    kv = synth.make_step_inputs(base.replace(R=1, M=1, W=0), seed=args.seed)
    k, v = kv.k.to(dev), kv.v.to(dev)
    g = bkv.geometry_of(k, wl.n_q_heads)
    keep = min(base.K, base.L)
    dstg = bkv.Geometry(g.n_layers, g.n_q_heads, g.n_kv_heads, g.head_dim, keep, g.dtype)
    kd = torch.empty(wl.n_layers, wl.n_kv_heads, keep, wl.head_dim, dtype=k.dtype, device=dev)
    vd = torch.empty_like(kd)
    idx = torch.empty(wl.n_layers, wl.n_kv_heads, keep, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()
    out = []
    for R, M in pairs:
        wp = base.replace(R=R, M=M)
        Ly, Hq, d, dt = wp.n_layers, wp.n_q_heads, wp.head_dim, wp.torch_dtype
        recent = torch.empty(Ly, Hq, R, d, dtype=dt)
        beacons = torch.empty(Ly, Hq, M, d, dtype=dt)
        window = torch.empty(Ly, Hq, wp.W, d, dtype=dt)
        for l in range(Ly):
            for qh in range(Hq):
                r_, b_, w_ = synth.head_queries(wp, args.seed, l, qh)
                recent[l, qh], beacons[l, qh] = r_.to(dt), b_.to(dt)
                if wp.W:
                    window[l, qh] = w_.to(dt)
        recent, beacons, window = recent.to(dev), beacons.to(dev), window.to(dev)
        bout = torch.empty_like(beacons)
        ws = torch.empty(bkv.bkv_workspace_size(g, wp.L, R, M, wp.W, wp.K), dtype=torch.uint8,
                         device=dev)

        def step(events=None):
            bkv.bkv_compress_step(g, k, v, wp.L, wp.K, recent, R, beacons, M, M,
                                  window if wp.W else None, wp.W, bout, 0.0, dstg, kd, vd,
                                  None, idx, ws, stream, events)

        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(bkv.STEP_EVENTS)]
              for _ in range(args.steps)]
        for row in ev:
            for e in row:
                e.record(stream)
        torch.cuda.synchronize()
        for i in range(args.steps):
            step(ev[i])
        torch.cuda.synchronize()
        st, where = bkv.bkv_read_device_status()
        if st != 0:
            raise RuntimeError(f"device status {st} at {where}")
        ph = {p: sum(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(args.steps)) / args.steps
              for j, p in enumerate(PHASES)}
        total = sum(ev[i][0].elapsed_time(ev[i][-1]) for i in range(args.steps)) / args.steps
        out.append({"n_recent": R, "n_beacon": M, "ms": total, "phases_ms": ph})
    line = {"metric": "compression step time vs (n_recent, n_beacon)", "unit": "ms",
            "workload": wl.name, "K": base.K, "L": base.L, "W": base.W,
            "higher_is_better": False, "data": "synthetic", "sweep": out}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# the CUDA path
# ----------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="qwen3_14b")
    ap.add_argument("--impl", default="bkv", choices=["bkv", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=None,
                    help="use only this many layers (small cases for profiler captures)")
    ap.add_argument("--aggregate", default="max", choices=["max", "mean"],
                    help="aggregation over the observation rows (mean: Table 2's ablation)")
    ap.add_argument("--overlap", action="store_true",
                    help="give the step a second stream: each head batch's top-K and compaction "
                         "overlap the next batch's aggregation (measured slower on B200 than one "
                         "stream, so off by default)")
    ap.add_argument("--in-place", action="store_true",
                    help="compact into the scored cache itself (bkv_compress_step with "
                         "k_dst == k)")
    ap.add_argument("--rm-sweep", default=None,
                    help="comma-separated R:M splits (Table 1): time the step for each")
    ap.add_argument("--budget", type=int, default=2048, help="K for --rm-sweep")
    ap.add_argument("--fps-sweep", default=None,
                    help="comma-separated history lengths: time Continual FPS against naive "
                         "FPS over each whole history instead of the step")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    from kv_cache_compression_bkv_b200 import synth
    wl = synth.WORKLOADS[args.workload]
    if args.layers:
        wl = wl.replace(n_layers=args.layers)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, wl, rank, world)
        return
    if args.fps_sweep:
        fps_sweep(args, wl)
        return
    if args.rm_sweep:
        rm_sweep(args, wl)
        return

    from kv_cache_compression_bkv_b200 import bkv

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    def barrier():
        if dist is not None:
            dist.barrier()

    inp = synth.make_step_inputs(wl, seed=args.seed + rank, pin=True)
    g = bkv.geometry_of(inp.k, wl.n_q_heads)
    keep = min(wl.K, wl.L)
    dstg = bkv.Geometry(g.n_layers, g.n_q_heads, g.n_kv_heads, g.head_dim, keep, g.dtype)
    names = ("k", "v", "recent", "beacons", "window")
    host = {n: getattr(inp, n) for n in names}
    devt = {n: torch.empty_like(host[n], device=dev) for n in names}
    for n in names:
        devt[n].copy_(host[n])
    if args.in_place:
        # the step compacts the cache it scored (each timed step then sees the
        # previous step's result: the same work on other data)
        dstg = g
        kd, vd = devt["k"][:, :, :keep], devt["v"][:, :, :keep]
    else:
        kd = torch.empty(wl.n_layers, wl.n_kv_heads, keep, wl.head_dim, dtype=inp.k.dtype,
                         device=dev)
        vd = torch.empty_like(kd)
    bout = torch.empty_like(devt["beacons"])
    idx = torch.empty(wl.n_layers, wl.n_kv_heads, keep, dtype=torch.int32, device=dev)
    ws = torch.empty(bkv.bkv_workspace_size(g, wl.L, wl.R, wl.M, wl.W, wl.K), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream()
    # the second stream on which each head batch's top-K and compaction overlap
    # the next batch's aggregation (high priority: its CTAs go first)
    aux = torch.cuda.Stream(device=dev, priority=-1) if args.overlap else None

    def step(events=None, t=devt, o=None, st=None, overlap=True):
        o = o or {"kd": kd, "vd": vd, "bout": bout, "idx": idx}
        return bkv.bkv_compress_step(g, t["k"], t["v"], wl.L, wl.K, t["recent"], wl.R,
                                     t["beacons"], wl.beacons_in, wl.M,
                                     t["window"] if wl.W else None, wl.W, o["bout"], 0.0, dstg,
                                     o["kd"], o["vd"], None, o["idx"], ws, st or stream, events,
                                     aggregate=args.aggregate,
                                     aux_stream=aux if overlap else None)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st, where = bkv.bkv_read_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} at {where} during warm-up")

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(bkv.STEP_EVENTS)]
          for _ in range(args.steps)]
    # torch creates an event lazily and refuses elapsed_time() on events it did
    # not record itself: record each once here; the library re-records them
    for row in ev:
        for e in row:
            e.record(stream)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.25)
    t_start.record(stream)
    for i in range(args.steps):
        step(ev[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    st, where = bkv.bkv_read_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} at {where} in the timed region")
    ms_local = t_start.elapsed_time(t_end) / args.steps
    phase_ms = {p: sum(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(args.steps)) / args.steps
                for j, p in enumerate(PHASES)}
    overlap_info = None
    if aux is not None:
        # with the overlap, events [3]..[5] bound only the part of the top-K and
        # compaction left after the last aggregation batch; each kernel's own
        # time comes from a few more steps run on one stream (after the timed
        # region, untimed for `value`)
        overlap_info = {"aggregate_ms": phase_ms["aggregate"],
                        "exposed_select_compact_ms": phase_ms["select"] + phase_ms["compact"]}
        n_iso = max(1, min(args.steps, 10))
        ev_iso = [[torch.cuda.Event(enable_timing=True) for _ in range(bkv.STEP_EVENTS)]
                  for _ in range(n_iso)]
        for row in ev_iso:
            for e in row:
                e.record(stream)
        for i in range(n_iso):
            step(ev_iso[i], overlap=False)
        torch.cuda.synchronize()
        phase_ms = {p: sum(ev_iso[i][j].elapsed_time(ev_iso[i][j + 1]) for i in range(n_iso))
                    / n_iso for j, p in enumerate(PHASES)}
        overlap_info["one_stream_step_ms"] = sum(
            ev_iso[i][0].elapsed_time(ev_iso[i][-1]) for i in range(n_iso)) / n_iso
    ms = max_over_ranks(ms_local, dist, dev)
    entries = wl.n_layers * wl.n_kv_heads * wl.L
    value = weak_scaling_value(entries, world, ms)

    # ---- end to end: pinned host inputs in, compacted cache out, every step.
    # Steps are pipelined over three streams as a serving loop would: step
    # i+1's inputs upload (into the other of two device input sets) while
    # step i computes and step i-1's outputs download (from the other of two
    # output sets); each step's copies and compute still all happen.
    e2e_steps = args.e2e_steps or max(3, min(args.steps, 10))
    ins = [devt, {n: torch.empty_like(devt[n]) for n in names}]
    if args.in_place:
        outs = [{"kd": ins[b]["k"][:, :, :keep], "vd": ins[b]["v"][:, :, :keep],
                 "bout": bout if b == 0 else torch.empty_like(bout),
                 "idx": idx if b == 0 else torch.empty_like(idx)} for b in range(2)]
    else:
        outs = [{"kd": kd, "vd": vd, "bout": bout, "idx": idx},
                {"kd": torch.empty_like(kd), "vd": torch.empty_like(vd),
                 "bout": torch.empty_like(bout), "idx": torch.empty_like(idx)}]
    out_host = {n: torch.empty(outs[0][n].shape, dtype=outs[0][n].dtype).pin_memory()
                for n in ("kd", "vd", "bout", "idx")}
    h2d = sum(host[n].numel() * host[n].element_size() for n in names if n != "window" or wl.W)
    d2h = sum(t.numel() * t.element_size() for t in out_host.values())
    s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(e2e_steps)]
    ev_done = [torch.cuda.Event() for _ in range(e2e_steps)]
    ev_out = [torch.cuda.Event() for _ in range(e2e_steps)]
    barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_up.wait_stream(stream)
    s_down.wait_stream(stream)
    for i in range(e2e_steps):
        b = i & 1
        with torch.cuda.stream(s_up):
            if i >= 2:
                s_up.wait_event(ev_done[i - 2])  # input set b is free again
            for n in names:
                if n != "window" or wl.W:
                    ins[b][n].copy_(host[n], non_blocking=True)
            ev_in[i].record(s_up)
        stream.wait_event(ev_in[i])
        if i >= 2:
            stream.wait_event(ev_out[i - 2])  # output set b has been read back
        step(t=ins[b], o=outs[b], st=stream)
        ev_done[i].record(stream)
        with torch.cuda.stream(s_down):
            s_down.wait_event(ev_done[i])
            for n in ("kd", "vd", "bout", "idx"):
                out_host[n].copy_(outs[b][n], non_blocking=True)
            ev_out[i].record(s_down)
    stream.wait_stream(s_down)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dist, dev)

    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return

    peaks = load_peaks()
    wm = work_model(wl, args.aggregate)
    # the captured counters are those of the default configuration
    traffic = (load_traffic() if args.workload == "qwen3_14b" and not args.layers
               and args.aggregate == "max" and not args.in_place else {})
    phases = {}
    for p in PHASES:
        m = wm[p]
        pk, pu = peak_for(m["bound"], peaks)
        sec = phase_ms[p] / 1e3
        ach = rate(m["work"], m["unit"], sec) if sec > 0 else 0.0
        phases[p] = {"ms": phase_ms[p], "bound": m["bound"], "achieved": ach, "peak": pk,
                     "unit": pu, "frac": ach / pk if pk else None,
                     "traffic": traffic.get(p)}
    dom = max(PHASES, key=lambda p: phase_ms[p])
    dm = phases[dom]
    per_launch = wm[dom]["work"]
    if "fps" in phases and phase_ms["fps"] > 0:
        # the same FPS work as FMAs against the (derived) FP32 FMA pipe peak
        fma_rate = wm["fps_fma"] / (phase_ms["fps"] / 1e3) / 1e12
        phases["fps"]["fma_tfma_s"] = fma_rate
        phases["fps"]["fma_frac_of_derived_fp32_peak"] = fma_rate / fp32_fma_peak_tfma(peaks)
    roofline = {"bound": dm["bound"], "achieved": dm["achieved"], "peak": dm["peak"],
                "unit": dm["unit"], "frac": dm["frac"], "traffic": traffic.get(dom), "kernel": dom,
                "peak_source": peaks["source"] + (" burst" if dm["bound"] == "tensor" else ""),
                "work_per_launch": per_launch}
    t_tensor = wm["step_flop"] / (peaks["bf16_tflops"] * 1e12)
    t_hbm = wm["step_bytes"] / (peaks["hbm_gbs"] * 1e9)
    t_roof = max(t_tensor, t_hbm)

    # the library's kernels per step: FPS, row statistics, then one
    # aggregation per head batch (4 with the overlap) and as many top-K and
    # compaction launches
    n_batches = 1 if aux is None else min(4, wl.n_layers * wl.n_kv_heads)
    gpu_launches = ((1 if wl.W else 0) + 1 + 3 * n_batches) * args.steps
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        n_thr = cpu_threads()
        e, t, used = oracle_sample(wl, args.seed, n_thr, wl.L, args.aggregate)
        cpu = {"value": e / t, "unit": UNIT, "cores": used, "kind": "oracle",
               "sample": f"{n_thr} (layer, KV head)s of {wl.name} at full size, the whole step "
                         f"each (FPS over W={wl.W}, scoring all L={wl.L} keys, top-K, "
                         f"compaction), one thread per head on {n_thr} host cores, "
                         f"{t:.1f} s wall"}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": dict(workload_config(wl, args),
                       l2="inputs larger than L2 (K/V cache %.1f GB per step)"
                          % (2 * inp.k.numel() * inp.k.element_size() / 1e9)),
        "step_us": ms * 1e3,
        "pct_roofline": 100.0 * t_roof / (ms / 1e3),
        "t_roof_us": t_roof * 1e6,
        "t_mufu_us": mufu_bound_s(wm, peaks) * 1e6,
        "roofline": roofline,
        "phases": phases,
        "cpu_baseline": cpu,
        "e2e": {"value": weak_scaling_value(entries, world, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "clocks": clk,
        "gpu_launches": gpu_launches,
    }
    if overlap_info is not None:
        line["overlap"] = dict(overlap_info, note=(
            "each of 4 head batches' top-K and compaction run on a second stream while the next "
            "batch is aggregated; phases give each kernel's time measured on one stream"))
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

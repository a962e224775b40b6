#!/usr/bin/env python
"""Benchmark of the persistent MoE decode-layer step on B200.

Prints ONE JSON line (rank 0). The metric is the layer step's µs/step and the
HBM bandwidth it sustains over the bytes the step must touch (router, shared
expert, and each selected expert once however many rows chose it), against the
measured B200 copy bandwidth. `value` is that bandwidth in GB/s (whole job:
bytes of all ranks / max-over-ranks time); `ms_per_step` is the step time.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl ours|reference]

One step = one moe_decode_step call (one persistent launch per layer) on a
batch from a pool of 32 seeded inputs. Every step streams more weight bytes than
the 126 MB L2 holds, and one-layer workloads alternate between two independently
seeded weight sets, so no step finds the previous step's weights in L2; the
same steps with a 256 MB L2-flush write between them are reported beside it
(l2_flushed). Under torchrun every rank runs an independent replica (the path
does not shard; no data-path collective): weak scaling.
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "MoE decode-layer µs/step and HBM GB/s (% of B200 peak) at batch 1–64"
FALLBACK_HBM_GBS = 6650.0
POOL = 32
FLUSH_BYTES = 256 << 20
PER_CONFIG = (1, 2, 3, 4)  # the full-size workloads timed after the headline
PER_CONFIG_FP8 = (1, 2)    # and the same layers with FP8 experts (synth.FP8_WORKLOADS)


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--config", type=int, default=1, help="workload index (synth.WORKLOADS)")
    ap.add_argument("--fp8", action="store_true",
                    help="the workload with FP8 expert weights (synth.FP8_WORKLOADS[config])")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU-baseline oracle budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="time only the headline workload (no per_config block)")
    ap.add_argument("--launch-log", default=None,
                    help="write every launch's workload, step, layer, unique experts and algorithmic "
                         "bytes (warm-up included) to this JSON file, to match ncu counters per launch")
    ap.add_argument("--ingest-traffic", nargs=4, metavar=("NCU_CSV", "LAUNCH_LOG", "WORKLOAD", "COMMAND"),
                    help="update profiles/traffic.json from an ncu DRAM-bytes capture and the --launch-log "
                         "of the same command (no GPU work)")
    ap.add_argument("--tc-min-batch", type=int, default=None,
                    help="batch-shape switch: steps of at least this many rows take the tensor-core "
                         "kernel (0: always the CUDA-core kernel); default: the library's")
    ap.add_argument("--profile-small", action="store_true",
                    help="the batch-1 layer with 64 experts instead of 896 (same per-expert shapes, "
                         "~2.9 GB of weights): the small case for full ncu captures of the CUDA-core kernel")
    ap.add_argument("--profile-small-tc", action="store_true",
                    help="batch 1, 128 experts of intermediate 512 (~2.9 GB of weights): the small case "
                         "for full ncu captures of the tensor-core kernel")
    ap.add_argument("--profile-small-b64", action="store_true",
                    help="batch 64 with the Zipf router, 128 experts of intermediate 512 (~2.9 GB of "
                         "weights): the small hot-expert case for full ncu captures of the tensor-core kernel")
    ap.add_argument("--profile-small-fp8", action="store_true",
                    help="batch 1, 128 FP8 experts of intermediate 512 (~1.5 GB of weights): the small case "
                         "for full ncu captures of the FP8 tensor-core kernel")
    return ap.parse_args(argv)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def step_bytes(wl, n_unique_per_layer, batch=None):
    """Algorithmic bytes of one step: every weight byte the step must read once
    (router, shared expert, each unique selected expert as stored: bf16, or E4M3 codes
    and their block scales) plus x, y and gamma."""
    B = wl.B if batch is None else batch
    H, E, Is = wl.H, wl.E, wl.Is
    per_layer_fixed = 2 * (E * H + 3 * Is * H + H) + (4 * E if wl.router == "zipf" else 0)
    total = 0
    for U in n_unique_per_layer:
        total += per_layer_fixed + int(U) * wl.expert_bytes() + 2 * B * H * 2
    return total


def kernel_source_hash():
    """sha256 over the kernel's sources: counters taken on other sources do not apply."""
    import hashlib

    hsh = hashlib.sha256()
    csrc = os.path.join(ROOT, "moe_decode_persistent_b200", "csrc")
    for name in ("moe_decode_kernel.cu", "kernel_params.h", "ptx.cuh"):
        with open(os.path.join(csrc, name), "rb") as f:
            hsh.update(f.read())
    return hsh.hexdigest()


def traffic_entry(workload):
    """The ncu DRAM-traffic record of a workload from profiles/traffic.json, or None when
    the workload was not captured or the kernel sources changed since the capture."""
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(tpath):
        return None
    with open(tpath) as f:
        t = json.load(f).get(workload)
    if t is None or t.get("kernel_sources_sha256") != kernel_source_hash():
        return None
    return t


def traffic_per_launch(workload):
    """DRAM bytes per launch (ncu counters), or None (see traffic_entry)."""
    t = traffic_entry(workload)
    return None if t is None else t.get("bytes_per_launch")


def ingest_traffic(csv_path, log_path, workload, command):
    """Update profiles/traffic.json from an ncu CSV (dram__bytes_read.sum and
    dram__bytes_write.sum of the captured moe_decode launches, in launch order) and this
    bench's --launch-log of the same command: each captured launch is matched to the
    step it ran (the -s count of skipped launches is read from `command`), and its DRAM
    bytes are set beside that step's own algorithmic bytes (all layers of the step when
    one launch runs the whole stack)."""
    import csv
    import re

    per_launch = {}
    with open(csv_path) as f:
        rows = [r for r in csv.reader(l for l in f if not l.startswith("=="))]
    head = rows[0]
    ix = {k: head.index(k) for k in ("ID", "Kernel Name", "Metric Name", "Metric Value")}
    for r in rows[1:]:
        if len(r) < len(head) or "moe_decode" not in r[ix["Kernel Name"]]:
            continue
        d = per_launch.setdefault(int(r[ix["ID"]]), {"kernel": r[ix["Kernel Name"]]})
        d[r[ix["Metric Name"]]] = float(r[ix["Metric Value"]].replace(",", ""))
    with open(log_path) as f:
        log = [e for e in json.load(f) if e["workload"] == workload]
    steps = sorted({e["step"] for e in log})
    skip = int(re.search(r"-s\s+(\d+)", command).group(1))
    fused = "fused" in next(iter(per_launch.values()))["kernel"]
    launches = []
    for n, lid in enumerate(sorted(per_launch)):
        d = per_launch[lid]
        traffic = d["dram__bytes_read.sum"] + d["dram__bytes_write.sum"]
        if fused:  # one launch per step
            step = steps[skip + n]
            alg = sum(e["algorithmic_bytes"] for e in log if e["step"] == step)
        else:  # one launch per layer, in step order
            e = sorted(log, key=lambda e: (e["step"], e["layer"]))[skip + n]
            step, alg = e["step"], e["algorithmic_bytes"]
        launches.append({"step": step, "dram_read": d["dram__bytes_read.sum"],
                         "dram_write": d["dram__bytes_write.sum"], "traffic": traffic,
                         "algorithmic_bytes": alg, "ratio": round(traffic / alg, 4)})
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    t = json.load(open(tpath)) if os.path.exists(tpath) else {}
    t[workload] = {"bytes_per_launch": round(sum(l["traffic"] for l in launches) / len(launches)),
                   "traffic_over_algorithmic": round(sum(l["traffic"] for l in launches)
                                                     / sum(l["algorithmic_bytes"] for l in launches), 4),
                   "launches": launches, "kernel": per_launch[sorted(per_launch)[0]]["kernel"],
                   "source": command, "kernel_sources_sha256": kernel_source_hash()}
    with open(tpath, "w") as f:
        json.dump(t, f, indent=1)
    return t[workload]


def workload_config(wl, flush):
    return {"workload": wl.name, "batch": wl.B, "hidden": wl.H, "experts": wl.E, "top_k": wl.k,
            "expert_inter": wl.I, "shared_inter": wl.Is, "layers": wl.layers,
            "router": wl.router, "rows": wl.rows, "expert_weights": wl.experts, "input_pool": POOL,
            "l2": flush, "parallelism": "replicas"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed region runs."""

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
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        # nvidia-smi's own start-up (its first driver queries) stays out of the timed
        # region: wait, at most 5 s, for its first sample
        t0 = time.perf_counter()
        while self.proc is not None and time.perf_counter() - t0 < 5.0:
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.02)
        time.sleep(0.25)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        self.proc.wait(timeout=10)
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------------------------------
# CPU oracle arm (baseline leg and --impl reference)
# ---------------------------------------------------------------------------------------

def cpu_oracle_full_steps(wl, pool, budget_s):
    """Time the oracle on full single-row layer steps of the pool's inputs, budget_s of
    oracle time in total: each input's step (weights regenerated on the host first, not
    timed) is repeated until its share of the budget is used (the oracle keeps no state
    between calls, so a repeat is the same work). Returns (GB/s, seconds, steps, inputs)."""
    import oracle

    shared = [wl.shared_host(l) for l in range(wl.layers)]
    w_router = [wl.w_router_host(l) for l in range(wl.layers)]
    dims = dict(H=wl.H, E=wl.E, k=wl.k, I=wl.I, Is=wl.Is, eps=wl.eps)
    per_input = budget_s / len(pool)
    t_tot, bytes_tot, steps = 0.0, 0, 0
    for v in range(len(pool)):
        x0 = pool[v][:1]
        layer_w = []
        x = x0
        for l in range(wl.layers):
            gamma, bias = wl.gamma_host(l), wl.bias_host(l)
            n = oracle.rmsnorm(x[0], gamma, wl.eps)
            sel = oracle.topk(oracle.router(n, w_router[l], bias), wl.k)
            experts = {int(e): wl.expert_host(l, int(e)) for e in sel}
            layer_w.append(dict(gamma=gamma, w_router=w_router[l], router_bias=bias, experts=experts,
                                ws_gate=shared[l][0], ws_up=shared[l][1], ws_down=shared[l][2]))
            if l + 1 < wl.layers:
                x = oracle.layer(dims, layer_w[-1], x)["y"]
        t_v = 0.0
        while t_v < per_input:
            x = x0
            uniq = []
            for l in range(wl.layers):
                t0 = time.perf_counter()
                r = oracle.layer(dims, layer_w[l], x)
                t_v += time.perf_counter() - t0
                x = r["y"]
                uniq.append(len(layer_w[l]["experts"]))
            bytes_tot += step_bytes(wl, uniq, batch=1)
            steps += 1
        t_tot += t_v
    return bytes_tot / t_tot / 1e9, t_tot, steps, len(pool)


def run_reference(args, wl):
    """--impl reference: the fp64 CPU oracle as it stands, timed on the host cores."""
    import oracle

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    pool = wl.x_pool_host(2)
    gamma, bias = wl.gamma_host(0), wl.bias_host(0)
    w_router = wl.w_router_host(0)
    sg, su, sd = wl.shared_host(0)
    n = oracle.rmsnorm(pool[0][0], gamma, wl.eps)
    sel = oracle.topk(oracle.router(n, w_router, bias), wl.k)
    experts = [wl.expert_host(0, int(e)) for e in sel]
    budget = max(0.02, min(1.0, 150.0 / max(1, args.steps + args.warmup)))

    def one_step(i):
        # a bounded sample of the layer: RMSNorm + router for one row, then SwiGLU
        # experts (shared first, then the row's selected experts, cycling) until the
        # per-step budget is used; bytes = weight bytes processed
        t0 = time.perf_counter()
        b = 0
        x = pool[i % len(pool)][0]
        nn = oracle.rmsnorm(x, gamma, wl.eps)
        oracle.router(nn, w_router, bias)
        b += 2 * (wl.E * wl.H + wl.H) + 2 * wl.H
        j = i
        while time.perf_counter() - t0 < budget:
            if j % (len(experts) + 1) == 0:
                oracle.swiglu(nn, sg, su, sd)
                b += 2 * 3 * wl.Is * wl.H
            else:
                g, u, d = experts[j % (len(experts) + 1) - 1]
                oracle.swiglu(nn, g, u, d)
                b += 2 * 3 * wl.I * wl.H
            j += 1
        return b, time.perf_counter() - t0

    for i in range(args.warmup):
        one_step(i)
    tot_b, tot_t = 0, 0.0
    for i in range(args.steps):
        b, t = one_step(i)
        tot_b += b
        tot_t += t
    value = tot_b / tot_t / 1e9
    cores = len(os.sched_getaffinity(0))
    sample = (f"per step: RMSNorm + router of one row of {wl.name}, then SwiGLU experts (shared, "
              f"then the row's {wl.k} selected, cycling) for ~{budget:.3f} s; weights pre-generated "
              f"on the host")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * tot_t / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(wl, "n/a (host)"),
            "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------------------

def aggregate(local_bytes, local_ms, world):
    """Whole-job totals: bytes summed over ranks, time = max over ranks."""
    if world == 1:
        return float(local_bytes), float(local_ms)
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    b = torch.tensor([float(local_bytes)], dtype=torch.float64, device=dev)
    t = torch.tensor([float(local_ms)], dtype=torch.float64, device=dev)
    dist.all_reduce(b, op=dist.ReduceOp.SUM)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(b.item()), float(t.item())


TIMING = ("value: one CUDA-event pair around the K back-to-back timed steps; us_per_step_p10/median/"
          "p90/max: a second pass of K steps with an event pair around every step (an event between two "
          "launches delays the second, so these run a few us above the back-to-back mean)")


def step_stats(step_ms, total_ms=None):
    """us_per_step: the back-to-back mean (total_ms / K) when given, else the per-step mean;
    the quantiles and the slowest step: the per-step times."""
    a = np.asarray(step_ms, dtype=np.float64) * 1e3  # µs
    mean = total_ms * 1e3 / len(a) if total_ms is not None else float(a.mean())
    return {"us_per_step": round(mean, 2), "us_per_step_p10": round(float(np.percentile(a, 10)), 2),
            "us_per_step_median": round(float(np.median(a)), 2),
            "us_per_step_p90": round(float(np.percentile(a, 90)), 2),
            "us_per_step_max": round(float(a.max()), 2), "slowest_step": int(a.argmax())}


L2_PROTOCOL = ("no flush: every step streams more weight bytes than the 126 MB L2, and single-layer "
               "workloads alternate between two independently seeded weight sets (two layers), so no "
               "step finds the previous step's weights in L2 (a decode step runs its layers in turn)")


class ConfigRun:
    """One workload on this rank's GPU: its weights (generated on the device; a one-layer
    workload gets two independently seeded weight sets, used alternately, like two layers
    of a model), a handle per set, a pool of POOL seeded input batches resident in HBM,
    and an L2-flush buffer for the secondary, flushed timing."""

    def __init__(self, wl, device, tc_min_batch=None):
        import dataclasses

        import torch

        import moe_decode_persistent_b200 as mdp

        self.wl = wl
        self.dev = f"cuda:{device}"
        # (the small profiling layers keep one set: a full ncu capture holds ~3 GB)
        one = wl.layers > 1 or wl.name.endswith("_profile")
        variants = [wl] if one else [wl, dataclasses.replace(wl, seed=wl.seed + 100)]
        self.sets = []
        for v in variants:
            layers = [v.device_layer_any(l, device=self.dev) for l in range(wl.layers)]
            h = mdp.MoeDecode(wl.H, wl.E, wl.k, wl.I, wl.Is, wl.B, layers, eps=wl.eps, device=device,
                              fp8=wl.is_fp8)
            if tc_min_batch is not None:
                h.set_tc_min_batch(tc_min_batch)
            self.sets.append((layers, h))
        self.h = self.sets[0][1]
        self.kernel_path = "tensor_core" if self.h.step_path(wl.B) == mdp.PATH_TENSOR_CORE else "cuda_core"
        self.pool_host = wl.x_pool_host(POOL)
        self.pool = torch.from_numpy(self.pool_host.view(np.int16)).view(torch.bfloat16).to(self.dev)
        self.y = torch.empty((wl.B, wl.H), dtype=torch.bfloat16, device=self.dev)
        self.flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=self.dev)

    def steps(self, K, W, stream, barrier, host=None, launch_log=None, flush=False, per_step=False):
        """W untimed warm-up steps immediately followed (no idle gap, so the clocks stay
        up) by K timed steps; step i runs weight set i mod (number of sets). One CUDA-event
        pair on `stream` brackets the K back-to-back steps (launches follow one another as
        in a decode loop); per_step: a pair around every step instead (an event recorded
        between two launches delays the second by a few µs, so these per-step times run a
        little above the back-to-back mean). flush: a 256 MB write before every step (the
        secondary, flushed figure; per-step events, so the writes stay out of the timing).
        host = (x_host, y_host): the host-buffer entry point instead. Returns the per-step
        ms (per_step) or the K steps' total ms as one value, and the unique-expert count of
        every timed step and layer."""
        assert per_step or not flush
        import torch

        wl = self.wl
        nu = torch.zeros((W + K, wl.layers), dtype=torch.int32, device=self.dev)
        dbg = lambda i: [dict(n_unique=nu[i, l:l + 1]) for l in range(wl.layers)]
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(K if per_step else 1)]

        # every step's handle, input view and debug record, made before any step runs (the
        # harness's own bookkeeping stays out of the timed steps' host time)
        src = self.pool if host is None else host[0]
        plan = [(self.sets[i % len(self.sets)][1], src[i % POOL], dbg(i)) for i in range(W + K)]

        def one(i, timed):
            h, x, d = plan[i]
            if flush:
                self.flush.zero_()
            if timed and per_step:
                ev[i - W][0].record(stream)
            if host is None:
                h.step(x, self.y, wl.B, wl.k, stream=stream, debug=d)
            else:
                h.step_host(x, host[1], wl.B, wl.k, stream=stream, debug=d)
            if timed and per_step:
                ev[i - W][1].record(stream)

        for i in range(W):
            one(i, False)
        # the timed region: barrier + synchronize on both sides; the warm-up runs right
        # before it, so the GPU does not idle (and drop its clocks) in between
        barrier()
        torch.cuda.synchronize()
        wall0 = time.perf_counter()
        if not per_step:
            ev[0][0].record(stream)
        for i in range(W, W + K):
            one(i, True)
        if not per_step:
            ev[0][1].record(stream)
        torch.cuda.synchronize()
        barrier()
        self.wall = time.perf_counter() - wall0
        for _, h in self.sets:
            status = h.status()
            if status != 0:
                import moe_decode_persistent_b200 as mdp

                raise RuntimeError(f"{wl.name}: device status {status}: {mdp.strerror(status)}")
        U = nu.cpu().numpy()
        if launch_log is not None:
            for i in range(W + K):
                for l in range(wl.layers):
                    launch_log.append({"workload": wl.name, "step": i, "layer": l, "timed": i >= W,
                                       "unique_experts": int(U[i, l]),
                                       "algorithmic_bytes": step_bytes(wl, [int(U[i, l])])})
        return [a.elapsed_time(b) for a, b in ev], U[W:]

    def close(self):
        import torch

        for _, h in self.sets:
            h.close()
        del self.sets, self.h, self.pool, self.flush, self.y
        torch.cuda.synchronize()
        torch.cuda.empty_cache()


def roofline_entry(wl, achieved, peak, peak_kind):
    t = traffic_entry(wl.name)
    return {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "traffic": None if t is None else t["bytes_per_launch"],
            "traffic_over_algorithmic": None if t is None else t.get("traffic_over_algorithmic"),
            "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                           else "fallback 6.65 TB/s",
            "kernel": "moe_decode_layer_kernel"}


def run_ours(args, wl):
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    def barrier():
        if world > 1:
            import torch.distributed as dist

            dist.barrier()

    stream = torch.cuda.current_stream()
    K, W = args.steps, args.warmup
    peak, peak_kind = measured_peaks()
    launch_log = [] if args.launch_log else None
    run = ConfigRun(wl, local, args.tc_min_batch)
    sampler = ClockSampler(local)
    sampler.start()
    tot_ms, U = run.steps(K, W, stream, barrier, launch_log=launch_log)
    wall = run.wall
    step_ms, _ = run.steps(K, W, stream, barrier, per_step=True)
    clocks = sampler.stop()
    bytes_steps = [step_bytes(wl, list(U[i])) for i in range(K)]
    local_ms = float(sum(tot_ms))
    tot_bytes, max_ms = aggregate(sum(bytes_steps), local_ms, world)
    value = tot_bytes / (max_ms * 1e-3) / 1e9
    achieved = sum(bytes_steps) / (local_ms * 1e-3) / 1e9  # this rank's launching stream
    # secondary figure: the same steps with a 256 MB write between steps (which also
    # evicts the kernel's instructions and leaves L2 full of dirty lines to write back)
    f_ms, fU = run.steps(K, W, stream, barrier, flush=True, per_step=True)
    f_bytes, f_max = aggregate(sum(step_bytes(wl, list(fU[i])) for i in range(K)), float(sum(f_ms)), world)
    l2_flushed = {"value": round(f_bytes / (f_max * 1e-3) / 1e9, 2), "unit": "GB/s", **step_stats(f_ms),
                  "l2": "flushed between timed steps (256 MB write)"}

    # end to end through the host-buffer entry point: H2D x, step, D2H y per step
    e2e = None
    if not args.no_e2e:
        xh = torch.from_numpy(run.pool_host.view(np.int16)).pin_memory()
        yh = torch.empty((wl.B, wl.H), dtype=torch.int16).pin_memory()
        e_step, U2 = run.steps(K, min(W, 10), stream, barrier, host=(xh, yh))
        e_ms = float(sum(e_step))
        e_bytes, e_max = aggregate(sum(step_bytes(wl, list(U2[i])) for i in range(K)), e_ms, world)
        e2e = {"value": round(e_bytes / (e_max * 1e-3) / 1e9, 2), "unit": "GB/s",
               "h2d_bytes_per_step": int(xh[0].numel() * 2), "d2h_bytes_per_step": int(yh.numel() * 2),
               "ms_per_step": round(e_max / K, 4)}

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": round(max_ms / K, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded counter-hash weights ~N(0,1/sqrt(fan_in)) and inputs, no trained weights",
        "config": dict(workload_config(wl, L2_PROTOCOL), kernel_path=run.kernel_path),
        **step_stats(step_ms, local_ms),
        "timing": TIMING,
        "l2_flushed": l2_flushed,
        "tokens_per_s": round(world * wl.B * K / (max_ms * 1e-3), 1),
        "unique_experts_mean": float(U.mean()),
        "bytes_per_step_mean": float(np.mean(bytes_steps)),
        "hbm_frac_of_peak": round(value / world / peak, 4),
        "roofline": roofline_entry(wl, achieved, peak, peak_kind),
        "e2e": e2e,
        "gpu_launches": K * run.h.launches_per_step(),
        "clocks": clocks,
        "wall_s_timed_region": round(wall, 4),
    }
    pool_host = run.pool_host
    run.close()

    # the other full-size workloads, each on its own weights: µs/step and GB/s over its
    # own unique-expert bytes, with its own clock record
    per_config = {}
    launches = line["gpu_launches"]
    others = [synth.WORKLOADS[c] for c in PER_CONFIG] + [synth.FP8_WORKLOADS[c] for c in PER_CONFIG_FP8]
    for cw in ([] if args.no_per_config else [o for o in others if o.name != wl.name]):
        r = ConfigRun(cw, local, args.tc_min_batch)
        smp = ClockSampler(local)
        smp.start()
        c_tot, cU = r.steps(K, W, stream, barrier, launch_log=launch_log)
        c_ms, _ = r.steps(K, W, stream, barrier, per_step=True)
        c_clocks = smp.stop()
        c_bytes = [step_bytes(cw, list(cU[i])) for i in range(K)]
        c_local = float(sum(c_tot))
        c_tot, c_max = aggregate(sum(c_bytes), c_local, world)
        c_ach = sum(c_bytes) / (c_local * 1e-3) / 1e9
        per_config[cw.name] = {
            "config": workload_config(cw, L2_PROTOCOL) | {"kernel_path": r.kernel_path},
            "dtype": "fp8 (e4m3) experts, bf16 activations" if cw.is_fp8 else "bf16",
            "value": round(c_tot / (c_max * 1e-3) / 1e9, 2), "unit": "GB/s",
            **step_stats(c_ms, c_local),
            "tokens_per_s": round(world * cw.B * K / (c_max * 1e-3), 1),
            "unique_experts_mean": float(cU.mean()), "bytes_per_step_mean": float(np.mean(c_bytes)),
            "roofline": roofline_entry(cw, c_ach, peak, peak_kind),
            "gpu_launches": K * r.h.launches_per_step(), "clocks": c_clocks}
        launches += K * r.h.launches_per_step()
        r.close()
    if per_config:
        line["per_config"] = per_config
        line["gpu_launches_all_configs"] = launches
    if args.launch_log and rank == 0:
        with open(args.launch_log, "w") as f:
            json.dump(launch_log, f)

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gbs, secs, steps, ninp = cpu_oracle_full_steps(wl, pool_host[:, :1], args.cpu_seconds)
        line["cpu_baseline"] = {
            "value": round(gbs, 4), "unit": "GB/s", "cores": len(os.sched_getaffinity(0)),
            "kind": "oracle",
            "sample": f"{steps} full single-row layer steps of {wl.name} over {ninp} distinct pool inputs "
                      f"({secs:.1f} s of oracle time; host weight regeneration not timed)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def main(argv=None):
    args = parse_args(argv)
    if args.ingest_traffic:
        print(json.dumps(ingest_traffic(*args.ingest_traffic), indent=1))
        return
    wl = synth.FP8_WORKLOADS[args.config] if args.fp8 else synth.WORKLOADS[args.config]
    if args.profile_small:
        wl = synth.Workload("b1_h7168_e64_k16_profile", B=1, H=7168, E=64, k=16, I=1024, Is=2048, seed=1)
    if args.profile_small_tc:
        wl = synth.Workload("b1_h7168_e128_i512_k16_profile", B=1, H=7168, E=128, k=16, I=512, Is=1024, seed=1)
    if args.profile_small_b64:
        wl = synth.Workload("b64_h7168_e128_i512_k16_zipf_profile", B=64, H=7168, E=128, k=16, I=512, Is=1024,
                            seed=3, router="zipf")
    if args.profile_small_fp8:
        wl = synth.Workload("b1_h7168_e128_i512_k16_fp8_profile", B=1, H=7168, E=128, k=16, I=512, Is=1024,
                            seed=1, experts="fp8")
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_ours(args, wl)


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""Benchmark of the MoE decode-layer step on B200: one JSON line on rank 0.

Metric: microseconds per decode layer-step (device time; no step finds its weights in
L2: a one-layer step cycles over 4 independently seeded weight copies, a stack streams
more than twice the L2 per step) and the weight bytes the step touched per second as a
fraction of the measured HBM peak.  Secondary figures: the same weights back to back
(warm) and a 256 MiB L2 flush before each step.  A "step" is one call of moe_decode_step: every kernel of the
layer (or of the 8-layer stack) on one batch of seeded synthetic inputs.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--prefetch 0|1]
  python bench.py --impl reference ...   (the CPU oracle, timed on the host cores)

Workloads (seeded synthetic inputs shaped like one GPU's tensor-parallel shard):
  tp16_b1        d=7168, d_o=8192, E=896, k=16, I=128, batch 1     (default)
  tp16_b2_ov0    same shapes, batch 2, two independent tokens (overlap ~0)
  tp16_b2_ov16   same shapes, batch 2, one token twice (overlap 16)
  tp8_b16/b64    d=7168, d_o=8192, E=896, k=16, I=256, batch 16 / 64
  stack8_b1/b64  8 layers of the tp16 shape in one step, batch 1 / 64

Multi-GPU: the step does not shard (one GPU per layer-step), so N ranks run N
independent replicas; the value is the whole job's time per layer-step
(max-over-ranks time / (N * steps * layers)), scaling "weak".
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "µs per decode layer-step and weight GB/s (% of HBM peak) at batch 1/2/16/64"
UNIT = "us/layer-step"

WORKLOADS = {
    "tp16_b1": ("TP16", 1, 1, "indep"),
    "tp16_b2_ov0": ("TP16", 2, 1, "indep"),
    "tp16_b2_ov16": ("TP16", 2, 1, "dup"),
    "tp8_b16": ("TP8", 16, 1, "indep"),
    "tp8_b64": ("TP8", 64, 1, "indep"),
    "stack8_b1": ("TP16", 1, 8, "indep"),
    "stack8_b64": ("TP16", 64, 8, "indep"),
    # profiling case: tp16 o_proj/router/expert shapes with 64 experts (~0.6 GB on the device)
    "tp16e64_b1": ("TP16E64", 1, 1, "indep"),
    "tp16e64_b2": ("TP16E64", 2, 1, "indep"),
    "tp8e64_b64": ("TP8E64", 64, 1, "indep"),
    "tp8e224k4_b16": ("TP8E224K4", 16, 1, "indep"),
    # profiling case for the next-layer prefetch: two such layers (~1.2 GB on the device)
    "stack2e64_b1": ("TP16E64", 1, 2, "indep"),
}

KERNEL_DIR = os.path.join(ROOT, "moe_decode_layer_02_b200", "csrc")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return float(j["hbm_gbs"]), float(j.get("bf16_tflops", 1590.0)), "measured"
    return 6650.0, 1590.0, "fallback"


def dims_of(name):
    import synth
    small = {"TP16E64": synth.Dims(7168, 8192, 64, 16, 128), "TP8E64": synth.Dims(7168, 8192, 64, 16, 256),
             # batch 16 with the TP8 shard's tokens-per-expert (16 * 4 / 224 = 16 * 16 / 896) in 2.5 GB
             "TP8E224K4": synth.Dims(7168, 8192, 224, 4, 256)}
    return small[name] if name in small else getattr(synth, name)


def seed_of(dname, L):
    import synth
    return synth.config_seed({"TP16": 1, "TP8": 3, "TP16E64": 21, "TP8E64": 23, "TP8E224K4": 25}[dname] + (10 if L > 1 else 0))


def rotation(L):
    """Weight copies a single-layer step cycles over (4 x >= 218 MB > 2 x the 126 MB L2)."""
    return 4 if L == 1 else 1


def token_inputs(seed, dims, B, L, mode):
    import numpy as np
    import synth
    attn = np.stack([np.stack([synth.host_token(seed, synth.ATTN, dims.d_o, layer=l, token=(0 if mode == "dup" else b))
                               for b in range(B)]) for l in range(L)])
    resid = np.stack([synth.host_token(seed, synth.RESID, dims.d, token=(0 if mode == "dup" else b)) for b in range(B)])
    return attn, resid


# --------------------------------------------------------------------------------------------
class Clocks:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx, self.proc, self.lines = gpu_index, None, []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------------------------
def algorithmic_bytes(dims, B, n_union):
    """Bytes each kernel must move at least once (weights dominate; activations included)."""
    d, do, E, k, I = dims.d, dims.d_o, dims.E, dims.k, dims.I
    return {
        "oproj_residual_rmsnorm": d * do * 2 + B * do * 2 + B * d * 2 + B * d * 4,
        "router_topk": E * d * 2 + d * 2 + B * d * 4 + B * d * 4 + B * E * 4,
        "gateup_rows": n_union * 2 * I * d * 2 + B * k * d * 4 + B * k * I * 4,
        "down_rows": n_union * d * I * 2 + B * k * I * 4 + B * d * 4 + B * d * 2,
        # small-M expert kernel: gate/up and down weights of the union, x and h in, out
        "experts_small_m": n_union * 3 * I * d * 2 + B * E * 4 + 2 * B * d * 4 + B * d * 2,
        # fused batch <= 2 layer kernel: every weight of the layer once, attn_out and the
        # residual in, the output out (its h, x and logits stay in L2)
        "layer_fused_small_m": d * do * 2 + E * d * 2 + d * 2 + n_union * 3 * I * d * 2 + B * (do * 2 + d * 4),
    }


def weight_bytes(dims, n_union_per_layer):
    d, do, E, I = dims.d, dims.d_o, dims.E, dims.I
    return sum(d * do * 2 + d * 2 + E * d * 2 + u * (2 * I * d * 2 + d * I * 2) for u in n_union_per_layer)


def code_only(text):
    """C++ source without comments or blank lines (string literals left as they are)."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    out = []
    for line in text.splitlines():
        i = line.find("//")
        if i >= 0 and line.count('"', 0, i) % 2 == 0:
            line = line[:i]
        line = line.rstrip()
        if line:
            out.append(line)
    return "\n".join(out)


def max_over_ranks(x, world, device):
    """The largest per-rank value over all ranks (a multi-GPU job's time is its slowest rank's)."""
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_us_per_layer_step(t_max_ms, world, steps, layers):
    """Whole-job figure: N replicas each run `steps` steps of `layers` layers in t_max_ms."""
    return t_max_ms * 1000.0 / (world * steps * layers)


def kernels_sha(kernel_dir=None):
    """Hash of the kernel code (comments ignored): ncu traffic figures are valid only for the
    code they were taken on."""
    import hashlib
    kdir = kernel_dir or KERNEL_DIR
    hs = hashlib.sha256()
    for f in sorted(os.listdir(kdir)):
        if f.endswith((".cu", ".cuh")):
            hs.update(f.encode())
            hs.update(code_only(open(os.path.join(kdir, f), encoding="utf-8").read()).encode())
    return hs.hexdigest()[:16]


def traffic_for(kernel_name, B, workload):
    """Per-launch DRAM bytes from the committed ncu summary, if taken on the current kernels."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    j = json.load(open(p))
    h = kernels_sha()
    ent = j.get(workload, {}).get(kernel_name)
    if not ent or ent.get("kernels_sha") != h:
        return None
    return ent.get("bytes_per_launch")


def run_ours(args, rank, world):
    import numpy as np
    import torch
    import torch.distributed as dist

    import moe_decode_layer_02_b200 as md
    import synth
    from moe_decode_layer_02_b200 import build as mdb

    dev = int(os.environ.get("LOCAL_RANK", 0))
    torch.cuda.set_device(dev)
    mdb.build()
    synth.build_device_fill()
    md.load()
    dname, B, L, mode = WORKLOADS[args.workload]
    dims = dims_of(dname)
    seed = seed_of(dname, L)
    sz = dims.sizes()
    R = rotation(L)
    weight_sets = []
    for r in range(R):  # independently seeded copies; a timed step uses copy i % R
        weights = []
        for l in range(L):
            t = {}
            for kind in (synth.W_O, synth.GAMMA, synth.W_R, synth.W_GU, synth.W_DOWN):
                x = torch.empty(sz[kind], dtype=torch.bfloat16, device="cuda")
                synth.device_fill(x, seed + 1000 * r, kind, layer=l)
                t[kind] = x
            weights.append((t[synth.W_O], t[synth.GAMMA], t[synth.W_R], t[synth.W_GU], t[synth.W_DOWN]))
        weight_sets.append(weights)
    attn_np, resid_np = token_inputs(seed, dims, B, L, mode)
    attn = torch.from_numpy(attn_np.view(np.int16)).cuda().view(torch.bfloat16)
    resid = torch.from_numpy(resid_np.view(np.int16)).cuda().view(torch.bfloat16)
    out = torch.empty((B, dims.d), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((L, B, dims.k), dtype=torch.int32, device="cuda")
    gate = torch.empty((L, B, dims.k), dtype=torch.float32, device="cuda")
    cfg = md.config(dims.d, dims.d_o, dims.E, dims.k, dims.I, max(B, 1), L, enable_prefetch=args.prefetch,
                    force_variant=args.force_variant)
    s = torch.cuda.current_stream()
    hs = [md.moe_decode_create(cfg, w, s) for w in weight_sets]
    h = hs[0]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")  # 256 MiB > 126 MB L2
    kps = md.moe_decode_kernels_per_step(h, B)

    def step(i=0):
        md.moe_decode_step(hs[i % R], B, attn, resid, out, idx, gate, s)

    for i in range(max(args.warmup, 3) * R):
        step(i)
    if args.profile_run:
        # Profiling mode (for ncu): a few plain graph replays, no timing.
        for i in range(args.profile_run):
            step(i)
        rc = max(abs(md.moe_decode_sync_status(x, s)) for x in hs)
        for x in hs:
            md.moe_decode_destroy(x)
        if rc:
            raise RuntimeError(md.strerror(-rc))
        return None
    n_union = []
    for r in range(R):
        step(r)
        rc = md.moe_decode_sync_status(hs[r], s)
        if rc:
            raise RuntimeError(md.strerror(rc))
        idx_np = idx.cpu().numpy()
        n_union += [len(np.unique(idx_np[l])) for l in range(L)]

    # ---- timed region: K steps; no step reuses weights that can still be in L2 -----------------
    # (one layer: the step cycles over R weight copies, R x bytes per step > 2 x L2; a stack of
    # layers streams more than 2 x L2 per step by itself)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with Clocks(dev) as clk:
        time.sleep(0.3)
        for i in range(args.steps):
            ev[i][0].record(s)
            step(i)
            ev[i][1].record(s)
        torch.cuda.synchronize()
        time.sleep(0.2)
    if world > 1:
        dist.barrier()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    rc = max(abs(md.moe_decode_sync_status(x, s)) for x in hs)
    if rc:
        raise RuntimeError(md.strerror(-rc))
    t_max_ms = max_over_ranks(sum(step_ms), world, "cuda")

    # ---- secondary: the same weights back to back (warm L2), and a 256 MiB L2 flush before each
    # step instead of the rotation (the flush leaves dirty lines whose write-back lands inside
    # the next step, so it overstates a cold step)
    w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w0.record(s)
    for _ in range(args.steps):
        step()
    w1.record(s)
    torch.cuda.synchronize()
    warm_us = w0.elapsed_time(w1) * 1000 / (args.steps * L)
    fl = []
    for i in range(min(args.steps, 20)):
        flush.fill_(i & 0xFF)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(s)
        step()
        f1.record(s)
        torch.cuda.synchronize()
        fl.append(f0.elapsed_time(f1))
    flushed_us = statistics.median(fl) * 1000 / L

    # ---- end to end through the host-buffer entry point (pinned host memory) -----------------
    a_h = torch.from_numpy(attn_np.view(np.int16)).pin_memory()
    r_h = torch.from_numpy(resid_np.view(np.int16)).pin_memory()
    o_h = torch.empty((B, dims.d), dtype=torch.int16).pin_memory()
    i_h = torch.empty((L, B, dims.k), dtype=torch.int32).pin_memory()
    g_h = torch.empty((L, B, dims.k), dtype=torch.float32).pin_memory()
    for x in hs:
        md.moe_decode_step_host(x, B, a_h, r_h, o_h, i_h, g_h, s)
    e_ms = []
    for i in range(args.steps):
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        md.moe_decode_step_host(hs[i % R], B, a_h, r_h, o_h, i_h, g_h, s)
        e1.record(s)
        e1.synchronize()
        e_ms.append(e0.elapsed_time(e1))
    h2d = attn_np.nbytes + resid_np.nbytes
    d2h = B * dims.d * 2 + 2 * L * B * dims.k * 4

    # ---- per-kernel durations (eager, event-bracketed launches, weights rotated as above) ------
    per = {}
    for i in range(max(5, min(args.steps, 20)) * R):
        torch.cuda.synchronize()
        for name, ms in md.moe_decode_profile_step(hs[i % R], B, attn, resid, out, idx, gate, s):
            per.setdefault(name, []).append(ms)
    for x in hs:
        md.moe_decode_destroy(x)
    return {"B": B, "L": L, "R": R, "dims": dims, "step_ms": step_ms, "t_max_ms": t_max_ms, "warm_us": warm_us,
            "flushed_us": flushed_us,
            "e2e_ms": e_ms, "h2d": h2d, "d2h": d2h, "per_kernel": per, "n_union": n_union,
            "clocks": clk.summary(), "kps": kps}


def cpu_baseline(args, budget_s=12.0):
    """The oracle as it stands, on a bounded sample of the workload (host cores)."""
    import numpy as np
    import oracle
    import synth
    from oracle.layer import LayerRef
    oracle.build()
    o = oracle.get()
    dname, B, L, mode = WORKLOADS[args.workload]
    dims = dims_of(dname)
    seed = seed_of(dname, L)
    ref = LayerRef(seed, dims, 0, oracle=o)
    attn_np, resid_np = token_inputs(seed, dims, B, 1, mode)
    # Warm the expert cache (host generation of weights is setup, not oracle work).
    f = ref.front(attn_np[0][:1], resid_np[:1])
    for e in f["idx"][0]:
        ref.expert(e)
    times, n = [], 0
    t_start = time.perf_counter()
    while time.perf_counter() - t_start < budget_s or n < 2:
        b = n % B
        t0 = time.perf_counter()
        f = ref.front(attn_np[0][b:b + 1], resid_np[b:b + 1])
        ref.moe(f, 0)
        times.append(time.perf_counter() - t0)
        n += 1
        if n >= 200:
            break
    per_token_s = statistics.median(times)
    us_per_layer_step = per_token_s * B * 1e6  # one layer-step = B tokens
    return {"value": us_per_layer_step, "unit": UNIT, "cores": o.threads(), "kind": "oracle",
            "sample": f"{n} single-token oracle layer passes of {args.workload} (median {per_token_s*1e3:.1f} ms "
                      f"per token, scaled x{B} tokens per layer-step; expert weights regenerated outside the timing)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="tp16_b1", choices=sorted(WORKLOADS))
    ap.add_argument("--prefetch", type=int, default=1)
    ap.add_argument("--force-variant", type=int, default=0, choices=[0, 1, 2],
                    help="kernel choice: 0 by batch size, 1 unfused batch <= 2 kernels, 2 large-batch "
                         "kernels at every batch (comparison runs)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-run", type=int, default=0,
                    help="profiling mode: warm up, replay the step N times, print nothing")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    dname, B, L, mode = WORKLOADS[args.workload]
    config = {"workload": args.workload, "batch": B, "layers": L, "shape": dname,
              "prefetch": bool(args.prefetch and L > 1),
              "force_variant": args.force_variant,
              "l2": (f"inputs larger than L2: the step cycles over {rotation(L)} independently seeded weight "
                     "copies, no flush" if rotation(L) > 1 else
                     f"inputs larger than L2: {L} layers of distinct weights per step, no flush"),
              "parallelism": f"replicas x{args.gpus}"}

    if args.impl == "reference":
        if rank != 0:
            return
        cb = cpu_baseline(args, budget_s=max(3.0, min(60.0, 2.0 * args.steps)))
        line = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": UNIT, "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": cb["value"] * L / 1000.0,
                "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": config, "cpu_baseline": cb,
                "e2e": {"value": cb["value"], "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    r = run_ours(args, rank, world)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0 or r is None:
        return
    hbm, bf16, src = peaks()
    dims = r["dims"]
    K = args.steps
    us_per_layer = job_us_per_layer_step(r["t_max_ms"], world, K, L)
    wbytes = weight_bytes(dims, r["n_union"]) / r["R"]  # n_union holds R copies x L layers
    per_step_ms = r["t_max_ms"] / K
    gbs = wbytes / (per_step_ms * 1e-3) / 1e9
    # dominant kernel by time share
    avg = {n: statistics.mean(v) for n, v in r["per_kernel"].items()}
    tot = sum(avg.values())
    dom = max(avg, key=avg.get)
    ab = algorithmic_bytes(dims, B, statistics.mean(r["n_union"]))
    key = dom
    dom_bytes = ab.get(key, 0)
    ach = dom_bytes / (avg[dom] * 1e-3) / 1e9
    e2e_us = statistics.mean(r["e2e_ms"]) * 1000 / L
    cb = None
    if world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(args)
    line = {
        "metric": METRIC, "value": round(us_per_layer, 3), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(per_step_ms, 5), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16 weights, fp32 accumulate", "data": "synthetic",
        "config": config,
        "weight_gbs": round(gbs, 1), "hbm_frac": round(gbs / hbm, 4), "hbm_peak_gbs": hbm, "peak_source": src,
        "weight_bytes_per_step": wbytes, "experts_touched": r["n_union"],
        "us_per_layer_step_p10_p50_p90": [round(x * 1000 / L, 2) for x in
                                          (sorted(r["step_ms"])[int(0.1 * (K - 1))],
                                           statistics.median(r["step_ms"]),
                                           sorted(r["step_ms"])[int(0.9 * (K - 1))])],
        "warm_us_per_layer_step": round(r["warm_us"], 3),
        "l2_flushed_us_per_layer_step": round(r["flushed_us"], 3),
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": round(ach, 1), "peak": hbm, "unit": "GB/s",
                     "frac": round(ach / hbm, 4), "traffic": traffic_for(dom, B, args.workload),
                     "algorithmic_bytes": dom_bytes, "avg_launch_us": round(avg[dom] * 1000, 3),
                     "share": round(avg[dom] / tot, 3), "peak_kind": f"{src} burst copy"},
        "kernels_us": {n: round(v * 1000, 2) for n, v in avg.items()},
        "e2e": {"value": round(e2e_us, 3), "unit": UNIT, "h2d_bytes_per_step": r["h2d"],
                "d2h_bytes_per_step": r["d2h"]},
        "gpu_launches": r["kps"] * K,
        "clocks": r["clocks"],
        "cpu_baseline": cb,
    }
    print(json.dumps(line))


if __name__ == "__main__":
    main()

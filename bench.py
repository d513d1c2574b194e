"""Benchmark of the ISA forward pass on B200: one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

A step is one ISA forward call over the headline workload (B=1, H=40, D=128,
L_src = L_ctx = 16384, b = 128, alpha_s = 0.25, alpha_f = 0.6: the 32K-token
case), inputs resident in HBM. `value` is the effective throughput in TFLOP/s
(FLOPs the pass executes: coarse scores, routing, exact and Taylor attention)
over all ranks; `ms_per_step` is the max over ranks.

Under torchrun the (batch, head) slices are the units that ranks share:
* `--scaling weak` (default): rank r computes batch element r of a global
  batch of N elements (its own draw of the workload's shape), so per-GPU work
  is fixed; no collective on the data path (NCCL only for the barrier and the
  max of the timings);
* `--scaling strong`: the workload's B*H slices are split into contiguous
  ranges over the ranks; with `--gather` the timed step also all-gathers O
  over NCCL so that every rank holds the whole output.

`--impl reference` times the CPU oracle (float64 numpy) as it stands on the
host cores over a bounded sample of the same workload (one head per step).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import isa_synth  # noqa: E402

METRIC = "ISA forward ms/call and effective TFLOPS at 32K tokens; fraction of roofline"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Datasheet figures, reported beside the measured ones: dense bf16 tensor peak and the ~8 TB/s HBM3e
NOMINAL = {"bf16_tflops": 2250.0, "hbm_gbs": 8000.0}
BAD_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


# ----------------------------------------------------------------------------- host-side logic (tested on CPU)

def no_sparse_count(alpha_ns: float, n_new: int) -> int:
    """k_ns = ceil(alpha_ns * n_new - 1e-4) exact key blocks per Taylor query block (0 for alpha_ns = 0)."""
    if alpha_ns <= 0:
        return 0
    return max(0, min(n_new, math.ceil(float(np.float32(alpha_ns)) * n_new - 1e-4)))


def _cdiv(a: int, b: int) -> int:
    return -(-a // b)


def flops_per_call(w, alpha_ns: float = 0.0) -> dict:
    """Multiply-adds of each stage x 2 for one call over all B*H slices (the pass's own counts).

    With alpha_ns > 0 a Taylor query row attends to the n_new - k_ns pooled rows
    and the k_ns * b keys of its exact blocks. With short last blocks (b dividing
    neither length) every block counts b rows and b keys: the work the kernels execute."""
    n_src, n_ctx = _cdiv(w.L_src, w.b), _cdiv(w.L_ctx, w.b)
    n_q = n_src + n_ctx
    k = max(0, min(n_ctx, math.ceil(float(np.float32(w.alpha_s)) * n_ctx - 1e-4)))
    n_flat = max(0, min(n_q, math.floor(float(np.float32(w.alpha_f)) * n_q + 1e-4)))
    n_new = n_src + k
    k_ns = no_sparse_count(alpha_ns, n_new)
    bh = w.B * w.H
    f = dict(coarse=2.0 * n_src * n_q * w.D * bh, route=2.0 * n_q * n_new * w.D * bh,
             exact=4.0 * (n_q - n_flat) * w.b * n_new * w.b * w.D * bh,
             taylor=4.0 * n_flat * w.b * ((n_new - k_ns) + k_ns * w.b) * w.D * bh)
    f["total"] = sum(f.values())
    return f


def hbm_bytes_per_call(w) -> dict:
    """Algorithmic HBM bytes of the pooling/top-k stage (read Q, K, V once) and the gather."""
    e = 2 if w.dtype == "bf16" else 4
    N = w.L_src + w.L_ctx
    n_ctx = _cdiv(w.L_ctx, w.b)
    k = max(0, min(n_ctx, math.ceil(float(np.float32(w.alpha_s)) * n_ctx - 1e-4)))
    return dict(pool=3.0 * w.B * w.H * N * w.D * e, gather=2.0 * 2.0 * w.B * w.H * k * w.b * w.D * e)


def pass_roofline(f: dict, hb: dict, ms: float, tflops: float, gbs: float) -> dict:
    """Whole-pass roofline: the attention FLOPs at `tflops` plus the pool and gather bytes at `gbs`,
    as a time, and that time over the measured `ms`."""
    t = (f["exact"] + f["taylor"]) / (tflops * 1e12) + (hb["pool"] + hb["gather"]) / (gbs * 1e9)
    return {"t_roof_ms": t * 1e3, "frac": t * 1e3 / ms}


def attention_source_sha1(w) -> str:
    """sha1 of the attention kernel source this workload runs on (CTA pairs for bf16 D=128)."""
    import hashlib
    name = "k_attention_pair.cu" if (w.dtype == "bf16" and w.D == 128) else "k_attention.cu"
    with open(os.path.join(ROOT, "block_sparse_attention_isa_b200", "csrc", name), "rb") as fh:
        return hashlib.sha1(fh.read()).hexdigest()


def reduce_max(x: float, dist=None) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    if dist is None or not dist.is_initialized():
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(flops_per_rank: float, max_ms: float, world: int) -> float:
    """Whole-job TFLOP/s: all ranks' FLOPs over the slowest rank's time."""
    return flops_per_rank * world / (max_ms * 1e-3) / 1e12


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except FileNotFoundError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.flush()
        with open(self.f.name) as g:
            rows = [r.strip().split(", ") for r in g if r.strip()]
        os.unlink(self.f.name)
        sm, mx, pw, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
                pw.append(float(r[3]))
            except ValueError:
                continue
            for n, val in zip(names, r[5:9]):
                if val.strip().lower() == "active":
                    reasons.add(n)
        busy = [s for s, p in zip(sm, pw) if p > 200] or sm
        return {"sm_mhz": statistics.median(busy) if busy else None, "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(pw) if pw else None, "samples": len(sm), "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------- arms

def workload_inputs(w, seed=0, full=None, batch=0):
    """Q, K, V of workload w; with `full` (w = full with fewer heads) its first heads, same draws.

    `batch` > 0 draws batch element `batch` instead (B = 1; the weak-scaling unit of rank `batch`)."""
    if batch:
        q = np.zeros((1, w.H, w.N, w.D), np.float32)
        k, v = np.zeros_like(q), np.zeros_like(q)
        for h in range(w.H):
            q[0, h], k[0, h], v[0, h] = isa_synth.make_slice(w, seed, batch, h, 0)
        return q, k, v
    att = isa_synth.attempts_for(full or w, seed)
    if att is not None and full is not None:
        att = att[:, :w.H]
    return isa_synth.make_inputs(w, seed, att)


def roofline_peak(peaks: dict, timed_s: float) -> tuple:
    """(peak TFLOP/s, kind) for a kernel timed over `timed_s` seconds: the burst GEMM figure
    when the timed region is shorter than a second (below the power cap's reaction time),
    else the sustained one."""
    if timed_s < 1.0 or "bf16_tflops_sustained" not in peaks:
        return peaks["bf16_tflops"], "burst"
    return peaks["bf16_tflops_sustained"], "sustained"


def bf16_bits(x):
    return isa_synth.round_to_bf16_bits(x)


def is_ragged(w) -> bool:
    return bool(w.L_src % w.b or w.L_ctx % w.b)


def cpu_oracle_sample(w, q, k, v, heads, seconds_cap=60.0, alpha_ns=0.0):
    """Run the oracle on some heads; returns (TFLOP/s, seconds, heads done)."""
    from oracle import isa_oracle as O
    from oracle import isa_oracle_ragged as R
    f = flops_per_call(w, alpha_ns)["total"] / (w.B * w.H)
    t0 = time.perf_counter()
    done = 0
    for h in heads:
        if is_ragged(w):
            R.isa_slice_ref_ragged(q[0, h], k[0, h], v[0, h], w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, alpha_ns)
        else:
            O.isa_slice_ref(q[0, h], k[0, h], v[0, h], w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f,
                            alpha_ns=alpha_ns)
        done += 1
        if time.perf_counter() - t0 > seconds_cap:
            break
    dt = time.perf_counter() - t0
    return f * done / dt / 1e12, dt, done


def workload_label(args, w) -> str:
    label = w.name + (f" (first {w.H} heads)" if args.heads else "")
    return label + (f", alpha_ns={args.alpha_ns:g}" if args.alpha_ns else "")


def run_reference(args, w):
    """The CPU oracle as it stands. Each step is a bounded sample of the workload: the context
    selection and routing of one head, then the output rows of every eighth query block of that
    head (both paths in their natural proportion); the work counted is exactly that sample's."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    if is_ragged(w):
        return run_reference_whole_heads(args, w)
    import numpy as np
    from oracle import isa_oracle as O
    n_heads = min(w.B * w.H, max(1, args.steps + args.warmup))
    att = isa_synth.attempts_for(getattr(args, "full_workload", None) or w, 0)
    if att is not None:
        att = att[:, :w.H]
    q, k, v = isa_synth.make_inputs(w, 0, att, heads=[(0, h) for h in range(n_heads)])
    parts = 8
    n_q = w.N // w.b
    kk = O.kept_context_blocks(w.alpha_s, w.L_ctx // w.b)
    n_new = w.L_src // w.b + kk
    per_head = O.executed_flops(1, 1, w.L_src, w.L_ctx, w.D, w.b, w.alpha_s, w.alpha_f)
    sel_route_flops = per_head["coarse"] + per_head["route"]
    a_ns = args.alpha_ns
    k_ns = no_sparse_count(a_ns, n_new)

    def step(s):
        h = s % n_heads
        sr = O.isa_select_route_ref(q[0, h], k[0, h], w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, a_ns)
        blocks = np.arange(s % parts, n_q, parts)
        rows = (blocks[:, None] * w.b + np.arange(w.b)[None, :]).ravel()
        O.isa_rows_ref(q[0, h], k[0, h], v[0, h], w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, rows, sr=sr,
                       alpha_ns=a_ns)
        taylor = set(int(t) for t in sr["taylor"])
        n_t = sum(int(bl) in taylor for bl in blocks)
        return sel_route_flops + 4.0 * w.b * w.D * ((len(blocks) - n_t) * n_new * w.b +
                                                     n_t * ((n_new - k_ns) + k_ns * w.b))

    for s in range(args.warmup):
        step(s)
    t0 = time.perf_counter()
    flops = sum(step(args.warmup + s) for s in range(args.steps))
    dt = time.perf_counter() - t0
    value = flops / dt / 1e12
    cores = os.cpu_count()
    sample = (f"per step: selection and routing of one head, then the rows of every {parts}th query block "
              f"of it ({args.steps} steps over {n_heads} of {w.B * w.H} heads)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": workload_label(args, w), "B": w.B, "H": w.H,
                       "N": w.N, "D": w.D, "b": w.b, "alpha_s": w.alpha_s, "alpha_f": w.alpha_f,
                       "alpha_ns": args.alpha_ns, "sample": sample},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_reference_whole_heads(args, w):
    """The reference arm for ragged lengths: each step is the ragged-length oracle over one
    whole head of the workload (as it stands, on the host cores)."""
    from oracle import isa_oracle_ragged as R
    n_heads = min(w.B * w.H, max(1, args.steps + args.warmup))
    q, k, v = isa_synth.make_inputs(w, 0, None, heads=[(0, h) for h in range(n_heads)])
    per_head = flops_per_call(w, args.alpha_ns)["total"] / (w.B * w.H)

    def step(s):
        h = s % n_heads
        R.isa_slice_ref_ragged(q[0, h], k[0, h], v[0, h], w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, args.alpha_ns)
        return per_head

    for s in range(args.warmup):
        step(s)
    t0 = time.perf_counter()
    flops = sum(step(args.warmup + s) for s in range(args.steps))
    dt = time.perf_counter() - t0
    value = flops / dt / 1e12
    sample = f"per step: one whole head ({args.steps} steps over {n_heads} of {w.B * w.H} heads)"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_label(args, w), "B": w.B, "H": w.H, "N": w.N, "D": w.D, "b": w.b,
                       "alpha_s": w.alpha_s, "alpha_f": w.alpha_f, "alpha_ns": args.alpha_ns, "sample": sample},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, w):
    import torch
    import torch.distributed as dist

    import block_sparse_attention_isa_b200 as isa
    from block_sparse_attention_isa_b200 import build as isa_build
    from block_sparse_attention_isa_b200 import sharding

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", device_id=torch.device("cuda", local),
                                timeout=__import__("datetime").timedelta(seconds=300))
    isa_build.build()
    dev = torch.device("cuda", local)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    strong = args.scaling == "strong" and world > 1

    # weak scaling: rank r computes its own batch element r; strong: rank r computes its range of
    # the workload's slices (every rank draws the same whole workload and uses its range)
    q, k, v = workload_inputs(w, full=getattr(args, "full_workload", None), batch=0 if strong else rank)
    tq, tk, tv = (torch.from_numpy(x).to(dev, dt) for x in (q, k, v))
    s0, s1 = sharding.slice_range(rank, world, w.B * w.H) if strong else (0, w.B * w.H)
    wr = w.with_(B=1, H=s1 - s0) if strong else w  # this rank's call
    if strong:
        tq, tk, tv = (t.reshape(w.B * w.H, w.N, w.D)[s0:s1].unsqueeze(0).contiguous() for t in (tq, tk, tv))
    out = torch.empty_like(tq)
    a_ns = args.alpha_ns
    dtc = isa.ISA_BF16 if w.dtype == "bf16" else isa.ISA_F32
    ws = torch.empty(isa.workspace_bytes(wr.B, wr.H, w.L_src, w.L_ctx, w.D, w.b, w.alpha_s, dtc, alpha_ns=a_ns),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    gather = strong and args.gather

    def step():
        isa.forward_into(tq, tk, tv, out, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, workspace=ws, stream=stream,
                         alpha_ns=a_ns)
        if gather:
            sharding.gather_output(out.reshape(s1 - s0, w.N, w.D), w.B, w.H)

    for _ in range(args.warmup):
        step()
    isa.device_status(ws, stream)

    # per-kernel events for every timed step
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    for row in ev:
        for e in row:
            e.record(stream)
    torch.cuda.synchronize()

    clocks = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ else local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for s in range(args.steps):
        isa.set_stage_events(ev[s])
        step()
    end.record(stream)
    isa.set_stage_events(None)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    isa.device_status(ws, stream)

    ms = start.elapsed_time(end) / args.steps
    max_ms = reduce_max(ms, dist)
    stage_ms = {name: sum(ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(args.steps)) / args.steps
                for i, name in enumerate(isa.STAGES)}
    f = flops_per_call(wr, a_ns)          # this rank's call
    f_job = flops_per_call(w, a_ns)       # one unit of the whole job (the workload)
    hb = hbm_bytes_per_call(wr)
    peaks, peaks_kind = load_peaks()
    attn_tflops = (f["exact"] + f["taylor"]) / (stage_ms["attention"] * 1e-3) / 1e12
    peak, peak_which = roofline_peak(peaks, args.steps * ms * 1e-3)
    peak_sust = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    pool_gbs = hb["pool"] / (stage_ms["pool_score_topk"] * 1e-3) / 1e9
    gather_gbs = hb["gather"] / max(stage_ms["gather"] * 1e-3, 1e-12) / 1e9
    # clock-normalised: the attention time scaled to the maximum SM clock (a power-capped run
    # that ran at a lower median clock reads as the same kernel at full clock)
    clock_ratio = (clk["sm_mhz"] / clk["sm_max_mhz"]) if clk.get("sm_mhz") and clk.get("sm_max_mhz") else None
    traffic = None
    prof = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(prof) and not a_ns and not strong:  # (counters of the plain path's attention kernel only)
        with open(prof) as fh:
            ent = json.load(fh).get(w.name, {})
        # the counters hold only for the kernel source they were taken on
        if ent.get("kernel_source_sha1") == attention_source_sha1(w):
            traffic = ent.get("attention")

    # end to end through the host-buffer entry point (pinned host memory, copies inside the timed region)
    e2e = None
    if not args.no_e2e and (rank == 0 or world > 1):
        hq, hk, hv = (t.cpu().pin_memory() for t in (tq, tk, tv))
        hout = torch.empty_like(hq).pin_memory()
        n_e2e = max(1, min(args.steps, 5))
        isa.forward_host(hq, hk, hv, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, out=hout, alpha_ns=a_ns)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for _ in range(n_e2e):
            isa.forward_host(hq, hk, hv, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, out=hout, alpha_ns=a_ns)
        e2e_ms = (time.perf_counter() - t0) / n_e2e * 1e3
        e2e_ms = reduce_max(e2e_ms, dist)
        nbytes = hq.numel() * hq.element_size()
        e2e_val = f_job["total"] / (e2e_ms * 1e-3) / 1e12 if strong else aggregate(f["total"], e2e_ms, world)
        e2e = {"value": e2e_val, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": 3 * nbytes, "d2h_bytes_per_step": nbytes}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tf, secs, done = cpu_oracle_sample(w, q, k, v, heads=range(w.H), seconds_cap=args.cpu_seconds,
                                           alpha_ns=a_ns)
        cpu = {"value": tf, "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
               "sample": f"{done} of {w.B * w.H} heads of the same workload, {secs:.1f} s of CPU time"}

    launches = isa.launch_count(wr.B, wr.H, w.L_src, w.L_ctx, w.D, w.b, w.alpha_s, w.alpha_f, dtc, alpha_ns=a_ns)
    if rank == 0:
        value = f_job["total"] / (max_ms * 1e-3) / 1e12 if strong else aggregate(f["total"], max_ms, world)
        parallelism = (f"heads split over {world} ranks" + (" + NCCL all-gather of O" if gather else "")
                       if strong else (f"dp{world} (rank r computes batch element r)" if world > 1 else "single GPU"))
        exact_t = f["exact"] / (stage_ms["attention"] * 1e-3) / 1e12
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": max_ms, "higher_is_better": True,
            "scaling": "strong" if strong else "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
            "config": {"workload": workload_label(args, w), "B": w.B, "H": w.H, "N": w.N, "D": w.D, "b": w.b,
                       "alpha_s": w.alpha_s, "alpha_f": w.alpha_f, "alpha_ns": a_ns,
                       "global_batch": w.B if strong else w.B * world, "seq_len": w.N, "parallelism": parallelism,
                       "l2": "inputs larger than L2 (Q, K, V = %.2f GB per step)" % (3 * tq.numel() * tq.element_size() / 1e9)},
            "roofline": {"bound": "tensor", "kernel": "attention (exact + Taylor paths)", "achieved": attn_tflops,
                         "peak": peak, "unit": "TFLOP/s", "frac": attn_tflops / peak,
                         "peak_kind": f"{peaks_kind} bf16 {peak_which} (timed region {args.steps * ms / 1e3:.2f} s)",
                         "frac_of_burst": attn_tflops / peaks["bf16_tflops"],
                         "frac_of_sustained": attn_tflops / peak_sust,
                         "frac_of_nominal": attn_tflops / NOMINAL["bf16_tflops"],
                         # the exact path's FLOPs over the whole attention time (Taylor items included):
                         # a lower bound on the exact path's own fraction
                         "exact_path_frac_lower_bound": exact_t / peak,
                         "flops_share": {"exact": f["exact"] / (f["exact"] + f["taylor"]),
                                         "taylor": f["taylor"] / (f["exact"] + f["taylor"])},
                         "traffic": traffic},
            # time x (median SM clock / max clock): what the stage would take at the max clock if it
            # scaled with the clock alone, against the burst peak (the one measured near the max
            # clock; the sustained peak was measured at the power-capped clock)
            "clock_normalised": None if clock_ratio is None else {
                "sm_mhz_median": clk["sm_mhz"], "sm_max_mhz": clk["sm_max_mhz"],
                "attention_ms_at_max_clock": stage_ms["attention"] * clock_ratio,
                "frac_at_max_clock": attn_tflops / clock_ratio / peaks["bf16_tflops"],
                "peak_kind": "measured bf16 burst" if peaks_kind == "measured" else "fallback bf16 burst"},
            "pass_roofline": {"measured": pass_roofline(f, hb, ms, peak, peaks["hbm_gbs"]),
                              "nominal": pass_roofline(f, hb, ms, NOMINAL["bf16_tflops"], NOMINAL["hbm_gbs"])},
            "stages_ms": stage_ms,
            "hbm_stages": {"pool_score_topk_gbs": pool_gbs, "gather_gbs": gather_gbs,
                           "pool_frac": pool_gbs / peaks["hbm_gbs"], "gather_frac": gather_gbs / peaks["hbm_gbs"],
                           "peak_gbs": peaks["hbm_gbs"], "peak_kind": peaks_kind,
                           "pool_frac_of_nominal": pool_gbs / NOMINAL["hbm_gbs"],
                           "gather_frac_of_nominal": gather_gbs / NOMINAL["hbm_gbs"]},
            "flops_per_call": f,
            "gpu_launches": launches * args.steps,
            "clocks": clk,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def backward_flops_per_call(w) -> dict:
    """FLOPs of the backward pass: algorithmic = the five products per path (S and dP recomputed,
    dV, dK, dQ), each 2 * rows * keys * D; executed = the seven the two kernels issue (S and dP are
    computed once in the dQ kernel and once, transposed, in the dK/dV kernel)."""
    n_src, n_ctx = _cdiv(w.L_src, w.b), _cdiv(w.L_ctx, w.b)
    n_q = n_src + n_ctx
    k = max(0, min(n_ctx, math.ceil(float(np.float32(w.alpha_s)) * n_ctx - 1e-4)))
    n_flat = max(0, min(n_q, math.floor(float(np.float32(w.alpha_f)) * n_q + 1e-4)))
    n_new = n_src + k
    bh = w.B * w.H
    unit = 2.0 * w.D * bh * w.b * ((n_q - n_flat) * n_new * w.b + n_flat * n_new)
    return {"algorithmic": 5.0 * unit, "executed": 7.0 * unit}


def run_backward(args, w):
    """Time the backward pass (isa_backward, after one training forward) at this workload."""
    import torch
    import block_sparse_attention_isa_b200 as isa
    from block_sparse_attention_isa_b200 import build as isa_build
    torch.cuda.set_device(0)
    isa_build.build()
    dev = torch.device("cuda", 0)
    q, k, v = workload_inputs(w, full=getattr(args, "full_workload", None))
    tq, tk, tv = (torch.from_numpy(x).to(dev, torch.bfloat16) for x in (q, k, v))
    g = torch.randn(tq.shape, generator=torch.Generator().manual_seed(5)).to(dev, torch.bfloat16)
    out, lse, ws = isa.forward_train(tq, tk, tv, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
    nb = isa.lib().isa_backward_workspace_bytes(w.B, w.H, w.L_src, w.L_ctx, w.D, w.b, w.alpha_s, 0)
    bws = torch.empty(nb, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        isa.backward(tq, tk, tv, out, lse, g, ws, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, bwd_workspace=bws)
    isa.device_status(ws)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.3)
    start.record()
    for _ in range(args.steps):
        isa.backward(tq, tk, tv, out, lse, g, ws, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, bwd_workspace=bws)
    end.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    isa.device_status(ws)
    ms = start.elapsed_time(end) / args.steps
    f = backward_flops_per_call(w)
    peaks, kind = load_peaks()
    peak, which = roofline_peak(peaks, args.steps * ms * 1e-3)
    line = {"metric": "ISA backward ms/call and TFLOPS", "value": f["algorithmic"] / (ms * 1e-3) / 1e12,
            "unit": "TFLOP/s", "ms_per_step": ms, "steps": args.steps, "warmup": args.warmup, "dtype": "bf16",
            "config": {"workload": workload_label(args, w), "B": w.B, "H": w.H, "N": w.N, "D": w.D, "b": w.b,
                       "alpha_s": w.alpha_s, "alpha_f": w.alpha_f},
            "flops": f, "executed_tflops": f["executed"] / (ms * 1e-3) / 1e12,
            "frac_algorithmic": f["algorithmic"] / (ms * 1e-3) / 1e12 / peak,
            "frac_executed": f["executed"] / (ms * 1e-3) / 1e12 / peak,
            "peak": peak, "peak_kind": f"{kind} bf16 {which}", "clocks": clk}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=isa_synth.HEADLINE)
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end measurement")
    ap.add_argument("--alpha-ns", type=float, default=0.0,
                    help="no-sparsity ratio: exact key blocks inside the Taylor path (bf16 only; 0 = plain path)")
    ap.add_argument("--scaling", default="weak", choices=["weak", "strong"],
                    help="N > 1: weak = one batch element per rank; strong = the workload's heads split over ranks")
    ap.add_argument("--gather", action="store_true", help="strong scaling: all-gather O over NCCL in every step")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward pass (training) instead of the forward; one GPU, not a bench line")
    ap.add_argument("--heads", type=int, default=0,
                    help="run only the first H heads of the workload (small profiling captures; not a bench line)")
    args = ap.parse_args()
    w = {**isa_synth.all_workloads(), **isa_synth.RAGGED}[args.workload]
    args.full_workload = None
    if args.heads:
        args.full_workload = w
        w = w.with_(H=min(args.heads, w.H))
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps
    if args.backward:
        run_backward(args, w)
    elif args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()

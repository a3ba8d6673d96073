#!/usr/bin/env python
"""Benchmark: full 3D-RoPE attention throughput on B200.

Headline metric: full 3D-RoPE attention TFLOP/s (4*N^2*d*heads per forward)
and its fraction of the measured B200 dense bf16 peak, on the 81-frame
480x832 clip: T'xH'xW' = 21x30x52 = 32,760 tokens, 12 heads x 128, B=1,
RoPE split (44, 42, 42), seeded synthetic bf16 N(0,1) inputs.

A step is one pass of the whole hot path: key RoPE pre-pass (rope3d_apply),
angle table, and the fused Q-RoPE + attention kernel.  Inputs are resident
in HBM before timing; Q, K, V and O together (403 MB) exceed the 126 MB L2.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--parallel replicas|ulysses]

For N > 1 launch one process per GPU with torch.distributed.run; by default
every rank runs an independent replica of the workload (weak scaling, no
collective on the data path) and rank 0 prints one JSON line.  With
--parallel ulysses the ranks split one sequence (strong scaling): token
slices are exchanged for head groups over peer memory and back.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

HEAD_DIM = 128
METRIC = "full 3D-RoPE attention TFLOP/s and % of B200 BF16 peak at 32,760 tokens"
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="c81f480")
    p.add_argument("--e2e-steps", type=int, default=None,
                   help="steps of the end-to-end loop (default: --steps); the pipelined loop's "
                        "first upload and last download are not overlapped, so they are spread "
                        "over these steps")
    p.add_argument("--no-extras", action="store_true", help="skip the secondary measurements")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-rows", type=int, default=512, help="oracle rows per head for cpu_baseline")
    p.add_argument("--parallel", choices=["replicas", "ulysses", "ring"], default="replicas",
                   help="N > 1: independent replicas per rank (default), or one sequence split "
                        "over the ranks with context parallelism, strong scaling: ulysses (token "
                        "slices <-> head groups; heads and tokens divide by N) or ring (K/V "
                        "blocks passed around; tokens divide by N)")
    p.add_argument("--case", choices=["temporal720", "spatial720", "window720", "cross720"],
                   help="run only this secondary kernel (warm-up + --steps launches, one "
                        "JSON line); a small, single-kernel command for profilers")
    args = p.parse_args()
    if args.e2e_steps is None:
        args.e2e_steps = args.steps
    return args


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, FALLBACK_HBM_GBS, "fallback"


def sustained_peak():
    """The measured sustained bf16 figure (seconds-long loop under the power
    cap), or None."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops_sustained"])
    except Exception:
        return None


def strip_comments(src):
    """C/C++ source without its comments and with runs of white space folded,
    so that a comment edit does not change a kernel's hash."""
    import re
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


def kernel_source_hash(files):
    """SHA-256 (16 hex digits) over the listed kernel sources, comments and
    white space excluded."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "full_spatiotemporal_attention_b200", "csrc")
    for f in files:
        with open(os.path.join(csrc, f), encoding="utf-8") as fh:
            h.update(f.encode() + b"\0" + strip_comments(fh.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current sources of that kernel (its `source_hash` over the listed
    `source_files` matches); otherwise None."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}_ncu.md")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and line.startswith("- "):
                key, _, val = line[2:].partition(":")
                vals[key.strip()] = val.strip().strip("`")
    try:
        if vals.get("source_hash") != kernel_source_hash(vals["source_files"].split(",")):
            return None
        return float(vals["dram_bytes_per_launch_full_size"])
    except (KeyError, ValueError, OSError):
        return None


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons during the timed region."""
    FIELDS = ("timestamp,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None

    def stop(self, t0=None, t1=None):
        """Stop sampling; keep the samples taken between wall times t0 and t1."""
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9 or (self.uuid and parts[1] != self.uuid):
                continue
            try:
                ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                ts += float("0." + parts[0].split(".")[1]) if "." in parts[0] else 0.0
                clk, cmax = float(parts[2]), float(parts[3])
            except ValueError:
                continue
            if t0 is not None and not (t0 - 0.05 <= ts <= t1 + 0.05):
                continue
            sm.append(clk)
            mx = cmax
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "samples": len(sm),
                "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------

def init_dist(backend="nccl"):
    """Join the job's process group when launched with WORLD_SIZE > 1 (one
    process per GPU, rendezvous from the MASTER_* environment).  The CPU
    tests use backend "gloo", which binds no GPU."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        if backend == "nccl":
            import torch
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def max_over_ranks(x, world, device):
    """The largest of every rank's x (the job's time is its slowest rank's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


REPLICA_SEED_STRIDE = 7919


def replica_workload(w, rank):
    """Rank r's replica: the same shapes with its own seed, so that the ranks
    of a weak-scaling job attend over independent sequences (rank 0 keeps the
    workload's own seed, hence the 1-GPU line's inputs)."""
    import dataclasses
    return w if rank == 0 else dataclasses.replace(w, seed=w.seed + REPLICA_SEED_STRIDE * rank)


def job_tflops(flops_per_rank, world, ms):
    """Whole-job throughput: every rank's FLOPs over the slowest rank's time."""
    return world * flops_per_rank / (ms / 1e3) / 1e12


def job_config(w, world):
    return {"workload": w.description, "grid": [w.T, w.H, w.W], "tokens": w.N,
            "heads": w.heads, "head_dim": HEAD_DIM, "batch": w.batch,
            "rope_split": list(w.dims), "theta": w.theta,
            "flops_per_step": full_flops(w), "global_batch": w.batch * world, "seq_len": w.N,
            "parallelism": f"replicas x{world} (independent sequences, no collective)",
            "l2": l2_note(w)}


def l2_note(w):
    mb = 4 * w.batch * w.heads * w.N * HEAD_DIM * 2 / 1e6
    if mb > 126:
        return f"inputs exceed L2 (Q,K,V,O = {mb:.0f} MB > 126 MB); no flush"
    return f"inputs fit in L2 (Q,K,V,O = {mb:.1f} MB)"


def to_dev(bits, device):
    import torch
    return torch.from_numpy(bits).view(torch.bfloat16).to(device)


def full_flops(w):
    return 4.0 * w.N * w.N * HEAD_DIM * w.heads * w.batch


def cpu_baseline(w, q, k, v, rows_per_head):
    import oracle
    import seeded_inputs as si
    og = oracle.Grid(w.T, w.H, w.W, w.n_text, w.dims, w.theta)
    rows = si.sample_rows(w, rows_per_head)
    t0 = time.perf_counter()
    oracle.attention(q, k, v, og, rows=rows)
    dt = time.perf_counter() - t0
    flops = w.batch * w.heads * rows.size * 4.0 * w.N * HEAD_DIM
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{rows.size} seeded query rows x {w.batch * w.heads} heads of {w.name} "
                      f"(N={w.N}); includes rotating all keys; {dt:.1f} s",
            "seconds": round(dt, 3),
            "extrapolated_full_forward_s": round(dt * w.N / rows.size, 1)}


def timed_loop(fn, steps, warmup, world, device, window=None):
    """Run fn(i) warmup times untimed, then `steps` times between CUDA events.
    fn may return a pair of events bracketing its dominant kernel.  If
    `window` is a list, the wall-clock start and end of the timed region are
    appended to it."""
    import torch
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize()
    barrier(world)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    inner = []
    if window is not None:
        window.append(time.time())
    start.record()
    for i in range(steps):
        ev = fn(i)
        if ev is not None:
            inner.append(ev)
    end.record()
    torch.cuda.synchronize()
    if window is not None:
        window.append(time.time())
    barrier(world)
    total = start.elapsed_time(end)
    inner_ms = [a.elapsed_time(b) for a, b in inner]
    return total / steps, (sum(inner_ms) / len(inner_ms) if inner_ms else None)


def e2e_pipelined(va, g, w, host_bits, steps, world, device, warmup=3):
    """Per-step time of the end-to-end loop through the public API: each step
    copies its Q, K, V from pinned host memory (H2D), runs attn3d_full_fwd
    (key pre-pass, table, attention) and reads its O back (D2H).  Device
    buffers are double-buffered and the copies run on their own streams, so
    step i+1's upload and step i-1's download overlap step i's kernels, as a
    serving loop streams requests; the timed region starts before the first
    upload and ends after the last download."""
    import torch
    comp = torch.cuda.current_stream(device)
    up = torch.cuda.Stream(device)
    down = torch.cuda.Stream(device)
    qh, kh, vh = (torch.from_numpy(x).view(torch.bfloat16).pin_memory() for x in host_bits)
    dev_in = [[torch.empty(qh.shape, dtype=torch.bfloat16, device=device) for _ in range(3)]
              for _ in range(2)]
    dev_out = [torch.empty(qh.shape, dtype=torch.bfloat16, device=device) for _ in range(2)]
    host_out = [torch.empty(qh.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    ws = torch.empty(va.workspace_bytes(w.batch, w.heads, w.N, g), dtype=torch.uint8, device=device)
    ev = lambda: torch.cuda.Event()
    uploaded, computed, downloaded = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def upload(i):
        b = i % 2
        with torch.cuda.stream(up):
            if i >= 2:
                up.wait_event(computed[b])          # step i-2 has read these buffers
            for d, h in zip(dev_in[b], (qh, kh, vh)):
                d.copy_(h, non_blocking=True)
            uploaded[b].record(up)

    def run(n, start=None):
        if start is not None:
            up.wait_event(start)
        upload(0)
        for i in range(n):
            b = i % 2
            if i + 1 < n:
                upload(i + 1)
            comp.wait_event(uploaded[b])
            if i >= 2:
                comp.wait_event(downloaded[b])      # step i-2's O has left this buffer
            q, k, v = dev_in[b]
            va.attn3d_full_fwd(q, k, v, g, out=dev_out[b], workspace=ws)
            computed[b].record(comp)
            with torch.cuda.stream(down):
                down.wait_event(computed[b])
                host_out[b].copy_(dev_out[b], non_blocking=True)
                downloaded[b].record(down)
        comp.wait_stream(down)
        comp.wait_stream(up)

    run(warmup)
    torch.cuda.synchronize()
    barrier(world)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(comp)
    run(steps, start=a)
    b.record(comp)
    torch.cuda.synchronize()
    barrier(world)
    return max_over_ranks(a.elapsed_time(b) / steps, world, device)


def bench_ours(args, rank, world, local):
    import torch
    import full_spatiotemporal_attention_b200 as va
    import seeded_inputs as si

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = replica_workload(si.WORKLOADS[args.workload], rank)
    qb, kb, vb = si.qkv(w)
    q, k, v = (to_dev(x, device) for x in (qb, kb, vb))
    g = va.Grid.make(w.T, w.H, w.W, w.n_text, w.dims, w.theta)
    kr = torch.empty_like(k)
    o = torch.empty_like(q)
    ws = torch.empty(va.workspace_bytes(w.batch, w.heads, w.N, g, k_rotated=True),
                     dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def step(i):
        # key pre-pass, then (table + fused Q-RoPE attention) bracketed by events
        va.rope3d_apply(k, g, out=kr)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        va.attn3d_full_fwd(q, kr, v, g, k_rotated=True, out=o, workspace=ws)
        b.record(stream)
        return a, b

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.5)
    window = []
    step_ms, attn_ms = timed_loop(step, args.steps, args.warmup, world, device, window=window)
    clocks = sampler.stop(*window)
    step_ms = max_over_ranks(step_ms, world, device)
    attn_ms = max_over_ranks(attn_ms, world, device)

    # key pre-pass alone (HBM-bound): bytes = read + write of K
    def rope_only(i):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        va.rope3d_apply(k, g, out=kr)
        b.record(stream)
        return a, b
    _, rope_ms = timed_loop(rope_only, max(args.steps, 10), 3, world, device)

    flops = full_flops(w)
    value = job_tflops(flops, world, step_ms)
    peak_tf, peak_gbs, peak_src = peaks()
    achieved = flops / (attn_ms / 1e3) / 1e12
    traffic = recorded_traffic("attn_fwd_kernel", w.name)

    # end to end through the public API with host buffers
    tensor_bytes = w.batch * w.heads * w.N * HEAD_DIM * 2
    e2e_ms = e2e_pipelined(va, g, w, (qb, kb, vb), args.e2e_steps, world, device)

    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded splitmix64 + Box-Muller bf16 N(0,1))",
        "config": job_config(w, world),
        "pct_of_peak": round(100.0 * value / world / peak_tf, 2),
        "e2e": {"value": round(job_tflops(flops, world, e2e_ms), 2), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms, 4),
                "h2d_bytes_per_step": 3 * tensor_bytes, "d2h_bytes_per_step": tensor_bytes,
                "pipelined": "double-buffered: step i+1's H2D and step i-1's D2H overlap "
                             "step i's kernels; every step's own copies are in the timed region"},
        "gpu_launches": 3 * args.steps,
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak_tf,
                     "unit": "TFLOP/s", "frac": round(achieved / peak_tf, 4),
                     "traffic": traffic, "kernel": "attn_fwd_kernel",
                     "peak_source": f"{peak_src} bf16 dense (burst)",
                     "kernel_ms": round(attn_ms, 4),
                     # context: the same kernel against the measured sustained
                     # figure (a seconds-long GEMM loop under the power cap)
                     "peak_sustained": sustained_peak(),
                     "frac_sustained": (round(achieved / sustained_peak(), 4)
                                        if sustained_peak() else None)},
        "rope_prepass": {"kernel": "rope_apply_kernel", "ms": round(rope_ms, 4),
                         "achieved_gbs": round(2 * tensor_bytes / (rope_ms / 1e3) / 1e9, 1),
                         "peak_gbs": peak_gbs,
                         "frac": round(2 * tensor_bytes / (rope_ms / 1e3) / 1e9 / peak_gbs, 4)},
        "clocks": clocks,
    }
    # The kernel is bound by the SM clock (tensor and softmax pipes), which
    # the power cap sets: its time in clock cycles is the clock-free figure.
    if clocks and clocks.get("sm_mhz") and clocks.get("sm_max_mhz"):
        line["roofline"]["clock_normalised"] = {
            "kernel_mcycles": round(attn_ms * clocks["sm_mhz"] / 1e3, 4),
            "achieved_at_max_clock": round(achieved * clocks["sm_max_mhz"] / clocks["sm_mhz"], 2),
            "note": "kernel time x median SM clock of the timed region; achieved scaled to sm_max_mhz",
        }

    if world == 1 and not args.no_extras:
        line["extras"] = extras(va, device, stream, peak_tf, peak_gbs)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, qb, kb, vb, args.cpu_rows)
    return line


def extras(va, device, stream, peak_tf, peak_gbs):
    """Secondary measurements: full vs factorised on the 720p clip (with the
    temporal pass in GB/s) and joint video+text attention."""
    import torch
    import seeded_inputs as si
    out = {}

    def ev_pair(fn):
        def run(i):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            return a, b
        return run

    # the 17-frame clip: full vs factorised cost ratio at 7,800 tokens
    w = si.WORKLOADS["c17f480"]
    q, k, v = (to_dev(x, device) for x in si.qkv(w))
    g = va.Grid.make(w.T, w.H, w.W, w.n_text, w.dims, w.theta)
    kr = va.rope3d_apply(k, g)
    o = torch.empty_like(q)
    o2 = torch.empty_like(q)
    ws = torch.empty(va.workspace_bytes(w.batch, w.heads, w.N, g, k_rotated=True),
                     dtype=torch.uint8, device=device)
    _, s_full = timed_loop(ev_pair(lambda: va.attn3d_full_fwd(q, kr, v, g, k_rotated=True, out=o,
                                                               workspace=ws)), 20, 3, 1, device)
    _, s_fact = timed_loop(ev_pair(lambda: va.attn_factorized_fwd(
        q, kr, v, g, k_rotated=True, out_spatial=o, out_temporal=o2, workspace=ws)), 20, 3, 1, device)
    f_full = 4.0 * w.N ** 2 * HEAD_DIM * w.heads
    hw = w.H * w.W
    f_fact = 4.0 * HEAD_DIM * w.heads * (w.T * hw * hw + hw * w.T ** 2)
    out["c17f480"] = {"tokens": w.N, "heads": w.heads, "full_ms": round(s_full, 4),
                      "full_tflops": round(f_full / s_full / 1e9, 1),
                      "factorised_ms": round(s_fact, 4),
                      "full_over_factorised_time": round(s_full / s_fact, 2),
                      "full_over_factorised_flops": round(f_full / f_fact, 2)}
    del q, k, v, kr, o, o2, ws
    torch.cuda.empty_cache()

    w = si.WORKLOADS["c81f720"]
    q, k, v = (to_dev(x, device) for x in si.qkv(w))
    g = va.Grid.make(w.T, w.H, w.W, w.n_text, w.dims, w.theta)
    kr = va.rope3d_apply(k, g)
    o = torch.empty_like(q)
    o2 = torch.empty_like(q)
    # sized for raw keys (the temporal pass below takes them)
    ws = torch.empty(va.workspace_bytes(w.batch, w.heads, w.N, g, k_rotated=False),
                     dtype=torch.uint8, device=device)
    _, full_ms = timed_loop(ev_pair(lambda: va.attn3d_full_fwd(q, kr, v, g, k_rotated=True, out=o,
                                                               workspace=ws)), 3, 2, 1, device)
    _, sp_ms = timed_loop(ev_pair(lambda: va.attn_factorized_fwd(
        q, kr, v, g, temporal=False, k_rotated=True, out_spatial=o, workspace=ws)), 10, 3, 1, device)
    # the temporal pass as the factorised call runs it (raw keys: only the t
    # range is turned), and with keys that come rotated
    _, tp_ms = timed_loop(ev_pair(lambda: va.attn_factorized_fwd(
        q, k, v, g, spatial=False, out_temporal=o2, workspace=ws)), 10, 3, 1, device)
    _, tpr_ms = timed_loop(ev_pair(lambda: va.attn_factorized_fwd(
        q, kr, v, g, spatial=False, k_rotated=True, out_temporal=o2, workspace=ws)), 10, 3, 1, device)
    hw = w.H * w.W
    f_full = 4.0 * w.N ** 2 * HEAD_DIM * w.heads
    f_sp = 4.0 * HEAD_DIM * w.heads * w.T * hw * hw
    tbytes = 4 * w.heads * w.N * HEAD_DIM * 2
    out["c81f720"] = {
        "tokens": w.N, "heads": w.heads,
        "full_ms": round(full_ms, 3), "full_tflops": round(f_full / full_ms / 1e9, 1),
        "spatial_ms": round(sp_ms, 4), "spatial_tflops": round(f_sp / sp_ms / 1e9, 1),
        "temporal_ms": round(tp_ms, 4), "temporal_gbs": round(tbytes / tp_ms / 1e6, 1),
        "temporal_frac_hbm": round(tbytes / tp_ms / 1e6 / peak_gbs, 4),
        "temporal_rotated_k_ms": round(tpr_ms, 4),
        "temporal_rotated_k_gbs": round(tbytes / tpr_ms / 1e6, 1),
        "full_over_factorised_time": round(full_ms / (sp_ms + tp_ms), 2),
        "full_over_factorised_flops": round(f_full / (f_sp + 4.0 * HEAD_DIM * w.heads * hw * w.T ** 2), 2),
    }
    # local 3D windows of 3 x 9 x 16 = 432 tokens on the same clip (keys pre-rotated)
    win = (3, 9, 16)
    vol = win[0] * win[1] * win[2]
    _, w_ms = timed_loop(ev_pair(lambda: va.attn_window_fwd(q, kr, v, g, win, k_rotated=True,
                                                              out=o, workspace=ws)), 10, 3, 1, device)
    f_w = 4.0 * w.N * vol * HEAD_DIM * w.heads
    t_f = f_w / (peak_tf * 1e12) * 1e3
    t_b = tbytes / (peak_gbs * 1e9) * 1e3
    out["window720"] = {"window": list(win), "tokens": w.N, "heads": w.heads, "ms": round(w_ms, 4),
                        "tflops": round(f_w / w_ms / 1e9, 1), "gbs": round(tbytes / w_ms / 1e6, 1),
                        "roofline_ms": round(max(t_f, t_b), 4),
                        "frac_of_roofline": round(max(t_f, t_b) / w_ms, 4)}
    del q, k, v, kr, o, o2, ws
    torch.cuda.empty_cache()

    def full_only(name):
        w = si.WORKLOADS[name]
        q, k, v = (to_dev(x, device) for x in si.qkv(w))
        g = va.Grid.make(w.T, w.H, w.W, w.n_text, w.dims, w.theta)
        kr = va.rope3d_apply(k, g)
        o = torch.empty_like(q)
        ws = torch.empty(va.workspace_bytes(w.batch, w.heads, w.N, g, k_rotated=True),
                         dtype=torch.uint8, device=device)
        _, ms = timed_loop(ev_pair(lambda: va.attn3d_full_fwd(q, kr, v, g, k_rotated=True, out=o,
                                                               workspace=ws)), 3, 2, 1, device)
        del q, k, v, kr, o, ws
        torch.cuda.empty_cache()
        f = 4.0 * w.N ** 2 * HEAD_DIM * w.heads
        return {"tokens": w.N, "heads": w.heads, "ms": round(ms, 3),
                "tflops": round(f / ms / 1e9, 1), "frac_of_peak": round(f / ms / 1e9 / peak_tf, 4)}

    out["joint720"] = full_only("joint720")
    # three reference images appended to the 720p clip: the same 40 heads,
    # 87,888 tokens, so the time should grow like N^2 (x1.35)
    ref = full_only("refimg720")
    ref["over_c81f720_time"] = round(ref["ms"] / full_ms, 3)
    ref["over_c81f720_flops"] = round((ref["tokens"] / w.N) ** 2, 3)
    out["refimg720"] = ref

    # Wan text cross-attention: 75,600 video queries x 512 text keys, no RoPE
    w = si.WORKLOADS["cross720"]
    q, k, v = (to_dev(x, device) for x in si.qkv(w))
    o = torch.empty_like(q)
    ws = torch.empty(va.cross_workspace_bytes(w.batch, w.heads, w.N, w.n_kv), dtype=torch.uint8,
                     device=device)
    _, x_ms = timed_loop(ev_pair(lambda: va.attn_cross_fwd(q, k, v, out=o, workspace=ws)), 10, 3, 1,
                         device)
    f_x = 4.0 * w.N * w.n_kv * HEAD_DIM * w.heads
    b_x = 2 * (2 * w.N + 2 * w.n_kv) * HEAD_DIM * w.heads   # read Q, K, V; write O
    out["cross720"] = {"queries": w.N, "keys": w.n_kv, "heads": w.heads, "ms": round(x_ms, 4),
                       "tflops": round(f_x / x_ms / 1e9, 1),
                       "frac_of_peak": round(f_x / x_ms / 1e9 / peak_tf, 4),
                       "gbs": round(b_x / x_ms / 1e6, 1),
                       "frac_of_hbm": round(b_x / x_ms / 1e6 / peak_gbs, 4)}
    del q, k, v, o, ws
    torch.cuda.empty_cache()

    # the context-parallel step on one rank (its exchange kernels then copy
    # locally): the 480p clip, scatter (Q, K, V with the key RoPE) and gather
    from full_spatiotemporal_attention_b200.ulysses import UlyssesAttention
    w = si.WORKLOADS["c81f480"]
    q, k, v = (to_dev(x, device) for x in si.qkv(w))
    g = va.Grid.make(w.T, w.H, w.W, w.n_text, w.dims, w.theta)
    ua = UlyssesAttention(g, w.batch, w.heads, world=1, rank=0, device=device)
    _, u_ms = timed_loop(ev_pair(lambda: ua(q, k, v)), 5, 3, 1, device)
    _, s_ms = timed_loop(ev_pair(lambda: ua.scatter(q, k, v)), 20, 3, 1, device)
    _, g_ms = timed_loop(ev_pair(ua.gather), 20, 3, 1, device)
    torch.cuda.synchronize()
    ua.close()
    tb = w.batch * w.heads * w.N * HEAD_DIM * 2
    out["ulysses480_1rank"] = {
        "step_ms": round(u_ms, 4), "tflops": round(full_flops(w) / u_ms / 1e9, 1),
        "scatter_ms": round(s_ms, 4), "scatter_gbs": round(6 * tb / s_ms / 1e6, 1),
        "scatter_frac_hbm": round(6 * tb / s_ms / 1e6 / peak_gbs, 4),
        "gather_ms": round(g_ms, 4), "gather_gbs": round(2 * tb / g_ms / 1e6, 1),
        "gather_frac_hbm": round(2 * tb / g_ms / 1e6 / peak_gbs, 4)}
    # the ring step on one rank: key/query load with RoPE, one block product
    # (the cross-attention form, with LSE) and the fp32 merge
    from full_spatiotemporal_attention_b200.ring import RingAttention
    ra = RingAttention(g, w.batch, w.heads, world=1, rank=0, device=device)
    _, r_ms = timed_loop(ev_pair(lambda: ra(q, k, v)), 5, 3, 1, device)
    torch.cuda.synchronize()
    ra.close()
    out["ring480_1rank"] = {"step_ms": round(r_ms, 4),
                            "tflops": round(full_flops(w) / r_ms / 1e9, 1)}
    del q, k, v, ua, ra
    torch.cuda.empty_cache()
    return out


def bench_ulysses(args, rank, world, local):
    """One sequence of the workload split over the ranks (Ulysses context
    parallelism through peer memory): each rank holds a contiguous token
    slice of every head; a step scatters it, runs full attention on whole
    sequences of its heads and gathers its slice of the output."""
    import numpy as np
    import torch
    import full_spatiotemporal_attention_b200 as va
    from full_spatiotemporal_attention_b200.ulysses import UlyssesAttention
    import seeded_inputs as si

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = si.WORKLOADS[args.workload]
    g = va.Grid.make(w.T, w.H, w.W, w.n_text, w.dims, w.theta)
    if args.parallel == "ring":
        return bench_ring(args, rank, world, device, w, g)
    ua = UlyssesAttention(g, w.batch, w.heads, world=world, rank=rank, device=device)
    t0, t1 = ua.plan.token_range
    host = [np.ascontiguousarray(x[:, :, t0:t1]) for x in si.qkv(w)]
    q, k, v = (to_dev(x, device) for x in host)
    stream = torch.cuda.current_stream(device)

    def step(i):
        ua(q, k, v)

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.5)
    window = []
    step_ms, _ = timed_loop(step, args.steps, args.warmup, world, device, window=window)
    clocks = sampler.stop(*window)
    step_ms = max_over_ranks(step_ms, world, device)

    # the three steps alone (every rank runs the same sequence)
    def phase(fn):
        def run(i):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            return a, b
        return run
    n = max(args.steps // 2, 5)
    _, sc_ms = timed_loop(phase(lambda: ua.scatter(q, k, v)), n, 3, world, device)
    _, at_ms = timed_loop(phase(ua.attend), n, 3, world, device)
    _, ga_ms = timed_loop(phase(ua.gather), n, 3, world, device)
    sc_ms, at_ms, ga_ms = (max_over_ranks(x, world, device) for x in (sc_ms, at_ms, ga_ms))

    # end to end: this rank's slice from pinned host memory, its output slice back
    qh, kh, vh = (torch.from_numpy(x).view(torch.bfloat16).pin_memory() for x in host)
    oh = torch.empty(qh.shape, dtype=torch.bfloat16).pin_memory()
    qd, kd, vd = (torch.empty_like(q) for _ in range(3))

    def e2e_step(i):
        qd.copy_(qh, non_blocking=True)
        kd.copy_(kh, non_blocking=True)
        vd.copy_(vh, non_blocking=True)
        oh.copy_(ua(qd, kd, vd), non_blocking=True)
    e2e_ms, _ = timed_loop(e2e_step, args.e2e_steps, 3, world, device)
    e2e_ms = max_over_ranks(e2e_ms, world, device)
    torch.cuda.synchronize()
    assert va.device_error() == 0, "a peer wait gave up"
    ua.close(barrier=(lambda: barrier(world)))

    flops = full_flops(w)
    peak_tf, peak_gbs, peak_src = peaks()
    shard = w.batch * w.heads * (w.N // world) * HEAD_DIM * 2   # one tensor's slice per rank
    attn_flops_rank = flops / world
    cfg = job_config(w, world)
    cfg.update(global_batch=w.batch,
               parallelism=f"ulysses x{world} (token slices <-> head groups over peer memory)")
    return {
        "metric": METRIC,
        "value": round(flops / (step_ms / 1e3) / 1e12, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms, 4),
        "higher_is_better": True,
        "scaling": "strong",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded splitmix64 + Box-Muller bf16 N(0,1))",
        "config": cfg,
        "pct_of_peak": round(100.0 * flops / (step_ms / 1e3) / 1e12 / world / peak_tf, 2),
        "e2e": {"value": round(flops / (e2e_ms / 1e3) / 1e12, 2), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": 3 * shard,
                "d2h_bytes_per_step": shard},
        "gpu_launches": 6 * args.steps,
        "roofline": {"bound": "tensor", "achieved": round(attn_flops_rank / (at_ms / 1e3) / 1e12, 2),
                     "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": round(attn_flops_rank / (at_ms / 1e3) / 1e12 / peak_tf, 4),
                     "traffic": None, "kernel": "attn_fwd_kernel",
                     "peak_source": f"{peak_src} bf16 dense (burst)", "kernel_ms": round(at_ms, 4)},
        "exchange": {
            "scatter_ms": round(sc_ms, 4), "gather_ms": round(ga_ms, 4),
            # per rank: Q, K, V slices read and written; O slices read and written
            "scatter_gbs": round(6 * shard / (sc_ms / 1e3) / 1e9, 1),
            "gather_gbs": round(2 * shard / (ga_ms / 1e3) / 1e9, 1),
            "bytes_to_peers_per_step": int(4 * shard * (world - 1) / world),
            "peak_gbs_local": peak_gbs},
        "clocks": clocks,
    }


def bench_ring(args, rank, world, device, w, g):
    """Ring context parallelism: each rank keeps its query slice and sees
    every rank's K/V block in turn; the step's time is the slowest rank's."""
    import numpy as np
    import torch
    import full_spatiotemporal_attention_b200 as va
    from full_spatiotemporal_attention_b200.ring import RingAttention
    import seeded_inputs as si
    ra = RingAttention(g, w.batch, w.heads, world=world, rank=rank, device=device)
    nl = w.N // world
    host = [np.ascontiguousarray(x[:, :, rank * nl:(rank + 1) * nl]) for x in si.qkv(w)]
    q, k, v = (to_dev(x, device) for x in host)
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.5)
    window = []
    def step(i):
        ra(q, k, v)
    step_ms, _ = timed_loop(step, args.steps, args.warmup, world, device, window=window)
    clocks = sampler.stop(*window)
    step_ms = max_over_ranks(step_ms, world, device)
    qh, kh, vh = (torch.from_numpy(x).view(torch.bfloat16).pin_memory() for x in host)
    oh = torch.empty(qh.shape, dtype=torch.bfloat16).pin_memory()
    qd, kd, vd = (torch.empty_like(q) for _ in range(3))

    def e2e_step(i):
        qd.copy_(qh, non_blocking=True)
        kd.copy_(kh, non_blocking=True)
        vd.copy_(vh, non_blocking=True)
        oh.copy_(ra(qd, kd, vd), non_blocking=True)
    e2e_ms, _ = timed_loop(e2e_step, args.e2e_steps, 3, world, device)
    e2e_ms = max_over_ranks(e2e_ms, world, device)
    torch.cuda.synchronize()
    assert va.device_error() == 0, "a peer wait gave up"
    ra.close(barrier=(lambda: barrier(world)))
    flops = full_flops(w)
    peak_tf, _, peak_src = peaks()
    shard = w.batch * w.heads * nl * HEAD_DIM * 2
    cfg = job_config(w, world)
    cfg.update(global_batch=w.batch,
               parallelism=f"ring x{world} (K/V blocks passed around the ranks over peer memory)")
    value = flops / (step_ms / 1e3) / 1e12
    return {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 4),
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded splitmix64 + Box-Muller bf16 N(0,1))", "config": cfg,
        "pct_of_peak": round(100.0 * value / world / peak_tf, 2),
        "e2e": {"value": round(flops / (e2e_ms / 1e3) / 1e12, 2), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": 3 * shard,
                "d2h_bytes_per_step": shard},
        # load; per block: table + product, merge, and (P > 1) the free
        # signal; per pass: free wait, pass, full wait
        "gpu_launches": (1 + 3 * world + (world if world > 1 else 0) + 3 * (world - 1)) * args.steps,
        "roofline": {"bound": "tensor", "achieved": round(value / world, 2), "peak": peak_tf,
                     "unit": "TFLOP/s", "frac": round(value / world / peak_tf, 4), "traffic": None,
                     "kernel": "whole ring step (no separate kernel timing)",
                     "peak_source": f"{peak_src} bf16 dense (burst)"},
        "clocks": clocks,
    }


def run_case(args):
    """One secondary kernel alone on the 720p clip, for profiling: `--warmup`
    untimed and `--steps` timed launches.  The temporal pass takes raw keys
    (as the factorised call passes them); the others take pre-rotated keys."""
    import torch
    import full_spatiotemporal_attention_b200 as va
    import seeded_inputs as si
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    w = si.WORKLOADS["cross720" if args.case == "cross720" else "c81f720"]
    q, k, v = (to_dev(x, device) for x in si.qkv(w))
    o = torch.empty_like(q)
    if args.case == "cross720":
        ws = torch.empty(va.cross_workspace_bytes(w.batch, w.heads, w.N, w.n_kv), dtype=torch.uint8,
                         device=device)
        fn = lambda: va.attn_cross_fwd(q, k, v, out=o, workspace=ws)
    else:
        g = va.Grid.make(w.T, w.H, w.W, w.n_text, w.dims, w.theta)
        kr = va.rope3d_apply(k, g)
        ws = torch.empty(va.workspace_bytes(w.batch, w.heads, w.N, g,
                                            k_rotated=args.case != "temporal720"),
                         dtype=torch.uint8, device=device)
        if args.case == "temporal720":
            fn = lambda: va.attn_factorized_fwd(q, k, v, g, spatial=False, out_temporal=o,
                                                workspace=ws)
        elif args.case == "spatial720":
            fn = lambda: va.attn_factorized_fwd(q, kr, v, g, temporal=False, k_rotated=True,
                                                out_spatial=o, workspace=ws)
        else:
            fn = lambda: va.attn_window_fwd(q, kr, v, g, (3, 9, 16), k_rotated=True, out=o,
                                            workspace=ws)
    stream = torch.cuda.current_stream(device)

    def step(i):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        return a, b
    _, ms = timed_loop(step, args.steps, args.warmup, 1, device)
    return {"case": args.case, "workload": w.description, "ms": round(ms, 4),
            "device_error": va.device_error()}


def bench_reference(args, rank, world):
    """The oracle, as it stands, on the host cores: each step computes a
    bounded sample of query rows of the same workload."""
    import oracle
    import seeded_inputs as si
    w = si.WORKLOADS[args.workload]
    q, k, v = si.qkv(w)
    og = oracle.Grid(w.T, w.H, w.W, w.n_text, w.dims, w.theta)
    rows = si.sample_rows(w, 16)
    flops = w.batch * w.heads * rows.size * 4.0 * w.N * HEAD_DIM
    for _ in range(args.warmup):
        oracle.attention(q, k, v, og, rows=rows)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.attention(q, k, v, og, rows=rows)
    dt = (time.perf_counter() - t0) / args.steps
    value = flops / dt / 1e12
    sample = (f"{rows.size} seeded query rows x {w.batch * w.heads} heads of {w.name} per step "
              f"(N={w.N}), all keys rotated each step")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": job_config(w, world),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse_args()
    if args.warmup < 3:
        sys.exit("--warmup must be >= 3")
    if args.impl == "reference":
        # the oracle runs on rank 0 only; other ranks leave without work
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        if rank == 0:
            print(json.dumps(bench_reference(args, rank, world)), flush=True)
        return
    if args.case:
        print(json.dumps(run_case(args)), flush=True)
        return
    rank, world, local = init_dist("nccl")
    line = (bench_ours if args.parallel == "replicas" else bench_ulysses)(args, rank, world, local)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

#!/usr/bin/env python3
"""Benchmark of the bifocal-RoPE attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

One step = one prefill of a Qwen3-8B-shaped attention layer at L = 131072
(B=1, Hq=32, Hkv=8, D=128, w_pretrained=32768, w0=4096, theta=1e6, G=4):
the RoPE operand pass (jetlong_prefill_rotate) followed by the attention
kernel (jetlong_prefill_attend), with inputs resident in HBM.  The headline
``value`` is algorithmic prefill TFLOP/s = 4 * B * Hq * D * L(L+1)/2 / time
(also given as prompt tokens per second, ``tokens_per_s``).
After the prefill steps, 256 decode steps on a 131072-token true-position
cache (Qwen3-8B shapes) are timed the same way and reported as microseconds
per token and achieved HBM bandwidth over the K+V bytes a step must read.
Both are also timed as a matched control -- the same kernels with the
bifocal rule off (w_pretrained = L, so G = 1: plain causal RoPE attention at
true positions) -- and the ratio is reported as the routing cost.  The
prefill is also timed in its unfused three-pass form (jetlong_prefill_three_pass)
to report what fusion saves, and prefill and decode are timed once more with
the frequency-interpolation remote map of the paper's remote-map ablation
(jetlong_prefill_interp, jetlong_decode_interp).

Every input is synthetic and seeded (zero_shot_rope_bifocal_b200.synth);
each is larger than the 126 MB L2 (q alone is 1 GiB), so no flush is needed
between steps.  Under torchrun each rank runs its own independent layer
(different seed): weak scaling, no collective in the data path; rank 0 prints
the JSON line with the max-over-ranks time and the summed work.

``--impl reference`` times the fp64 CPU oracle on the host's cores instead,
on a bounded sample of query rows of the same workload, in the same unit.
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "bifocal-attn prefill TFLOP/s (% BF16 peak) @128K; decode µs/token (% HBM BW)"
PREFILL_WORKLOAD = "qwen3_8b_128k"
DECODE_WORKLOAD = "decode_8b_128k"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# DRAM bytes (read + write) of one attention-kernel launch at the headline
# workload, from an ncu capture (dram__bytes_read.sum + dram__bytes_write.sum)
# of the kernel's own sources (its device code and the PTX wrappers it uses),
# whose code lines' SHA-256 is recorded here; the capture and its command are summarised
# in the profile named below.  The line reports it only while those sources
# are unchanged, and null otherwise.
TRAFFIC_RECORD = {"bytes": 6.09e9, "read_bytes": 4.96e9, "write_bytes": 1.13e9,
                  "sources_sha256": "d9af5b67481394ad8719dc287076d6144d1107ee97e1a41247bd3ce3c857b105",
                  "profile": "profiles/prefill_attention_qwen3_8b_L131072_dram.md"}
TRAFFIC_SOURCES = ("zero_shot_rope_bifocal_b200/csrc/prefill_sm100.cu",
                   "zero_shot_rope_bifocal_b200/csrc/sm100_ptx.cuh")
NOMINAL = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}


# ---------------------------------------------------------------- accounting
def prefill_flops(B: int, Hq: int, L: int, D: int) -> int:
    """Algorithmic FLOPs: every causal pair gets one Q.K dot (2D) and one P.V axpy (2D)."""
    return 4 * B * Hq * D * (L * (L + 1) // 2)


def prefill_operand_bytes(B: int, Hq: int, Hkv: int, L: int, D: int) -> int:
    """Bytes the attention kernel must move at least: q read once (BF16; the
    kernel rotates it as it loads it), the FP16 key operands read once (k at
    true and remote positions, v) and the BF16 output written once."""
    return B * L * Hq * D * 2 + 3 * B * Hkv * L * D * 2 + B * L * Hq * D * 2


def row_flops(Hq: int, D: int, rows) -> int:
    return sum(4 * Hq * D * (int(i) + 1) for i in rows)


def decode_bytes(B: int, Hkv: int, L: int, D: int) -> int:
    """K and V BF16 bytes one decode step must stream."""
    return 2 * B * L * Hkv * D * 2


def kernel_sources_sha256() -> str:
    """SHA-256 of the kernel sources' code lines (comment-only lines and
    blank lines left out, so that a comment edit keeps the record)."""
    import hashlib
    h = hashlib.sha256()
    for rel in TRAFFIC_SOURCES:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as fh:
            for line in fh:
                t = line.strip()
                if t and not t.startswith("//"):
                    h.update(t.encode() + b"\n")
    return h.hexdigest()


def measured_traffic():
    """(bytes, source) of the recorded capture if it is of the current kernel, else (None, why)."""
    if TRAFFIC_RECORD is None:
        return None, "no capture recorded"
    if TRAFFIC_RECORD["sources_sha256"] != kernel_sources_sha256():
        return None, "kernel changed since the recorded capture"
    return TRAFFIC_RECORD["bytes"], TRAFFIC_RECORD["profile"]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- ranks
def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), \
        int(os.environ.get("LOCAL_RANK", "0"))


def reduce_max(x: float, world: int, device=None) -> float:
    """Max over ranks (host plumbing for the timing report)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(x: float, world: int, device=None) -> float:
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi (every 25 ms, so
    that the ~0.7 s prefill region gets about 25 samples).

    The sampler starts on entry and waits for its first sample, so that the
    timed region that follows is covered; ``window(t0, t1)`` (times from
    ``now()``) restricts the summary to the samples taken inside it.
    """

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_S = 0.025

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []  # (arrival time, csv line)
        self.thread = None
        self.t0 = None
        self.t1 = None

    @staticmethod
    def now() -> float:
        return time.monotonic()

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", str(int(self.PERIOD_S * 1000))],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            deadline = time.monotonic() + 5.0
            while not self.lines and time.monotonic() < deadline and self.proc.poll() is None:
                time.sleep(0.02)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def window(self, t0: float, t1: float) -> None:
        self.t0, self.t1 = t0, t1

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            if self.thread is not None:
                self.thread.join(timeout=2)

    def summary(self):
        lines = self.lines
        if self.t0 is not None:
            # a sample reports the state when it was taken, shortly before it
            # arrives: keep those that arrived inside the window or within one
            # period after it
            lines = [(t, ln) for t, ln in lines if self.t0 <= t <= self.t1 + self.PERIOD_S]
        if not lines:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for _, ln in lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- oracle timing
def oracle_rows_per_sec(w, seconds: float, q_rows_src, k, v, rows):
    """Time the CPU oracle on query rows of workload ``w`` for about ``seconds``.

    Returns (flops_done, elapsed, rows_done)."""
    import oracle
    import torch
    done_rows, flops, t0 = [], 0, time.perf_counter()
    for i, r in enumerate(rows):
        q1 = q_rows_src[:, i:i + 1]
        oracle.prefill_rows(q1, k, v, w.w_pretrained, w.w0, w.theta, [r], q_holds_rows=True)
        done_rows.append(r)
        flops += row_flops(w.Hq, w.D, [r])
        if time.perf_counter() - t0 >= seconds:
            break
    return flops, time.perf_counter() - t0, done_rows


def oracle_rate_extras(w, flops: float, seconds: float, rows_done) -> dict:
    """Rows per second of the timed oracle sample, and the time the whole
    prefill of ``w`` would take at the sample's FLOP rate (an extrapolation:
    row costs grow with the row index, so the rate, not the row count, is
    scaled)."""
    rate = flops / seconds
    return {"rows_per_s": len(rows_done) / seconds,
            "extrapolated_full_prefill_s": prefill_flops(w.B, w.Hq, w.L, w.D) / rate}


def cpu_sample_inputs(w, n_rows: int, device):
    """Inputs of ``w`` for oracle timing: the query rows to time and K/V as fp32 numpy."""
    import torch
    from zero_shot_rope_bifocal_b200.synth import prefill_inputs
    x = prefill_inputs(w, device=device)
    g = torch.Generator().manual_seed(1234)
    rows = sorted(torch.randint(w.L // 2, w.L, (n_rows,), generator=g).tolist())
    ridx = torch.tensor(rows, device=x.q.device)
    q_rows = x.q.index_select(1, ridx).to("cpu", torch.float32).numpy()
    k = x.k.to("cpu", torch.float32).numpy()
    v = x.v.to("cpu", torch.float32).numpy()
    del x
    return q_rows, k, v, rows


def threads_used() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


# ---------------------------------------------------------------- reference arm
def workload_config(w, world: int) -> dict:
    """The ``config`` both arms report for the headline prefill workload."""
    return {"workload": PREFILL_WORKLOAD, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D, "L": w.L,
            "w_pretrained": w.w_pretrained, "w0": w.w0, "rope_theta": w.theta,
            "G": -(-w.L // w.w_pretrained) if w.L > w.w_pretrained else 1,
            "l2": "inputs larger than L2 (q 1 GiB, k/v 256 MiB each); no flush",
            "parallelism": f"independent layer per rank x{world}"}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from zero_shot_rope_bifocal_b200.synth import WORKLOADS
    w = WORKLOADS[PREFILL_WORKLOAD]
    q_rows, k, v, rows = cpu_sample_inputs(w, 64, "cpu")
    per_step = max(2.0, args.reference_seconds / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_rows_per_sec(w, per_step, q_rows, k, v, rows)
    tot_f, tot_t, all_done = 0, 0.0, []
    for s in range(args.steps):
        rot = rows[s % len(rows):] + rows[:s % len(rows)]
        qrot = q_rows[:, [rows.index(r) for r in rot]]
        f, t, done = oracle_rows_per_sec(w, per_step, qrot, k, v, rot)
        tot_f, tot_t, all_done = tot_f + f, tot_t + t, all_done + done
    nrows = len(all_done)
    value = tot_f / tot_t / 1e12
    line = {
        "impl": "reference", "metric": METRIC,
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) Q/K/V, K per-channel LogNormal(0,0.5) scale)",
        "config": workload_config(w, world),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads_used(),
                         "kind": "oracle",
                         "sample": f"{nrows} query rows (all 32 heads) of the 128K prefill, "
                                   f"random rows in [L/2, L), ~{per_step:.0f} s per step",
                         **oracle_rate_extras(w, tot_f, tot_t, all_done)},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- native arm
# ---------------------------------------------------------------- per-config sweep
L2_BYTES = 126 * 2 ** 20


def sweep_prefill(jl, torch, dev, stream, name: str, w0: int | None = None, reps: int = 5) -> dict:
    """One named prefill workload (the RoPE operand pass plus the attention
    kernel): median per-step and per-kernel times over ``reps`` steps, each
    preceded by an L2 flush outside the timed events.  Warm-up steps run back
    to back first, so that the clocks have left their idle state (the first
    millisecond after an idle gap runs measurably slower)."""
    from zero_shot_rope_bifocal_b200.synth import WORKLOADS, prefill_inputs
    w = WORKLOADS[name] if w0 is None else WORKLOADS[name].with_(w0=w0)
    x = prefill_inputs(w, device=dev)
    B, L, Hq, Hkv, D = w.B, w.L, w.Hq, w.Hkv, w.D
    out = torch.empty((B, L, Hq, D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, Hq, L), dtype=torch.float32, device=dev)
    ws = torch.empty(jl.jetlong_prefill_workspace_size(B, Hq, Hkv, L, D), dtype=torch.uint8,
                     device=dev)
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)

    def rotate():
        jl.jetlong_prefill_rotate(x.k, x.v, w.w_pretrained, w.theta, ws, stream=stream)

    def attend():
        jl.jetlong_prefill_attend(x.q, out, lse, Hkv, w.w_pretrained, w.w0, w.theta, ws,
                                  stream=stream)

    n_warm = max(3, int(20.0 / max(prefill_flops(B, Hq, L, D) / 1e12, 1.0)))  # ~20 ms of work
    for _ in range(min(n_warm, 50)):
        rotate()
        attend()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    step_ms, attn_ms = [], []
    for _ in range(reps):
        flush.zero_()
        ev[0].record(stream)
        rotate()
        ev[1].record(stream)
        attend()
        ev[2].record(stream)
        torch.cuda.synchronize(dev)
        step_ms.append(ev[0].elapsed_time(ev[2]))
        attn_ms.append(ev[1].elapsed_time(ev[2]))
    if jl.jetlong_device_status() != jl.JL_OK:
        raise RuntimeError(f"device status not OK after the {name} prefill")
    flops = prefill_flops(B, Hq, L, D)
    t_step, t_attn = statistics.median(step_ms), statistics.median(attn_ms)
    return {"workload": name, "Hq": Hq, "Hkv": Hkv, "L": L, "w_pretrained": w.w_pretrained,
            "w0": w.w0, "G": -(-L // w.w_pretrained) if L > w.w_pretrained else 1,
            "step_ms": t_step, "attend_ms": t_attn, "tflops": flops / (t_step * 1e-3) / 1e12,
            "attend_tflops": flops / (t_attn * 1e-3) / 1e12,
            "tokens_per_s": B * L / (t_step * 1e-3), "steps": reps,
            "l2": "flushed before every timed step"}


def sweep_decode(jl, torch, dev, stream, name: str, n_cache: int, n_loop: int = 256,
                 reps: int = 8) -> dict:
    """Decode steps on ``n_cache`` distinct true-position caches used in
    turn (so that, together larger than L2, no step is served from L2),
    captured once as a CUDA graph of ``n_loop`` steps and replayed."""
    from zero_shot_rope_bifocal_b200.synth import WORKLOADS, decode_inputs
    w = WORKLOADS[name]
    caches = []
    for c in range(n_cache):
        d = decode_inputs(w.with_(seed=w.seed + 1000 * c), device=dev)
        kc = torch.empty_like(d.k_raw)
        jl.jetlong_rope_cache(d.k_raw, kc, 0, w.theta, stream=stream)
        caches.append((d.q, kc, d.v))
        del d
    out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev)
    ws = torch.empty(jl.jetlong_decode_workspace_size(w.B, w.Hq, w.Hkv, w.L, w.D),
                     dtype=torch.uint8, device=dev)

    def dstep(i, st):
        q, kc, v = caches[i % n_cache]
        jl.jetlong_decode(q, kc, v, w.L, w.w_pretrained, w.w0, w.theta, out=out, lse=lse,
                          workspace=ws, stream=st)

    for i in range(3 * n_cache):
        dstep(i, stream)
    torch.cuda.synchronize(dev)
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        for i in range(n_loop):
            dstep(i, cap)
    g.replay()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    del g
    if jl.jetlong_device_status() != jl.JL_OK:
        raise RuntimeError(f"device status not OK after the {name} decode")
    us = 1e3 * e0.elapsed_time(e1) / (n_loop * reps)
    nbytes = decode_bytes(w.B, w.Hkv, w.L, w.D)
    return {"workload": name, "L": w.L, "G": -(-w.L // w.w_pretrained) if w.L > w.w_pretrained
            else 1, "us_per_token": us, "tokens_per_s": w.B * 1e6 / us,
            "achieved_gbs": nbytes / (us * 1e-6) / 1e9, "bytes_per_token": nbytes,
            "steps": n_loop * reps, "caches": n_cache,
            "l2": f"{n_cache} distinct caches of {nbytes / 2 ** 20:.0f} MiB used in turn"}


def run_native(args):
    import torch
    import torch.distributed as dist
    from zero_shot_rope_bifocal_b200 import jetlong as jl
    from zero_shot_rope_bifocal_b200.synth import WORKLOADS, decode_inputs, prefill_inputs

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
    jl.lib()  # fail loudly if the library is missing

    def barrier():
        if world > 1:
            dist.barrier()

    w = WORKLOADS[PREFILL_WORKLOAD].with_(seed=WORKLOADS[PREFILL_WORKLOAD].seed + 100 * rank)
    x = prefill_inputs(w, device=dev)
    B, L, Hq, Hkv, D = w.B, w.L, w.Hq, w.Hkv, w.D
    out = torch.empty((B, L, Hq, D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, Hq, L), dtype=torch.float32, device=dev)
    ws = torch.empty(jl.jetlong_prefill_workspace_size(B, Hq, Hkv, L, D), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev_mid=None, ev_end=None):
        jl.jetlong_prefill_rotate(x.k, x.v, w.w_pretrained, w.theta, ws, stream=stream)
        if ev_mid is not None:
            ev_mid.record(stream)
        jl.jetlong_prefill_attend(x.q, out, lse, Hkv, w.w_pretrained, w.w0, w.theta, ws,
                                  stream=stream)
        if ev_end is not None:
            ev_end.record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if jl.jetlong_device_status() != jl.JL_OK:
        raise RuntimeError("device status not OK after warm-up")

    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    mids = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    with ClockSampler(local) as clocks:
        barrier()
        torch.cuda.synchronize(dev)
        tw0 = clocks.now()
        ev0.record(stream)
        for s in range(args.steps):
            step(mids[s], ends[s])
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        clocks.window(tw0, clocks.now())
        barrier()
    t_ms = ev0.elapsed_time(ev1)
    attn_ms = sum(mids[s].elapsed_time(ends[s]) for s in range(args.steps)) / args.steps
    rot_ms = (t_ms - attn_ms * args.steps) / args.steps
    if jl.jetlong_device_status() != jl.JL_OK:
        raise RuntimeError("device status not OK after timing")
    t_max = reduce_max(t_ms, world, dev)

    # ---- matched control: the same kernels with the bifocal rule off
    # (w_pretrained = L, so G = 1: plain causal RoPE at true positions), on the
    # same inputs; it prices the routing (remote visits, edge tiles, rotation).
    def ctl_step(ev_mid=None, ev_end=None):
        jl.jetlong_prefill_rotate(x.k, x.v, L, w.theta, ws, stream=stream)
        if ev_mid is not None:
            ev_mid.record(stream)
        jl.jetlong_prefill_attend(x.q, out, lse, Hkv, L, w.w0, w.theta, ws, stream=stream)
        if ev_end is not None:
            ev_end.record(stream)

    ctl_step()
    n_ctl = max(1, min(args.steps, 3))
    barrier()
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    for s in range(n_ctl):
        ctl_step(mids[s], ends[s])
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    ctl_step_ms = reduce_max(ev0.elapsed_time(ev1), world, dev) / n_ctl
    ctl_attn_ms = sum(mids[s].elapsed_time(ends[s]) for s in range(n_ctl)) / n_ctl
    if jl.jetlong_device_status() != jl.JL_OK:
        raise RuntimeError("device status not OK after the control prefill")

    # ---- the unfused three-pass form (A + B - C merge) on the same inputs:
    # what fusing the passes into one kernel saves
    ws3 = torch.empty(jl.jetlong_prefill_three_pass_workspace_size(B, Hq, Hkv, L, D),
                      dtype=torch.uint8, device=dev)

    def three_step():
        jl.jetlong_prefill_three_pass(x.q, x.k, x.v, w.w_pretrained, w.w0, w.theta, out=out,
                                      lse=lse, workspace=ws3, stream=stream)

    three_step()
    barrier()
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    for _ in range(n_ctl):
        three_step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    three_ms = reduce_max(ev0.elapsed_time(ev1), world, dev) / n_ctl
    del ws3
    if jl.jetlong_device_status() != jl.JL_OK:
        raise RuntimeError("device status not OK after the three-pass prefill")
    # ---- the frequency-interpolation remote map (the remote-map ablation):
    # the same attention kernel on operands rotated with interpolated
    # frequencies at true positions
    def interp_step():
        jl.jetlong_prefill_interp(x.q, x.k, x.v, w.w_pretrained, w.w0, w.theta, out=out, lse=lse,
                                  workspace=ws, stream=stream)

    interp_step()
    barrier()
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    for _ in range(n_ctl):
        interp_step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    interp_ms = reduce_max(ev0.elapsed_time(ev1), world, dev) / n_ctl
    if jl.jetlong_device_status() != jl.JL_OK:
        raise RuntimeError("device status not OK after the interpolation prefill")
    flops_rank = prefill_flops(B, Hq, L, D) * args.steps
    flops_all = reduce_sum(flops_rank, world, dev)
    value = flops_all / (t_max * 1e-3) / 1e12

    # ---- decode: 256 steps on a 128K true-position cache
    wd = WORKLOADS[DECODE_WORKLOAD].with_(seed=WORKLOADS[DECODE_WORKLOAD].seed + 100 * rank)
    d = decode_inputs(wd, device=dev)
    kc = torch.empty_like(d.k_raw)
    jl.jetlong_rope_cache(d.k_raw, kc, 0, wd.theta, stream=stream)
    del d.k_raw
    dq = d.q
    dout = torch.empty((wd.B, wd.Hq, wd.D), dtype=torch.bfloat16, device=dev)
    dlse = torch.empty((wd.B, wd.Hq), dtype=torch.float32, device=dev)
    dws = torch.empty(jl.jetlong_decode_workspace_size(wd.B, wd.Hq, wd.Hkv, wd.L, wd.D),
                      dtype=torch.uint8, device=dev)

    def dstep(st=None):
        jl.jetlong_decode(dq, kc, d.v, wd.L, wd.w_pretrained, wd.w0, wd.theta, out=dout, lse=dlse,
                          workspace=dws, stream=stream if st is None else st)

    for _ in range(max(3, args.warmup)):
        dstep()
    # 256-step loops, repeated so that the timed region lasts long enough for
    # the clock sampler; the mean over all steps is reported.  The loop is
    # captured once in a CUDA graph (as a serving loop would run it, with no
    # per-step host launch cost) and replayed; if capture fails, the steps
    # are launched from the host and the line says so.
    n_loop = args.decode_steps
    n_rep = max(1, args.decode_reps)
    n_dec = n_loop * n_rep
    torch.cuda.synchronize(dev)
    graph, dec_loop = None, f"{n_rep} x {n_loop} steps, CUDA graph replays"
    try:
        cap = torch.cuda.Stream(dev)
        cap.wait_stream(stream)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            for _ in range(n_loop):
                dstep(cap)
        graph = g
        graph.replay()
    except Exception as e:  # noqa: BLE001 - report and fall back to host launches
        graph, dec_loop = None, f"{n_rep} x {n_loop} steps, host launches (graph: {type(e).__name__})"
    torch.cuda.synchronize(dev)
    if jl.jetlong_device_status() != jl.JL_OK:
        raise RuntimeError("device status not OK after the decode warm-up")
    with ClockSampler(local) as dclocks:
        barrier()
        torch.cuda.synchronize(dev)
        tw0 = dclocks.now()
        ev0.record(stream)
        if graph is not None:
            for _ in range(n_rep):
                graph.replay()
        else:
            for _ in range(n_dec):
                dstep()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        dclocks.window(tw0, dclocks.now())
        barrier()
    dec_ms = reduce_max(ev0.elapsed_time(ev1), world, dev)
    if jl.jetlong_device_status() != jl.JL_OK:
        raise RuntimeError("device status not OK after decode timing")
    # the same steps launched one by one from Python, for comparison
    barrier()
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    for _ in range(n_loop):
        dstep()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    host_loop_us = 1e3 * reduce_max(ev0.elapsed_time(ev1), world, dev) / n_loop
    del graph
    us_tok = 1e3 * dec_ms / n_dec
    dec_gbs = decode_bytes(wd.B, wd.Hkv, wd.L, wd.D) / (us_tok * 1e-6) / 1e9

    # matched control decode (G = 1: every key local, no correction rotation)
    def dstep_ctl():
        jl.jetlong_decode(dq, kc, d.v, wd.L, wd.L, wd.w0, wd.theta, out=dout, lse=dlse,
                          workspace=dws, stream=stream)

    for _ in range(3):
        dstep_ctl()
    barrier()
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    for _ in range(n_loop):
        dstep_ctl()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    ctl_us_tok = 1e3 * reduce_max(ev0.elapsed_time(ev1), world, dev) / n_loop
    if jl.jetlong_device_status() != jl.JL_OK:
        raise RuntimeError("device status not OK after the control decode")

    # the frequency-interpolation decode, host launches like host_loop_us
    def dstep_interp():
        jl.jetlong_decode_interp(dq, kc, d.v, wd.L, wd.w_pretrained, wd.w0, wd.theta, out=dout,
                                 lse=dlse, workspace=dws, stream=stream)

    for _ in range(3):
        dstep_interp()
    barrier()
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    for _ in range(n_loop):
        dstep_interp()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    interp_us_tok = 1e3 * reduce_max(ev0.elapsed_time(ev1), world, dev) / n_loop
    if jl.jetlong_device_status() != jl.JL_OK:
        raise RuntimeError("device status not OK after the interpolation decode")

    # the two-form key cache: the remote form of every key written once for
    # this G (timed), then decode steps that read remote keys from it
    kr = torch.empty(kc.shape, dtype=torch.float16, device=dev)
    jl.jetlong_remote_cache(kc, kr, 0, wd.L, wd.L, wd.w_pretrained, wd.theta, stream=stream)
    barrier()
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    jl.jetlong_remote_cache(kc, kr, 0, wd.L, wd.L, wd.w_pretrained, wd.theta, stream=stream)
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    rebuild_ms = reduce_max(ev0.elapsed_time(ev1), world, dev)

    def dstep_two(st=None):
        jl.jetlong_decode_two_form(dq, kc, kr, d.v, wd.L, wd.w_pretrained, wd.w0, wd.theta,
                                   out=dout, lse=dlse, workspace=dws,
                                   stream=stream if st is None else st)

    for _ in range(3):
        dstep_two()
    torch.cuda.synchronize(dev)
    cap2 = torch.cuda.Stream(dev)
    cap2.wait_stream(stream)
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g2, stream=cap2):
        for _ in range(n_loop):
            dstep_two(cap2)
    g2.replay()
    n_rep2 = 8
    barrier()
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    for _ in range(n_rep2):
        g2.replay()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    del g2
    two_us_tok = 1e3 * reduce_max(ev0.elapsed_time(ev1), world, dev) / (n_loop * n_rep2)
    del kr
    if jl.jetlong_device_status() != jl.JL_OK:
        raise RuntimeError("device status not OK after the two-form decode")

    # prefill chunks of 4 to 4096 tokens closing the same 128K cache (below
    # CHUNK_TENSOR_MIN tokens the decode kernels run them, from there on the
    # prefill kernel, its keys split across CTAs while the query tiles are few)
    chunks = []
    for n_chunk in (4, 16, 64, 1024, 4096):
        P0 = wd.L - n_chunk
        cq = torch.randn((wd.B, n_chunk, wd.Hq, wd.D), device=dev).to(torch.bfloat16)
        cout = torch.empty((wd.B, n_chunk, wd.Hq, wd.D), dtype=torch.bfloat16, device=dev)
        clse = torch.empty((wd.B, wd.Hq, n_chunk), dtype=torch.float32, device=dev)
        cws = torch.empty(jl.jetlong_prefill_chunk_workspace_size(wd.B, wd.Hq, wd.Hkv, P0,
                                                                  n_chunk, wd.D),
                          dtype=torch.uint8, device=dev)

        def cstep():
            jl.jetlong_prefill_chunk(cq, kc, d.v, P0, wd.w_pretrained, wd.w0, wd.theta,
                                     out=cout, lse=clse, workspace=cws, stream=stream)

        for _ in range(3):
            cstep()
        n_crep = 10
        barrier()
        torch.cuda.synchronize(dev)
        ev0.record(stream)
        for _ in range(n_crep):
            cstep()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        chunk_ms = reduce_max(ev0.elapsed_time(ev1), world, dev) / n_crep
        if jl.jetlong_device_status() != jl.JL_OK:
            raise RuntimeError("device status not OK after the prefill chunk")
        pairs = n_chunk * P0 + n_chunk * (n_chunk + 1) // 2  # causal (query, key) pairs
        chunks.append({"n": n_chunk, "P0": P0, "ms": chunk_ms,
                       "us_per_query": 1e3 * chunk_ms / n_chunk,
                       "path": "decode kernels" if n_chunk < jl.CHUNK_TENSOR_MIN else "prefill kernel",
                       "tflops": 4 * wd.B * wd.Hq * wd.D * pairs / (chunk_ms * 1e-3) / 1e12})
        del cq, cout, clse, cws

    # ---- end to end through the public API from pinned host buffers
    hq = x.q.cpu().pin_memory()
    hk = x.k.cpu().pin_memory()
    hv = x.v.cpu().pin_memory()
    # Double-buffered device inputs and outputs: step i's upload (one copy
    # stream) overlaps step i-1's compute, and its download (another copy
    # stream) overlaps step i+1's compute, as a caller streaming many layers
    # or prompts would run it.  Every step still copies its own inputs in
    # and its own result out inside the timed region.
    dbuf = [(torch.empty_like(x.q), torch.empty_like(x.k), torch.empty_like(x.v)) for _ in range(2)]
    obuf = [(torch.empty_like(out), torch.empty_like(lse)) for _ in range(2)]
    hbuf = [(torch.empty(out.shape, dtype=out.dtype).pin_memory(),
             torch.empty(lse.shape, dtype=lse.dtype).pin_memory()) for _ in range(2)]
    del x
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_up = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_down = [torch.cuda.Event() for _ in range(2)]

    def e2e_run(n_steps):
        up.wait_stream(stream)
        for i in range(n_steps):
            b2 = i % 2
            dq2, dk2, dv2 = dbuf[b2]
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(ev_comp[b2])  # step i-2's compute is done with this buffer
                dq2.copy_(hq, non_blocking=True)
                dk2.copy_(hk, non_blocking=True)
                dv2.copy_(hv, non_blocking=True)
                ev_up[b2].record(up)
            stream.wait_event(ev_up[b2])
            if i >= 2:
                stream.wait_event(ev_down[b2])  # step i-2's download has left this buffer
            jl.jetlong_prefill(dq2, dk2, dv2, w.w_pretrained, w.w0, w.theta, out=obuf[b2][0],
                               lse=obuf[b2][1], workspace=ws, stream=stream)
            ev_comp[b2].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(ev_comp[b2])
                hbuf[b2][0].copy_(obuf[b2][0], non_blocking=True)
                hbuf[b2][1].copy_(obuf[b2][1], non_blocking=True)
                ev_down[b2].record(down)
        stream.wait_stream(up)
        stream.wait_stream(down)

    e2e_run(2)
    n_e2e = max(2, args.steps)
    barrier()
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    e2e_run(n_e2e)
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = reduce_max(ev0.elapsed_time(ev1), world, dev) / n_e2e
    # latency of one call from host buffers, nothing overlapped: upload,
    # prefill, download, in order on one stream
    ev_l0 = torch.cuda.Event(enable_timing=True)
    ev_l1 = torch.cuda.Event(enable_timing=True)
    lat = []
    for _ in range(2):
        barrier()
        torch.cuda.synchronize(dev)
        ev_l0.record(stream)
        dq2, dk2, dv2 = dbuf[0]
        dq2.copy_(hq, non_blocking=True)
        dk2.copy_(hk, non_blocking=True)
        dv2.copy_(hv, non_blocking=True)
        jl.jetlong_prefill(dq2, dk2, dv2, w.w_pretrained, w.w0, w.theta, out=obuf[0][0],
                           lse=obuf[0][1], workspace=ws, stream=stream)
        hbuf[0][0].copy_(obuf[0][0], non_blocking=True)
        hbuf[0][1].copy_(obuf[0][1], non_blocking=True)
        ev_l1.record(stream)
        torch.cuda.synchronize(dev)
        lat.append(reduce_max(ev_l0.elapsed_time(ev_l1), world, dev))
    e2e_latency_ms = min(lat)
    e2e_val = reduce_sum(prefill_flops(B, Hq, L, D), world, dev) / (e2e_ms * 1e-3) / 1e12
    h2d = (hq.numel() + hk.numel() + hv.numel()) * 2
    d2h = hbuf[0][0].numel() * 2 + hbuf[0][1].numel() * 4

    # ---- every workload of the benchmark plan: prefill at 16K / 64K (with the
    # w0 sweep) and 128K, decode at 32K / 64K / 128K
    sweep = {"prefill": [], "decode": []}
    if not args.no_sweep:
        for name, w0s in (("qwen3_1p7b_16k", [None]), ("qwen3_1p7b_64k", [None]),
                          ("qwen3_8b_64k", [2048, 4096, 8192]), ("qwen3_8b_128k", [None])):
            for w0 in w0s:
                sweep["prefill"].append(sweep_prefill(jl, torch, dev, stream, name, w0))
        for name, n_cache in (("decode_8b_32k", 3), ("decode_8b_64k", 2), ("decode_8b_128k", 1)):
            sweep["decode"].append(sweep_decode(jl, torch, dev, stream, name, n_cache))

    # ---- CPU oracle baseline (rank 0, N=1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        q_rows, kk, vv, rows = cpu_sample_inputs(w, 64, dev)
        f, t, done = oracle_rows_per_sec(w, args.cpu_seconds, q_rows, kk, vv, rows)
        cpu = {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": threads_used(), "kind": "oracle",
               "sample": f"{len(done)} query rows (all 32 heads) of the 128K prefill, random rows "
                         f"in [L/2, L), {t:.1f} s of fp64 NumPy",
               **oracle_rate_extras(w, f, t, done)}

    if rank == 0:
        peaks, src = load_peaks()
        traffic, traffic_src = measured_traffic()
        attn_tflops = prefill_flops(B, Hq, L, D) / (attn_ms * 1e-3) / 1e12
        peak = peaks["bf16_tflops_sustained"]
        line = {
            "metric": METRIC,
            "value": value, "unit": "TFLOP/s",
            "tokens_per_s": value * 1e12 / prefill_flops(B, Hq, L, D) * B * L,
            "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16",
            "precision": "BF16 inputs and outputs; FP16 tensor-core operands (rotated Q/K, V, "
                         "P) with FP32 accumulation; FP32 softmax statistics",
            "data": "synthetic (seeded N(0,1) Q/K/V, K per-channel LogNormal(0,0.5) scale)",
            "config": workload_config(w, world),
            "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": peak,
                         "unit": "TFLOP/s", "frac": attn_tflops / peak,
                         "peak_source": f"{src} bf16_tflops_sustained",
                         "nominal_frac": attn_tflops / NOMINAL["bf16_tflops"],
                         "kernel": "bifocal_prefill_kernel<128>", "kernel_ms": attn_ms,
                         "traffic": traffic, "traffic_source": traffic_src,
                         "algorithmic_bytes": prefill_operand_bytes(B, Hq, Hkv, L, D)},
            "breakdown_ms": {"rotate": rot_ms, "attend": attn_ms},
            "decode": {"workload": DECODE_WORKLOAD, "us_per_token": us_tok,
                       "tokens_per_s": wd.B * 1e6 / us_tok, "steps": n_dec,
                       "loop": dec_loop, "host_loop_us_per_token": host_loop_us,
                       "achieved_gbs": dec_gbs, "peak_gbs": peaks["hbm_gbs"],
                       "frac": dec_gbs / peaks["hbm_gbs"],
                       "nominal_frac": dec_gbs / NOMINAL["hbm_gbs"],
                       "bytes_per_token": decode_bytes(wd.B, wd.Hkv, wd.L, wd.D),
                       "clocks": dclocks.summary()},
            "control": {
                "what": "same kernels, bifocal rule off (w_pretrained = L, G = 1): plain causal "
                        "RoPE attention at true positions, same inputs",
                "prefill_attend_ms": ctl_attn_ms,
                "prefill_attend_tflops": prefill_flops(B, Hq, L, D) / (ctl_attn_ms * 1e-3) / 1e12,
                "prefill_step_ms": ctl_step_ms,
                "routing_cost_prefill": attn_ms / ctl_attn_ms - 1.0,
                "decode_us_per_token": ctl_us_tok,
                "routing_cost_decode": us_tok / ctl_us_tok - 1.0},
            "prefill_chunk": {
                "what": "chunks of n queries at positions L-n..L-1 closing the 128K cache "
                        "(jetlong_prefill_chunk, one G from L); tflops counts 4.Hq.D per causal "
                        "(query, key) pair",
                "chunks": chunks},
            "three_pass": {
                "what": "unfused inclusion-exclusion form: rotate + passes A (remote, causal), "
                        "B (true, band), C (remote, band) + merge kernel, same inputs",
                "ms_per_step": three_ms,
                "tflops": prefill_flops(B, Hq, L, D) / (three_ms * 1e-3) / 1e12,
                "fused_speedup": three_ms / (t_max / args.steps)},
            "freq_interp": {
                "what": "remote-map ablation: remote pairs at true positions with YaRN-style "
                        "interpolated frequencies (ramp 1..32 turns, s = L / w_pretrained), "
                        "same inputs; prefill = rotate + attend, decode host-launched",
                "prefill_step_ms": interp_ms,
                "prefill_tflops": prefill_flops(B, Hq, L, D) / (interp_ms * 1e-3) / 1e12,
                "decode_us_per_token": interp_us_tok,
                "vs_alias_prefill_step": interp_ms / (t_max / args.steps),
                "vs_alias_decode_host_launched": interp_us_tok / host_loop_us},
            "configs": {
                "what": "each workload of the benchmark plan on this rank: prefill = RoPE operand "
                        "pass + attention kernel, median of 5 steps after an L2 flush; decode = "
                        "graph replays of 256-step loops",
                "prefill": [dict(c, attend_frac=c["attend_tflops"] / peak) for c in sweep["prefill"]],
                "decode": [dict(c, frac=c["achieved_gbs"] / peaks["hbm_gbs"])
                           for c in sweep["decode"]]},
            "two_form": {
                "what": "decode reading remote keys from an FP16 remote form of the cache "
                        "(jetlong_remote_cache once per G, jetlong_decode_two_form per step), "
                        "CUDA-graph replays of 256-step loops like the headline decode",
                "decode_us_per_token": two_us_tok,
                "achieved_gbs": decode_bytes(wd.B, wd.Hkv, wd.L, wd.D) / (two_us_tok * 1e-6) / 1e9,
                "vs_rotating_decode": two_us_tok / us_tok,
                "routing_cost_decode": two_us_tok / ctl_us_tok - 1.0,
                "rebuild_ms_all_rows": rebuild_ms,
                "rebuild_every_tokens": wd.w_pretrained},
            "e2e": {"value": e2e_val, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": n_e2e,
                    "pipelined": "step i's H2D and step i-1's D2H overlap compute on two copy "
                                 "streams (double buffers)",
                    "latency_ms_one_call": e2e_latency_ms,
                    "latency_note": "one call with nothing overlapped: H2D of q, k, v, the "
                                    "prefill, D2H of out and lse, in order on one stream"},
            "gpu_launches": 2 * args.steps + 2 * n_dec,  # timed regions: 2 per prefill step, 2 per decode
            "clocks": clocks.summary(),
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--decode-steps", type=int, default=256)
    ap.add_argument("--decode-reps", type=int, default=80)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--reference-seconds", type=float, default=120.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the per-workload sweep (16K-128K prefill, 32K-128K decode)")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)  # at least three untimed warm-up steps
    if args.impl == "reference":
        return run_reference(args)
    return run_native(args)


if __name__ == "__main__":
    sys.exit(main())

"""Benchmark of the SambaY scan + Gated Memory Unit hot path on B200.

One step = one pass of the prefill hot path over one batch: the Mamba
selective scan of a 2048-token prompt (batch 1, d_inner 5120, d_state 16,
conv 4, dt_rank 160) writing the memory readout M, then one GMU layer
Y = (M ⊙ SiLU(X W1^T)) W2 with d_model 2560, in bfloat16 I/O with float32
accumulation and state.  Metric: tokens/s over the step.  A decode
sub-benchmark (64 sequences, one token each per step: scan step + GMU step)
is reported beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun, one process per GPU, each an independent replica
(weak scaling: the sequences of different ranks share nothing, so there is
no collective on the data path).  Rank 0 prints one JSON line.
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

from gated_memory_sharing_b200 import synth  # noqa: E402

WORKLOAD = "prefill_b1_l2048"
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of a
# kernel, from one ncu capture of the benchmarked workload (profiles/); a kernel
# changed since its capture has no entry (reported as null).
DRAM_TRAFFIC = {
    # profiles/prefill_b1_l2048_launches.md (bench.py --steps 3 --warmup 3 --no-cpu-baseline --no-decode)
    "conv_silu": 21034496 + 98560,
    "x_proj": 43948032 + 768,
    "xdbl_reduce": 14177280 + 0,
    "dt_proj": 3319296 + 0,
    "selective_scan": 84559616 + 2436352,
    "gmu_gate_gemm": 57772544 + 907008,
    "gmu_out_gemm": 47287040 + 243456,
    "gmu_out_tail": 18881792 + 0,
}
METRIC = "scan+GMU prefill tokens/s"
UNIT = "tokens/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
# Special-function-unit exp2 rate per SM per clock (4 lanes per sub-partition
# x 4 sub-partitions; checked on this B200 with an ex2.approx throughput probe)
SFU_EX2_PER_SM_CLK = 16
L2_FLUSH_BYTES = 256 << 20   # > 126 MB L2


class L2Flush:
    """Evicts the step's data from the 126 MB L2 between iterations: writes a
    buffer twice the L2's size, then reads another one, so the next step finds
    neither its inputs nor dirty lines (whose write-back would otherwise land
    on the first kernel of the step)."""

    def __init__(self, device):
        import torch
        self.w = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
        self.r = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)

    def __call__(self, i):
        self.w.fill_(float(i))
        self.sink = self.r.amax()
DECODE_BATCH = 64
DECODE_RING = 64             # decode steps per captured graph


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


# --------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self._t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self._t = threading.Thread(target=self._read, daemon=True)
        self._t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self._t:
            self._t.join(timeout=2)
        sm, smax, power, reasons = [], [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        # median over the samples taken under load (top half of power draw)
        if power:
            cut = statistics.median(power)
            loaded = [s for s, p in zip(sm, power) if p >= cut] or sm
        else:
            loaded = sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


# --------------------------------------------------------------------- helpers

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend):
    import torch.distributed as dist
    from datetime import timedelta
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend=backend, timeout=timedelta(seconds=120))
    return dist


def max_over_ranks(x: float, world: int, device) -> float:
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


# --------------------------------------------------------------------- reference arm

def run_reference(args, world, rank):
    """The float64 oracle on the host cores, on a bounded sample per step."""
    if rank != 0:
        return
    from oracle import sambay_ref as ref
    d, seed = synth.workload(WORKLOAD)
    w = synth.scan_weights(d, seed)
    gw = synth.gmu_weights(d, seed)
    sample = 256
    u = synth.scan_inputs(d, seed, seqlen=sample)
    X = synth.gmu_inputs(d, seed, rows=sample)

    def step():
        r = ref.scan_prefill_ref(u, w)
        ref.gmu_ref(X, r["M"][0], gw["W1"], gw["W2"])

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    value = args.steps * sample / el
    cores = len(os.sched_getaffinity(0))
    desc = f"first {sample} tokens of the {d.seqlen}-token prompt (scan + GMU rows) per step"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "batch": d.batch, "seq_len": d.seqlen,
                   "d_model": d.d_model, "d_inner": d.d_inner, "d_state": d.d_state,
                   "sample_tokens": sample},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def kernel_work(name, d, sms, peaks, peak_kind):
    """(bound, algorithmic units per launch, unit, peak) of one kernel of the
    prefill step on dims d.  Algorithmic = what the method must compute or move
    once: exps for the scan, 2*M*N*K flops for the GEMMs, bytes read + written
    by the memory-bound kernels (inputs once, outputs once)."""
    T, Di, Dm, N, R = d.tokens, d.d_inner, d.d_model, d.d_state, d.dt_rank
    ldx, Rp = R + 2 * N, (R + 63) // 64 * 64
    hbm = peaks["hbm_gbs"]
    if name == "selective_scan":
        peak = SFU_EX2_PER_SM_CLK * sms * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e9
        return "alu", T * Di * N, "Gexp/s", peak, \
            f"SFU ex2: {SFU_EX2_PER_SM_CLK}/SM/clk x {sms} SMs x max SM clock ({peak_kind} clock)"
    if name in ("gmu_gate_gemm", "gmu_out_gemm"):
        return "tensor", 2.0 * T * Dm * Di, "TFLOP/s", peaks["bf16_tflops"], f"{peak_kind} burst bf16"
    if name == "conv_silu":      # u in (bf16), uc split pair out (2 x bf16)
        return "hbm", T * Di * (2 + 4), "GB/s", hbm, f"{peak_kind} HBM copy"
    if name == "x_proj":         # uc pair in, x_proj_w in, (delta|B|C) f32 out
        return "hbm", T * Di * 4 + ldx * Di * 2 + T * ldx * 4, "GB/s", hbm, f"{peak_kind} HBM copy"
    if name == "xdbl_reduce":    # (delta|B|C) out + split delta pair out; partials are scratch
        return "hbm", T * ldx * 4 + T * 2 * Rp * 2, "GB/s", hbm, f"{peak_kind} HBM copy"
    if name == "dt_proj":        # delta pair + W_dt in, dt f32 out
        return "hbm", T * 2 * Rp * 2 + Di * R * 2 + T * Di * 4, "GB/s", hbm, f"{peak_kind} HBM copy"
    return None


def cpu_baseline_oracle(min_seconds=10.0, max_reps=4):
    """The oracle as it stands, on the full benchmark step, timed on this host."""
    from oracle import sambay_ref as ref
    d, seed = synth.workload(WORKLOAD)
    w = synth.scan_weights(d, seed)
    gw = synth.gmu_weights(d, seed)
    u = synth.scan_inputs(d, seed)
    X = synth.gmu_inputs(d, seed)
    reps, t0 = 0, time.perf_counter()
    while reps < max_reps and (reps == 0 or time.perf_counter() - t0 < min_seconds):
        r = ref.scan_prefill_ref(u, w)
        ref.gmu_ref(X, r["M"][0], gw["W1"], gw["W2"])
        reps += 1
    el = time.perf_counter() - t0
    return {"value": reps * d.tokens / el, "unit": UNIT, "cores": len(os.sched_getaffinity(0)),
            "kind": "oracle",
            "sample": f"the whole step ({d.tokens} tokens: scan + one GMU layer) x {reps}, "
                      f"{el:.1f} s of float64 NumPy"}


# --------------------------------------------------------------------- our arm

def run_ours(args, world, rank, local):
    import torch
    from gated_memory_sharing_b200 import abi, build
    from gated_memory_sharing_b200.layers import GMULayer, ScanLayer, to_device

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    if rank == 0:
        build.build()
    barrier(world)
    abi.load()
    peaks, peak_kind = load_peaks()

    d, seed = synth.workload(WORKLOAD)
    w = synth.scan_weights(d, seed)
    gw = synth.gmu_weights(d, seed)
    # each rank: its own sequence (weak scaling), the same weights
    u_np = synth.scan_inputs(d, seed + 7919 * rank)
    X_np = synth.gmu_inputs(d, seed + 7919 * rank)
    scan = ScanLayer(w, d.d_model, abi.BF16)
    gmu = GMULayer(gw["W1"], gw["W2"], abi.BF16)
    u = to_device(u_np, abi.BF16)
    X = to_device(X_np, abi.BF16)
    T, Di, Dm = d.tokens, d.d_inner, d.d_model
    M = torch.empty_like(u)
    Y = torch.empty_like(X)
    h, cs = scan.new_state(d.batch)
    flush = L2Flush(device)
    stream = torch.cuda.current_stream()

    def step():
        scan.prefill(u, h, cs, M=M, fresh=True)

    def gmu_step():
        gmu.forward(X, M.view(T, Di), residual=False, Y=Y)

    # warm-up (also sets kernel attributes outside the timed region)
    for _ in range(max(args.warmup, 3)):
        step()
        gmu_step()
    torch.cuda.synchronize()
    assert abi.sambay_device_status() == 0

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)

    # ---- device-resident timed region: K steps, L2 flushed between steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush(i)
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
        gmu_step()
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    scan_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(args.steps)]
    gmu_ms = [ev[i][1].elapsed_time(ev[i][2]) for i in range(args.steps)]
    step_ms = [a + b for a, b in zip(scan_ms, gmu_ms)]
    total_ms = max_over_ranks(sum(step_ms), world, device)
    value = world * args.steps * T / (total_ms / 1e3)

    # ---- per-kernel timing: the same steps again, each of the library's
    # launches bracketed by CUDA events on its stream
    per_kernel = {}
    launches_per_step = None
    kt_steps = max(3, min(args.steps, 20))
    barrier(world)
    torch.cuda.synchronize()
    for i in range(kt_steps):
        flush(i)
        with abi.KernelTimer(max_launches=32) as kt:
            step()
            gmu_step()
        torch.cuda.synchronize()
        launches_per_step = len(kt.names)
        for name, ms in kt.durations_ms():
            per_kernel.setdefault(name, []).append(ms)
    barrier(world)

    # ---- end to end through the ABI with host buffers
    u_host = u.cpu().pin_memory()
    X_host = X.cpu().pin_memory()
    Y_host = torch.empty(Y.shape, dtype=Y.dtype).pin_memory()
    ev2 = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush(i)
        ev2[i][0].record(stream)
        u.copy_(u_host, non_blocking=True)
        X.copy_(X_host, non_blocking=True)
        step()
        gmu_step()
        Y_host.copy_(Y, non_blocking=True)
        ev2[i][1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(sum(ev2[i][0].elapsed_time(ev2[i][1]) for i in range(args.steps)),
                            world, device)
    e2e_value = world * args.steps * T / (e2e_ms / 1e3)

    # ---- decode sub-benchmark: 64 sequences, one token each per step
    decode = None
    if not args.no_decode:
        decode = bench_decode(args, scan, gmu, d, seed + 7919 * rank, flush, stream, world, device, peaks)
    clk = clocks.stop()
    assert abi.sambay_device_status() == 0

    # ---- roofline of every kernel; the dominant one (longest per step) leads
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    kernels = []
    for name, ms_list in per_kernel.items():
        launches = len(ms_list) / kt_steps
        ms = statistics.mean(ms_list)
        entry = {"kernel": name, "launches_per_step": launches, "ms": ms}
        kw = kernel_work(name, d, sms, peaks, peak_kind)
        if kw is not None:
            bound, units, unit, peak, peak_note = kw
            scale = 1e12 if unit == "TFLOP/s" else 1e9
            achieved = units / (ms / 1e3) / scale
            entry.update({"bound": bound, "algorithmic_per_launch": units, "achieved": achieved,
                          "peak": peak, "unit": unit, "frac": achieved / peak, "peak_note": peak_note})
        kernels.append(entry)
    kernels.sort(key=lambda e: -e["ms"] * e["launches_per_step"])
    dom = kernels[0]
    roofline = {"bound": dom.get("bound"), "achieved": dom.get("achieved"), "peak": dom.get("peak"),
                "unit": dom.get("unit"), "frac": dom.get("frac"),
                "traffic": DRAM_TRAFFIC.get(dom["kernel"]), "kernel": dom["kernel"],
                "ms_per_launch": dom["ms"], "peak_note": dom.get("peak_note")}
    scan_mean_ms = statistics.mean(scan_ms)
    gmu_mean_ms = statistics.mean(gmu_ms)

    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "batch": d.batch, "seq_len": d.seqlen,
                   "d_model": Dm, "d_inner": Di, "d_state": d.d_state, "d_conv": d.d_conv,
                   "dt_rank": d.dt_rank, "gmu_layers": 1, "parallelism": f"replicas x{world}",
                   "l2": "flushed between steps (256 MB write, then a 256 MB read of another buffer so no "
                         "dirty lines remain; outside the step events)"},
        "roofline": roofline,
        "breakdown_ms": {"scan_prefill": scan_mean_ms, "gmu_forward": gmu_mean_ms},
        "kernels": kernels,
        "e2e": {"value": e2e_value, "unit": UNIT,
                "h2d_bytes_per_step": u.numel() * 2 + X.numel() * 2,
                "d2h_bytes_per_step": Y.numel() * 2},
        "gpu_launches": launches_per_step * args.steps,   # counted by the library's launch hook
        "clocks": clk,
    }
    if decode is not None:
        out["decode"] = decode
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline_oracle()
    if rank == 0:
        print(json.dumps(out), flush=True)
    barrier(world)
    if world > 1:
        dist.destroy_process_group()


def bench_decode(args, scan, gmu, d, seed, flush, stream, world, device, peaks):
    import torch
    from gated_memory_sharing_b200.layers import to_device
    B, Di, Dm = DECODE_BATCH, d.d_inner, d.d_model
    dd = synth.Dims(B, 16, Dm, Di, d.d_state, d.d_conv, d.dt_rank, synth.BF16)
    u0 = to_device(synth.scan_inputs(dd, seed + 1), 1)                       # 16-token prompt
    ring_u = to_device(synth.scan_inputs(dd, seed + 2, seqlen=DECODE_RING, tag="u_dec"), 1)
    ring_x = to_device(synth.gmu_inputs(dd, seed + 3, rows=B * DECODE_RING, tag="X_dec"), 1)
    ring_u = ring_u.transpose(0, 1).contiguous()                              # [ring, B, Di]
    ring_x = ring_x.view(DECODE_RING, B, Dm)
    _, h, cs = scan.prefill(u0)
    m = torch.empty(B, Di, dtype=torch.bfloat16, device=device)
    y = torch.empty(DECODE_RING, B, Dm, dtype=torch.bfloat16, device=device)

    def steps():
        for i in range(DECODE_RING):
            scan.step(ring_u[i], h, cs, m_t=m)
            gmu.step(ring_x[i], m, residual=True, Y=y[i])

    steps()                      # warm-up, workspaces, kernel attributes
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        steps()
    for _ in range(max(args.warmup, 3)):
        g.replay()
    torch.cuda.synchronize()
    reps = max(args.steps // 4, 5)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
    barrier(world)
    torch.cuda.synchronize()
    for i in range(reps):
        flush(i)
        ev[i][0].record(stream)
        g.replay()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    total_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev), world, device)
    step_us = 1e3 * total_ms / (reps * DECODE_RING)
    # per-kernel breakdown of a few eager steps (launch gaps excluded)
    from gated_memory_sharing_b200 import abi
    per_kernel = {}
    for i in range(4):
        with abi.KernelTimer(max_launches=32) as kt:
            scan.step(ring_u[i], h, cs, m_t=m)
            gmu.step(ring_x[i], m, residual=True, Y=y[i])
        torch.cuda.synchronize()
        for name, ms in kt.durations_ms():
            per_kernel.setdefault(name, []).append(1e3 * ms)
    kernels_us = {k: statistics.mean(v) for k, v in per_kernel.items()}
    # algorithmic bytes per decode step (every byte the step must move once)
    state = B * Di * d.d_state * 4 * 2 + B * Di * d.d_conv * 2 * 2
    weights = (d.dt_rank + 2 * d.d_state) * Di * 2 + Di * d.dt_rank * 2 + Di * (d.d_conv + 1) * 2 \
        + Di * d.d_state * 4 + 2 * Di * 4 + 2 * Di * Dm * 2
    acts = B * (2 * Di + 3 * Dm) * 2
    nbytes = state + weights + acts
    achieved = nbytes / (step_us / 1e6) / 1e9
    del g
    return {"metric": "decode tokens/s (scan step + GMU step)", "unit": UNIT,
            "value": world * B / (step_us / 1e6), "us_per_step": step_us, "batch": B,
            "steps_timed": reps * DECODE_RING,
            "setup": "16-token prompt prefill; the decode state has a fixed size, so the step "
                     "cost does not depend on the position",
            "l2": "flushed between graph replays of 64 back-to-back steps (256 MB write + 256 MB read)",
            "kernels_us": kernels_us,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                         "algorithmic_bytes_per_step": nbytes}}


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_env()
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()

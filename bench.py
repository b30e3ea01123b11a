"""Benchmark of the SambaY scan + Gated Memory Unit hot path on B200.

The headline step is one pass of the prefill hot path over one batch: the
Mamba selective scan of a 2048-token prompt (batch 1, d_model 2560, d_inner
5120, d_state 16, conv 4, dt_rank 160) writing the memory readout M, then one
GMU layer Y = (M ⊙ SiLU(X W1^T)) W2, in bfloat16 I/O with float32
accumulation and state.  Metric: tokens/s.  The other seeded workloads of the
method are measured in the same run and reported under "workloads":

  decode_b64               64 sequences, 2048-token prompt, then decode steps
                           (scan step + one GMU layer with residual); the full
                           32768-step horizon is also timed back to back
  long_prefill_b4_l32768   4 x 32768 tokens: scan + one GMU layer
  sharing_b2_l8192         one scan of 2 x 8192 tokens whose M feeds 8 GMU
                           layers (X <- X + GMU_l(X, M))
  sharing_decode_b16       16 sequences decoding through the scan step and
                           the 8 GMU layers
  cross_attn_vs_gmu_b64    one decoded token of 64 sequences through a
                           cross-attention layer over the KV cache (2048 and
                           34816 cached tokens: the 2K prompt and the end of
                           32K generated ones) and through a GMU layer: bytes
                           and time per decoded token of each
  sambay2_prefill_b1_l2048 the SambaY-2 memory readout (Mamba-2 SSD scan) of
                           a 2048-token prompt, 80 heads of 64, d_state 128
  mamba_layer_b1_l2048     the whole Mamba layer from X at the headline sizes:
                           in_proj, the scan, (y ⊙ SiLU(X W_z^T)) W_out + X
  sambay_mlp_b1_l2048      SambaY-MLP at the headline sizes: the SwiGLU hidden
                           activation of X_self as the memory of a GMU layer
                           gated by X_cross

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--only-headline] [--no-cpu-baseline]

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

HEADLINE = "prefill_b1_l2048"
LAYER_WORKLOADS = ("mamba_layer_b1_l2048", "sambay_mlp_b1_l2048")
WORKLOADS = ("prefill_b1_l2048", "decode_b64", "long_prefill_b4_l32768", "sharing_b2_l8192",
             "sharing_decode_b16", "cross_attn_vs_gmu_b64", "sambay2_prefill_b1_l2048") + LAYER_WORKLOADS
UNIT = "tokens/s"
METRICS = {
    "prefill_b1_l2048": "scan+GMU prefill tokens/s",
    "decode_b64": "scan+GMU decode tokens/s",
    "long_prefill_b4_l32768": "scan+GMU prefill tokens/s",
    "sharing_b2_l8192": "scan+8xGMU prefill tokens/s",
    "sharing_decode_b16": "scan+8xGMU decode tokens/s",
    "cross_attn_vs_gmu_b64": "cross-attention decode tokens/s at 2048 cached tokens",
    "sambay2_prefill_b1_l2048": "SambaY-2 (Mamba-2 SSD) memory readout prefill tokens/s",
    "mamba_layer_b1_l2048": "Mamba layer (in_proj + scan + gated out_proj) prefill tokens/s",
    "sambay_mlp_b1_l2048": "SambaY-MLP memory (SwiGLU hidden activation) + GMU prefill tokens/s",
}
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch, from an
# earlier ncu capture of the headline workload, for kernels unchanged since
# that capture; any other kernel reports null.
DRAM_TRAFFIC_EARLIER_CAPTURE = {
    "selective_scan": 84601856 + 6615552,
}
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
# Special-function-unit exp2 rate per SM per clock (4 lanes per sub-partition
# x 4 sub-partitions; checked on this B200 with an ex2.approx throughput probe)
SFU_EX2_PER_SM_CLK = 16
L2_FLUSH_BYTES = 256 << 20   # > 126 MB L2
DECODE_RING = 256            # decode inputs cycle through this many steps


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


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


# --------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed regions run."""

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


def dev_normal(shape, seed, device):
    """Seeded N(0, 1) bf16 draws made on the device (the GPU arm's activations;
    the weights come from the shared seeded generator module)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def workload_dims(name):
    """(dims, seed, gmu layers, decode?) of a bench workload."""
    if name in LAYER_WORKLOADS:
        d, seed = synth.workload(HEADLINE)
        return d, seed, 1, False
    if name == "sambay2_prefill_b1_l2048":
        return synth.SSD_WORKLOAD, synth.SSD_WORKLOAD_SEED, 0, False
    if name == "cross_attn_vs_gmu_b64":
        d, seed = synth.workload("decode_b64")
        return d, seed, 1, False
    if name == "sharing_decode_b16":
        d, seed = synth.workload("sharing_b2_l8192")
        return (synth.Dims(synth.SHARING_DECODE_BATCH, 1024, d.d_model, d.d_inner, d.d_state, d.d_conv,
                           d.dt_rank, synth.BF16), seed, synth.SHARING_LAYERS, True)
    d, seed = synth.workload(name)
    if name == "decode_b64":
        return d, seed, 1, True
    layers = synth.SHARING_LAYERS if name == "sharing_b2_l8192" else 1
    return d, seed, layers, False


def config_of(name, d, layers, decode):
    if name == "sambay2_prefill_b1_l2048":
        return {"workload": name, "batch": d.batch, "seq_len": d.seqlen, "nheads": d.nheads, "headdim": d.headdim,
                "d_inner": d.nheads * d.headdim, "d_state": d.d_state, "d_conv": d.d_conv, "ngroups": 1}
    c = {"workload": name, "batch": d.batch, "seq_len": d.seqlen, "d_model": d.d_model,
         "d_inner": d.d_inner, "d_state": d.d_state, "d_conv": d.d_conv, "dt_rank": d.dt_rank,
         "gmu_layers": layers}
    if name == "mamba_layer_b1_l2048":
        c.pop("gmu_layers")
        c["layer"] = "in_proj (x branch) + scan + gated out_proj + residual"
    if name == "sambay_mlp_b1_l2048":
        c = {"workload": name, "batch": d.batch, "seq_len": d.seqlen, "d_model": d.d_model, "d_ff": d.d_inner,
             "gmu_layers": 1}
    if decode:
        c["prompt"] = d.seqlen
        c.pop("seq_len")
        c["decode_steps"] = synth.DECODE_STEPS.get("decode_b64" if name == "decode_b64" else "sharing_b2_l8192")
    return c


# --------------------------------------------------------------------- the oracle on the host

def _oracle_prefill(u, X, w, gws, residual):
    from oracle import sambay_ref as ref
    r = ref.scan_prefill_ref(u, w)
    M = r["M"].reshape(-1, u.shape[-1])
    if len(gws) == 1:
        ref.gmu_ref(X, M, gws[0]["W1"], gws[0]["W2"], residual=residual)
    else:
        ref.gmu_layers_ref(X, M, [g["W1"] for g in gws], [g["W2"] for g in gws])


def cpu_baseline(name, budget_s=8.0, reps_max=4):
    """The oracle as it stands, timed on this host on a bounded sample of the
    workload: whole prefill steps where affordable, otherwise a prefix of one
    sequence; decode steps of every sequence of the batch."""
    from oracle import sambay_ref as ref
    d, seed, layers, decode = workload_dims(name)
    cores = len(os.sched_getaffinity(0))
    if name == "sambay2_prefill_b1_l2048":
        from oracle import ssd_ref
        L = 128
        w = synth.ssd_weights(d, seed)
        xbc, dt_raw = synth.ssd_inputs(d, seed, seqlen=L)
        reps, t0 = 0, time.perf_counter()
        while reps < reps_max and (reps == 0 or time.perf_counter() - t0 < budget_s):
            ssd_ref.mamba2_scan_ref(xbc, dt_raw, w)
            reps += 1
        el = time.perf_counter() - t0
        return {"value": reps * L / el, "unit": UNIT, "cores": cores, "kind": "oracle",
                "sample": f"the first {L} tokens of the sequence (conv + SSD recurrence, all {d.nheads} heads) "
                          f"x {reps}, {el:.1f} s of float64 NumPy"}
    if name == "cross_attn_vs_gmu_b64":
        S, N = 4, d.seqlen
        q, K, V = synth.attention_inputs(S, N, synth.ATTN_Q_HEADS, synth.ATTN_KV_HEADS, synth.ATTN_HEAD_DIM, seed)
        reps, t0 = 0, time.perf_counter()
        while reps < 20 and (reps == 0 or time.perf_counter() - t0 < budget_s):
            ref.cross_attention_decode_ref(q, K, V)
            reps += 1
        el = time.perf_counter() - t0
        return {"value": reps * S / el, "unit": UNIT, "cores": cores, "kind": "oracle",
                "sample": f"cross-attention decode of {S} sequences over {N} cached tokens x {reps}, "
                          f"{el:.1f} s of float64 NumPy"}
    if name in LAYER_WORKLOADS:
        L = 256
        X = synth.gmu_inputs(d, seed, rows=L)
        reps, t0 = 0, time.perf_counter()
        if name == "mamba_layer_b1_l2048":
            w, bw = synth.scan_weights(d, seed), synth.mamba_block_weights(d, seed)
            run = lambda: ref.mamba_layer_ref(X[None], w, bw["W_in"], bw["W_z"], bw["W_out"])
            what = "in_proj + scan + gated out_proj"
        else:
            mw, gw = synth.mlp_weights(d, seed), synth.gmu_weights(d, seed)
            Xc = synth.gmu_inputs(d, seed, rows=L, tag="X_cross")
            run = lambda: ref.sambay_mlp_gmu_ref(Xc, X, mw["W_g"], mw["W_u"], gw["W1"], gw["W2"], residual=True)
            what = "SwiGLU memory + GMU layer"
        while reps < reps_max and (reps == 0 or time.perf_counter() - t0 < budget_s):
            run()
            reps += 1
        el = time.perf_counter() - t0
        return {"value": reps * L / el, "unit": UNIT, "cores": cores, "kind": "oracle",
                "sample": f"the first {L} tokens ({what}) x {reps}, {el:.1f} s of float64 NumPy"}
    w = synth.scan_weights(d, seed)
    gws = [synth.gmu_weights(d, seed, layer=l) for l in range(layers)]
    if decode:
        B = d.batch
        dd = synth.Dims(B, 16, d.d_model, d.d_inner, d.d_state, d.d_conv, d.dt_rank, synth.BF16)
        r = ref.scan_prefill_ref(synth.scan_inputs(dd, seed, tag="u_cpu"), w)
        h, cs = r["ssm_state"], r["conv_state"]
        steps, t0 = 0, time.perf_counter()
        while steps < 64 and (steps == 0 or time.perf_counter() - t0 < budget_s):
            u_t = synth.scan_inputs(dd, seed + steps, seqlen=1, tag="u_cpu_t")[:, 0]
            x = synth.gmu_inputs(dd, seed + steps, rows=B, tag="x_cpu_t")
            m, h, cs = ref.scan_step_ref(u_t, w, h, cs)
            ref.gmu_layers_ref(x, m, [g["W1"] for g in gws], [g["W2"] for g in gws])
            steps += 1
        el = time.perf_counter() - t0
        return {"value": steps * B / el, "unit": UNIT, "cores": cores, "kind": "oracle",
                "sample": f"{steps} decode steps of all {B} sequences (scan step + {layers} GMU layer(s)) "
                          f"after a 16-token prompt, {el:.1f} s of float64 NumPy"}
    if d.tokens <= 4096:
        u, X, tokens = synth.scan_inputs(d, seed), synth.gmu_inputs(d, seed), d.tokens
        what = f"the whole step ({tokens} tokens)"
    else:
        L = 512
        u = synth.scan_inputs(d, seed, batch=1, seqlen=L)
        X = synth.gmu_inputs(d, seed, rows=L)
        tokens = L
        what = f"the first {L} tokens of one sequence"
    reps, t0 = 0, time.perf_counter()
    while reps < reps_max and (reps == 0 or time.perf_counter() - t0 < budget_s):
        _oracle_prefill(u, X, w, gws, residual=layers > 1)
        reps += 1
    el = time.perf_counter() - t0
    return {"value": reps * tokens / el, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{what}: scan + {layers} GMU layer(s), x {reps}, {el:.1f} s of float64 NumPy"}


def run_reference(args, world, rank):
    """--impl reference: the float64 oracle on the host cores, each step a
    bounded sample of the headline workload (rank 0 only)."""
    if rank != 0:
        return
    name = args.workload
    d, seed, layers, decode = workload_dims(name)
    for _ in range(args.warmup):
        cpu_baseline(name, budget_s=0.0, reps_max=1)
    t0 = time.perf_counter()
    vals = [cpu_baseline(name, budget_s=0.0, reps_max=1) for _ in range(args.steps)]
    el = time.perf_counter() - t0
    value = statistics.mean(v["value"] for v in vals)
    base = dict(vals[0])
    base["value"] = value
    print(json.dumps({
        "impl": "reference", "metric": METRICS[name], "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(name, d, layers, decode),
        "cpu_baseline": base,
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# --------------------------------------------------------------------- roofline bookkeeping

def prefill_kernel_work(name, d, layers, sms, peaks, peak_kind):
    """(bound, algorithmic units per launch, unit, peak, note) of one kernel of a
    prefill step.  Algorithmic = what the method must compute or move once:
    exps for the scan, 2*M*N*K flops for a projection GEMM (its K-split tail,
    summed inside the same kernel, included), bytes read + written by the
    memory-bound kernels (inputs once, outputs once)."""
    T, Di, Dm, N, R = d.tokens, d.d_inner, d.d_model, d.d_state, d.dt_rank
    ldx, Rp = R + 2 * N, (R + 63) // 64 * 64
    hbm = peaks["hbm_gbs"]
    if name == "selective_scan":
        peak = SFU_EX2_PER_SM_CLK * sms * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e9
        return "alu", T * Di * N, "Gexp/s", peak, \
            f"SFU ex2: {SFU_EX2_PER_SM_CLK}/SM/clk x {sms} SMs x max SM clock ({peak_kind} clock)"
    if name in ("gmu_gate_gemm", "gmu_out_gemm", "in_proj", "mlp_up", "mlp_gate"):
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


def kernel_report(name, per_kernel, kt_steps, d, layers, sms, peaks, peak_kind):
    """Per-kernel entries (time, algorithmic work, achieved rate against the
    peak) of a prefill-shaped step, and the roofline of the dominant one."""
    kernels = []
    for kname, ms_list in per_kernel.items():
        cnt = len(ms_list) / kt_steps
        ms = statistics.mean(ms_list)
        entry = {"kernel": kname, "launches_per_step": cnt, "ms": ms}
        kw = prefill_kernel_work(kname, d, layers, sms, peaks, peak_kind)
        if kw is not None:
            bound, units, unit, peak, note = kw
            scale = 1e12 if unit == "TFLOP/s" else 1e9
            achieved = units / (ms / 1e3) / scale
            entry.update({"bound": bound, "algorithmic_per_launch": units, "achieved": achieved,
                          "peak": peak, "unit": unit, "frac": achieved / peak, "peak_note": note})
        kernels.append(entry)
    kernels.sort(key=lambda e: -e["ms"] * e["launches_per_step"])
    dom = kernels[0]
    roofline = {"bound": dom.get("bound"), "achieved": dom.get("achieved"), "peak": dom.get("peak"),
                "unit": dom.get("unit"), "frac": dom.get("frac"),
                "traffic": DRAM_TRAFFIC_EARLIER_CAPTURE.get(dom["kernel"]) if name == HEADLINE else None,
                "traffic_note": "from an earlier ncu capture of this kernel on this workload (unchanged "
                                "kernel), else null",
                "kernel": dom["kernel"], "ms_per_launch": dom["ms"], "peak_note": dom.get("peak_note")}
    return kernels, roofline


def decode_bytes(d, B, layers):
    """Algorithmic bytes of one decode step: the fp32 state and the conv window
    read and written, every weight read once, the activations in and out."""
    Di, Dm, N, K, R = d.d_inner, d.d_model, d.d_state, d.d_conv, d.dt_rank
    state = B * Di * N * 4 * 2 + B * Di * K * 2 * 2
    scan_w = (R + 2 * N) * Di * 2 + Di * R * 2 + Di * (K + 1) * 2 + Di * N * 4 + 2 * Di * 4
    gmu_w = layers * 2 * Di * Dm * 2
    acts = B * (2 * Di + 2 * Dm) * 2
    return state + scan_w + gmu_w + acts


# --------------------------------------------------------------------- our arm: prefill

def bench_prefill(args, ctx, name):
    import torch
    from gated_memory_sharing_b200 import abi
    from gated_memory_sharing_b200.layers import GMULayer, ScanLayer
    world, rank, device, flush, stream, peaks, peak_kind, sms = ctx
    d, seed, layers, _ = workload_dims(name)
    w = synth.scan_weights(d, seed)
    gws = [synth.gmu_weights(d, seed, layer=l) for l in range(layers)]
    scan = ScanLayer(w, d.d_model, abi.BF16)
    gmus = [GMULayer(g["W1"], g["W2"], abi.BF16) for g in gws]
    # each rank: its own sequences (weak scaling), the same weights
    u = dev_normal((d.batch, d.seqlen, d.d_inner), seed + 7919 * rank, device)
    X0 = dev_normal((d.tokens, d.d_model), seed + 7919 * rank + 1, device)
    T, Di = d.tokens, d.d_inner
    M = torch.empty_like(u)
    X = X0.clone()
    Y = torch.empty_like(X0)
    h, cs = scan.new_state(d.batch)
    residual = layers > 1

    def step():
        scan.prefill(u, h, cs, M=M, fresh=True)
        if residual:
            for g in gmus:
                g.forward(X, M.view(T, Di), residual=True, Y=X)
        else:
            gmus[0].forward(X, M.view(T, Di), residual=False, Y=Y)

    def reset():
        if residual:
            X.copy_(X0)

    for _ in range(max(args.warmup, 3)):
        reset()
        step()
    torch.cuda.synchronize()
    assert abi.sambay_device_status() == 0
    steps = args.steps if name == HEADLINE else max(3, min(args.steps, 10))

    # ---- device-resident timed region: K steps, L2 flushed between steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    for i in range(steps):
        reset()
        flush(i)
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    total_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev), world, device)
    value = world * steps * T / (total_ms / 1e3)

    # ---- per-kernel timing: the same steps again, each of the library's
    # launches bracketed by CUDA events on its stream
    per_kernel = {}
    launches = None
    kt_steps = 3
    for i in range(kt_steps):
        reset()
        flush(i)
        with abi.KernelTimer(max_launches=64) as kt:
            step()
        torch.cuda.synchronize()
        launches = len(kt.names)
        for kname, ms in kt.durations_ms():
            per_kernel.setdefault(kname, []).append(ms)

    # ---- end to end through the ABI with host buffers: every step copies its
    # inputs in from pinned host memory and its result out, as a serving loop
    # runs them: two device buffer sets, the copy-in of step i + 1 and the
    # copy-out of step i - 1 on their own streams while step i computes (the
    # library's calls all on the compute stream, so its workspaces never serve
    # two steps at once).  Time: the first copy-in's start to the last
    # copy-out's end.  The steps' inputs arrive from the host, so the L2 is
    # not flushed in between.
    u_host = u.cpu().pin_memory()
    X_host = X0.cpu().pin_memory()
    sets = []
    for k in range(2):
        sk = {"u": torch.empty_like(u), "X": torch.empty_like(X0), "M": torch.empty_like(M),
              "Y": torch.empty_like(X0)}
        sk["h"], sk["cs"] = scan.new_state(d.batch)
        sk["out"] = sk["X"] if residual else sk["Y"]
        sk["host"] = torch.empty(sk["out"].shape, dtype=sk["out"].dtype).pin_memory()
        sets.append(sk)

    def step_on(sk):
        scan.prefill(sk["u"], sk["h"], sk["cs"], M=sk["M"], fresh=True)
        if residual:
            for g in gmus:
                g.forward(sk["X"], sk["M"].view(T, Di), residual=True, Y=sk["X"])
        else:
            gmus[0].forward(sk["X"], sk["M"].view(T, Di), residual=False, Y=sk["Y"])

    s_in, s_out = torch.cuda.Stream(device=device), torch.cuda.Stream(device=device)
    e_comp = [torch.cuda.Event() for _ in range(steps)]
    e_out = [torch.cuda.Event() for _ in range(steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e0.record(s_in)
    for i in range(steps):
        sk = sets[i % 2]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(e_out[i - 2])       # set i % 2's last result has left
            sk["u"].copy_(u_host, non_blocking=True)
            sk["X"].copy_(X_host, non_blocking=True)
        stream.wait_stream(s_in)
        step_on(sk)
        e_comp[i].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(e_comp[i])
            sk["host"].copy_(sk["out"], non_blocking=True)
            e_out[i].record(s_out)
    s_out.wait_stream(stream)
    e1.record(s_out)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, device)
    assert abi.sambay_device_status() == 0

    kernels, roofline = kernel_report(name, per_kernel, kt_steps, d, layers, sms, peaks, peak_kind)
    h2d = u.numel() * 2 + X0.numel() * 2
    return {
        "metric": METRICS[name], "value": value, "unit": UNIT, "ms_per_step": total_ms / steps,
        "steps": steps, "config": config_of(name, d, layers, False),
        "l2": "flushed between steps (256 MB write, then a 256 MB read of another buffer so no dirty lines "
              "remain; outside the step events)",
        "roofline": roofline, "kernels": kernels,
        "e2e": {"value": world * steps * T / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": sets[0]["out"].numel() * 2,
                "note": "pinned host buffers; each step's copy-in and copy-out overlap its neighbours' compute "
                        "(two device buffer sets, separate copy streams)"},
        "gpu_launches": launches * steps,
    }


# --------------------------------------------------------------------- our arm: f1 / f3 layers

def bench_layer(args, ctx, name):
    """The layers around the path at the headline sizes (batch 1, 2048 tokens,
    d_model 2560, d_inner = d_ff 5120): the whole Mamba layer from X, or the
    SambaY-MLP memory read by one GMU layer.  Same timing rules as the
    headline (L2 flushed between steps, CUDA events on the stream)."""
    import torch
    from gated_memory_sharing_b200 import abi
    from gated_memory_sharing_b200.layers import GMULayer, MambaLayer, MLPMemory
    world, rank, device, flush, stream, peaks, peak_kind, sms = ctx
    d, seed, layers, _ = workload_dims(name)
    T, Dm, Di = d.tokens, d.d_model, d.d_inner
    X = dev_normal((d.batch, d.seqlen, Dm), seed + 7919 * rank + 3, device)
    if name == "mamba_layer_b1_l2048":
        layer = MambaLayer(synth.scan_weights(d, seed), synth.mamba_block_weights(d, seed), Dm, abi.BF16)
        h, cs = layer.scan.new_state(d.batch)
        ins, out = [X], None

        def step():
            nonlocal out
            out = layer.prefill(X, h, cs, fresh=True)[0]
    else:
        mw, gw = synth.mlp_weights(d, seed), synth.gmu_weights(d, seed)
        mlp, gmu = MLPMemory(mw["W_g"], mw["W_u"], abi.BF16), GMULayer(gw["W1"], gw["W2"], abi.BF16)
        X_self, X_cross = X.view(T, Dm), dev_normal((T, Dm), seed + 7919 * rank + 4, device)
        M = torch.empty(T, Di, dtype=torch.bfloat16, device=device)
        Y = torch.empty_like(X_cross)
        ins, out = [X_self, X_cross], Y

        def step():
            mlp.forward(X_self, M)
            gmu.forward(X_cross, M, residual=True, Y=Y)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    assert abi.sambay_device_status() == 0
    steps = max(3, min(args.steps, 10))
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    for i in range(steps):
        flush(i)
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    total_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev), world, device)
    value = world * steps * T / (total_ms / 1e3)

    per_kernel, launches, kt_steps = {}, None, 3
    for i in range(kt_steps):
        flush(i)
        with abi.KernelTimer(max_launches=64) as kt:
            step()
        torch.cuda.synchronize()
        launches = len(kt.names)
        for kname, ms in kt.durations_ms():
            per_kernel.setdefault(kname, []).append(ms)
    kernels, roofline = kernel_report(name, per_kernel, kt_steps, d, layers, sms, peaks, peak_kind)

    # end to end: the inputs in from pinned host memory, the output back, per step
    hosts = [t.cpu().pin_memory() for t in ins]
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(steps):
        for t, hst in zip(ins, hosts):
            t.copy_(hst, non_blocking=True)
        step()
        out_host.copy_(out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, device)
    assert abi.sambay_device_status() == 0
    return {
        "metric": METRICS[name], "value": value, "unit": UNIT, "ms_per_step": total_ms / steps,
        "steps": steps, "config": config_of(name, d, layers, False),
        "l2": "flushed between steps (256 MB write, then a 256 MB read of another buffer so no dirty lines "
              "remain; outside the step events)",
        "roofline": roofline, "kernels": kernels,
        "e2e": {"value": world * steps * T / (e2e_ms / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": sum(t.numel() * 2 for t in ins), "d2h_bytes_per_step": out.numel() * 2},
        "gpu_launches": launches * steps,
    }


# --------------------------------------------------------------------- our arm: decode

def bench_decode(args, ctx, name):
    import torch
    from gated_memory_sharing_b200 import abi
    from gated_memory_sharing_b200.layers import DecodeChain, GMULayer, ScanLayer
    world, rank, device, flush, stream, peaks, peak_kind, sms = ctx
    d, seed, layers, _ = workload_dims(name)
    B, Di, Dm = d.batch, d.d_inner, d.d_model
    w = synth.scan_weights(d, seed)
    gws = [synth.gmu_weights(d, seed, layer=l) for l in range(layers)]
    scan = ScanLayer(w, Dm, abi.BF16)
    chain = DecodeChain(scan, [GMULayer(g["W1"], g["W2"], abi.BF16) for g in gws])
    rs = seed + 7919 * rank
    # the prompt (the workload's stated length), then a ring of per-step inputs
    u0 = dev_normal((B, d.seqlen, Di), rs, device)
    ring_u = dev_normal((DECODE_RING, B, Di), rs + 1, device)
    ring_x = dev_normal((DECODE_RING, B, Dm), rs + 2, device)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    _, h, cs = scan.prefill(u0)
    t1.record(stream)
    torch.cuda.synchronize()
    prompt_ms = t0.elapsed_time(t1)
    del u0
    m = torch.empty(B, Di, dtype=torch.bfloat16, device=device)
    x = torch.empty(B, Dm, dtype=torch.bfloat16, device=device)

    def one(i):
        x.copy_(ring_x[i % DECODE_RING])
        chain.step(ring_u[i % DECODE_RING], h, cs, x, m_t=m)

    for i in range(4):           # warm-up, workspaces, kernel attributes
        one(i)
    torch.cuda.synchronize()
    # one step per graph (replayed with the L2 flushed before it), and a graph
    # of 64 back-to-back steps
    g1 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g1):
        chain.step(ring_u[0], h, cs, x, m_t=m)
    g64 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g64):
        for i in range(64):
            x.copy_(ring_x[i])
            chain.step(ring_u[i], h, cs, x, m_t=m)
    for _ in range(max(args.warmup, 3)):
        g1.replay()
        g64.replay()
    torch.cuda.synchronize()
    assert abi.sambay_device_status() == 0

    # ---- headline: L2 flushed before every step (between two steps of this
    # layer a model streams every other layer's weights through L2)
    reps = max(args.steps, 20)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
    barrier(world)
    torch.cuda.synchronize()
    for i in range(reps):
        flush(i)
        ev[i][0].record(stream)
        g1.replay()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    total_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev), world, device)
    step_us = 1e3 * total_ms / reps

    # ---- the stated horizon back to back (graphs of 64 steps, no flush)
    horizon = synth.DECODE_STEPS["decode_b64" if name == "decode_b64" else "sharing_b2_l8192"]
    horizon_ms = None
    if not args.no_horizon:
        hz = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        barrier(world)
        torch.cuda.synchronize()
        hz[0].record(stream)
        for _ in range(horizon // 64):
            g64.replay()
        hz[1].record(stream)
        torch.cuda.synchronize()
        barrier(world)
        horizon_ms = max_over_ranks(hz[0].elapsed_time(hz[1]), world, device)

    # ---- per-kernel breakdown of single steps (L2 flushed before each)
    per_kernel = {}
    launches = None
    for i in range(4):
        flush(i)
        with abi.KernelTimer(max_launches=64) as kt:
            chain.step(ring_u[i], h, cs, x, m_t=m)
        torch.cuda.synchronize()
        launches = len(kt.names)
        for kname, ms in kt.durations_ms():
            per_kernel.setdefault(kname, []).append(1e3 * ms)
    kernels_us = {k: statistics.mean(v) for k, v in per_kernel.items()}

    # ---- end to end: per step u_t and X from pinned host memory in, X (the
    # layers' output) back out
    u_host = ring_u[:64].cpu().pin_memory()
    x_host = ring_x[:64].cpu().pin_memory()
    y_host = torch.empty(64, B, Dm, dtype=torch.bfloat16).pin_memory()
    u_dev = torch.empty(B, Di, dtype=torch.bfloat16, device=device)
    e2e_steps = reps
    ev2 = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    barrier(world)
    torch.cuda.synchronize()
    ev2[0].record(stream)
    for i in range(e2e_steps):
        u_dev.copy_(u_host[i % 64], non_blocking=True)
        x.copy_(x_host[i % 64], non_blocking=True)
        chain.step(u_dev, h, cs, x, m_t=m)
        y_host[i % 64].copy_(x, non_blocking=True)
    ev2[1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(ev2[0].elapsed_time(ev2[1]), world, device)

    nbytes = decode_bytes(d, B, layers)
    achieved = nbytes / (step_us / 1e6) / 1e9
    dom = max(kernels_us.items(), key=lambda kv: kv[1])
    del g1, g64
    return {
        "metric": METRICS[name], "value": world * B / (step_us / 1e6), "unit": UNIT,
        "us_per_step": step_us, "ms_per_step": step_us / 1e3, "steps": reps,
        "config": config_of(name, d, layers, True),
        "l2": "flushed before every timed step (256 MB write + 256 MB read, outside the step events)",
        "prompt_prefill_ms": prompt_ms,
        "horizon": None if horizon_ms is None else
                   {"steps": horizon, "ms": horizon_ms, "us_per_step": 1e3 * horizon_ms / horizon,
                    "note": "back-to-back steps in graphs of 64, L2 not flushed"},
        "kernels_us": kernels_us,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                     "algorithmic_bytes_per_step": nbytes, "kernel": "whole decode step",
                     "dominant_kernel": dom[0], "dominant_kernel_us": dom[1],
                     "peak_note": f"{peak_kind} HBM copy"},
        "e2e": {"value": world * e2e_steps * B / (e2e_ms / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": B * (Di + Dm) * 2, "d2h_bytes_per_step": B * Dm * 2},
        "gpu_launches": launches * reps,
    }


# --------------------------------------------------------------------- our arm: SambaY-2 prefill

def bench_ssd(args, ctx, name):
    """The SambaY-2 variant's memory readout over a prompt: conv over
    [x | B | C], softplus dt, and the chunked Mamba-2 SSD scan."""
    import torch
    from gated_memory_sharing_b200 import abi
    from gated_memory_sharing_b200.layers import Mamba2Scan
    world, rank, device, flush, stream, peaks, peak_kind, sms = ctx
    d, seed, _, _ = workload_dims(name)
    layer = Mamba2Scan(synth.ssd_weights(d, seed))
    rs = seed + 7919 * rank
    xbc = dev_normal((d.batch, d.seqlen, d.channels), rs, device)
    dt_raw = (0.5 * dev_normal((d.batch, d.seqlen, d.nheads), rs + 1, device).float()).to(torch.bfloat16)
    M, h, cs = layer.prefill(xbc, dt_raw)

    def step():
        layer.prefill(xbc, dt_raw, h, cs, M=M, fresh=True)

    for _ in range(max(args.warmup, 3)):
        step()
    steps = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    for i in range(steps):
        flush(i)
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    total_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev), world, device)
    ms = total_ms / steps
    per_kernel = {}
    for i in range(3):
        flush(i)
        with abi.KernelTimer(max_launches=16) as kt:
            step()
        torch.cuda.synchronize()
        launches = len(kt.names)
        for kname, kms in kt.durations_ms():
            per_kernel.setdefault(kname, []).append(1e3 * kms)
    kernels_us = {k: statistics.mean(v) for k, v in per_kernel.items()}
    # algorithmic bytes: the in_proj slices in, M out, the fp32 state in and
    # out, the conv window; the weights are a few KB
    T, P, N, H = d.batch * d.seqlen, d.headdim, d.d_state, d.nheads
    nbytes = T * d.channels * 2 + T * H * 2 + T * H * P * 2 + 2 * d.batch * H * P * N * 4
    achieved = nbytes / (ms / 1e3) / 1e9
    # end to end: the in_proj slices from pinned host memory in, M back out
    xh = xbc.cpu().pin_memory()
    dh = dt_raw.cpu().pin_memory()
    mh = torch.empty(M.shape, dtype=M.dtype).pin_memory()
    xd, dd = torch.empty_like(xbc), torch.empty_like(dt_raw)
    e2e_ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    barrier(world)
    torch.cuda.synchronize()
    e2e_ev[0].record(stream)
    for _ in range(steps):
        xd.copy_(xh, non_blocking=True)
        dd.copy_(dh, non_blocking=True)
        layer.prefill(xd, dd, h, cs, M=M, fresh=True)
        mh.copy_(M, non_blocking=True)
    e2e_ev[1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e2e_ev[0].elapsed_time(e2e_ev[1]), world, device)
    dom = max(kernels_us.items(), key=lambda kv: kv[1])
    return {
        "metric": METRICS[name], "value": world * T / (ms / 1e3), "unit": UNIT, "ms_per_step": ms,
        "steps": steps, "config": config_of(name, d, 0, False),
        "l2": "flushed before every timed step (256 MB write + 256 MB read, outside the step events)",
        "kernels_us": kernels_us,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": None, "algorithmic_bytes_per_step": nbytes,
                     "kernel": "whole SambaY-2 readout (conv + SSD scan + conv state)",
                     "dominant_kernel": dom[0], "dominant_kernel_us": dom[1], "peak_note": f"{peak_kind} HBM copy"},
        "e2e": {"value": world * steps * T / (e2e_ms / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": (xbc.numel() + dt_raw.numel()) * 2, "d2h_bytes_per_step": M.numel() * 2},
        "gpu_launches": launches * steps,
    }


# --------------------------------------------------------------------- our arm: attention vs GMU

def bench_attn_vs_gmu(args, ctx, name):
    """The pages' decode I/O claim on this machine: a cross-attention layer reads
    the whole KV cache per decoded token, a GMU layer its two weight matrices
    (shared by the batch)."""
    import torch
    from gated_memory_sharing_b200 import abi
    from gated_memory_sharing_b200.layers import GMULayer, workspace
    world, rank, device, flush, stream, peaks, peak_kind, sms = ctx
    d, seed = synth.workload("decode_b64")
    B, Dm, Di = d.batch, d.d_model, d.d_inner
    Hq, Hkv, dh = synth.ATTN_Q_HEADS, synth.ATTN_KV_HEADS, synth.ATTN_HEAD_DIM
    rs = seed + 7919 * rank
    res = {}
    steps = max(5, min(args.steps, 20))

    def timed(fn):
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        for _ in range(3):
            fn()
        barrier(world)
        torch.cuda.synchronize()
        for i in range(steps):
            flush(i)
            ev[i][0].record(stream)
            fn()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        barrier(world)
        return max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev), world, device) / steps

    n_max = synth.DECODE_STEPS["decode_b64"] + d.seqlen
    q = dev_normal((B, Hq, dh), rs, device)
    Kc = dev_normal((B, n_max, Hkv, dh), rs + 1, device)
    Vc = dev_normal((B, n_max, Hkv, dh), rs + 2, device)
    out = torch.empty(B, Hq, dh, dtype=torch.bfloat16, device=device)
    for N in (d.seqlen, n_max):
        # the first N tokens of each sequence's cache: [B, N, Hkv, dh] views of the
        # full cache are not dense, so each length has its own dense copy
        K = Kc[:, :N].contiguous()
        V = Vc[:, :N].contiguous()
        dims = abi.AttnDims(B, N, Hq, Hkv, dh)
        ws = workspace(abi.sambay_cross_attn_decode_workspace(dims), device)
        ms = timed(lambda: abi.sambay_cross_attn_decode(dims, q, K, V, out, 0.0, ws))
        nbytes = 2 * B * N * Hkv * dh * 2 + 2 * B * Hq * dh * 2
        res[N] = {"cached_tokens": N, "us_per_step": 1e3 * ms, "bytes_per_step": nbytes,
                  "bytes_per_decoded_token": nbytes / B, "tokens_per_s": world * B / (ms / 1e3),
                  "achieved_gbs": nbytes / (ms / 1e3) / 1e9}
        del K, V
    del Kc, Vc
    gw = synth.gmu_weights(d, seed)
    gmu = GMULayer(gw["W1"], gw["W2"], abi.BF16)
    X = dev_normal((B, Dm), rs + 3, device)
    M = dev_normal((B, Di), rs + 4, device)
    Y = torch.empty_like(X)
    ms_g = timed(lambda: gmu.step(X, M, residual=True, Y=Y))
    gbytes = 2 * Di * Dm * 2 + B * (2 * Dm + Di + Dm) * 2
    a0 = res[d.seqlen]
    return {
        "metric": METRICS[name], "value": a0["tokens_per_s"], "unit": UNIT, "ms_per_step": a0["us_per_step"] / 1e3,
        "steps": steps,
        "config": {"workload": name, "batch": B, "q_heads": Hq, "kv_heads": Hkv, "head_dim": dh, "d_model": Dm,
                   "d_inner": Di, "cached_tokens": [d.seqlen, n_max]},
        "l2": "flushed before every timed call (256 MB write + 256 MB read, outside the events)",
        "cross_attention": list(res.values()),
        "gmu_layer": {"us_per_step": 1e3 * ms_g, "bytes_per_step": gbytes, "bytes_per_decoded_token": gbytes / B,
                      "tokens_per_s": world * B / (ms_g / 1e3), "achieved_gbs": gbytes / (ms_g / 1e3) / 1e9},
        "bytes_per_token_ratio": {str(N): r["bytes_per_decoded_token"] / (gbytes / B) for N, r in res.items()},
        "time_ratio": {str(N): r["us_per_step"] / (1e3 * ms_g) for N, r in res.items()},
        "roofline": {"bound": "hbm", "achieved": a0["achieved_gbs"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": a0["achieved_gbs"] / peaks["hbm_gbs"], "traffic": None,
                     "kernel": "cross_attn_decode (2048 cached tokens)", "peak_note": f"{peak_kind} HBM copy"},
        "e2e": None,
        "gpu_launches": steps,
    }


def run_ours(args, world, rank, local):
    import torch
    from gated_memory_sharing_b200 import abi, build

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    if rank == 0:
        build.build()
    barrier(world)
    abi.load()
    peaks, peak_kind = load_peaks()
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    ctx = (world, rank, device, L2Flush(device), torch.cuda.current_stream(), peaks, peak_kind, sms)
    names = [args.workload] if args.only_headline else \
        [args.workload] + [n for n in WORKLOADS if n != args.workload]

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    results = {}
    for name in names:
        if name == "cross_attn_vs_gmu_b64":
            results[name] = bench_attn_vs_gmu(args, ctx, name)
            continue
        if name == "sambay2_prefill_b1_l2048":
            results[name] = bench_ssd(args, ctx, name)
            continue
        if name in LAYER_WORKLOADS:
            results[name] = bench_layer(args, ctx, name)
            continue
        fn = bench_decode if workload_dims(name)[3] else bench_prefill
        results[name] = fn(args, ctx, name)
        torch.cuda.synchronize()
        assert abi.sambay_device_status() == 0, f"device status after {name}"
    clk = clocks.stop()

    head = results[args.workload]
    out = {
        "metric": head["metric"], "value": head["value"], "unit": UNIT, "n_gpus": world,
        "steps": head["steps"], "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": dict(head["config"], parallelism=f"replicas x{world}", l2=head["l2"]),
        "roofline": head["roofline"],
        "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"],
        "clocks": clk,
        "peaks": peak_kind,
    }
    for k in ("kernels", "kernels_us", "horizon", "prompt_prefill_ms", "us_per_step"):
        if k in head:
            out[k] = head[k]
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        for name in names:
            results[name]["cpu_baseline"] = cpu_baseline(name)
        out["cpu_baseline"] = results[args.workload]["cpu_baseline"]
    out["workloads"] = {n: r for n, r in results.items() if n != args.workload}
    if rank == 0:
        print(json.dumps(out), flush=True)
    barrier(world)
    if world > 1:
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=WORKLOADS, default=HEADLINE)
    ap.add_argument("--only-headline", action="store_true", help="measure the headline workload only")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-horizon", action="store_true",
                    help="decode workloads: skip the back-to-back run over the stated horizon (profiling runs)")
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

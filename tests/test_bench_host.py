"""bench.py's bookkeeping on the host: the roofline arithmetic of the
per-kernel report, the workload table, and the oracle baselines of the layer
workloads (no GPU)."""

import math

import pytest

import bench

PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "sm_max_mhz": 1965.0}


def test_every_workload_has_a_metric_and_dims():
    assert bench.HEADLINE in bench.WORKLOADS
    for name in bench.WORKLOADS:
        assert name in bench.METRICS
        d, seed, layers, decode = bench.workload_dims(name)
        assert d.batch >= 1 and layers >= 0 and isinstance(decode, bool)
        assert bench.config_of(name, d, layers, decode)["workload"] == name


def test_kernel_report_roofline_arithmetic():
    """Achieved rates and fractions from their definitions: exp2 per second
    against 16 per SM per clock for the scan, 2*M*N*K per second against the
    bf16 peak for a projection GEMM, bytes per second against HBM for x_proj."""
    d, _, layers, _ = bench.workload_dims(bench.HEADLINE)
    T, Di, Dm, N, R = d.tokens, d.d_inner, d.d_model, d.d_state, d.dt_rank
    ms = {"selective_scan": 0.120, "gmu_out_gemm": 0.050, "x_proj": 0.020, "not_a_kernel_of_the_path": 0.001}
    per_kernel = {k: [v] * 3 for k, v in ms.items()}
    kernels, roof = bench.kernel_report(bench.HEADLINE, per_kernel, 3, d, layers, 148, PEAKS, "test")
    by = {k["kernel"]: k for k in kernels}

    assert [k["kernel"] for k in kernels] == sorted(ms, key=lambda k: -ms[k])   # longest first
    assert all(k["launches_per_step"] == 1.0 for k in kernels)

    sfu = 16 * 148 * 1965e6 / 1e9                       # Gexp/s
    scan = T * Di * N / (ms["selective_scan"] * 1e-3) / 1e9
    assert math.isclose(by["selective_scan"]["peak"], sfu)
    assert math.isclose(by["selective_scan"]["achieved"], scan)
    assert math.isclose(by["selective_scan"]["frac"], scan / sfu)
    assert by["selective_scan"]["bound"] == "alu"

    gemm = 2.0 * T * Dm * Di / (ms["gmu_out_gemm"] * 1e-3) / 1e12
    assert by["gmu_out_gemm"]["bound"] == "tensor"
    assert math.isclose(by["gmu_out_gemm"]["frac"], gemm / PEAKS["bf16_tflops"])

    ldx = R + 2 * N
    xbytes = T * Di * 4 + ldx * Di * 2 + T * ldx * 4    # uc pair in, weight in, (delta|B|C) out
    assert by["x_proj"]["bound"] == "hbm"
    assert math.isclose(by["x_proj"]["achieved"], xbytes / (ms["x_proj"] * 1e-3) / 1e9)

    assert "bound" not in by["not_a_kernel_of_the_path"]
    assert roof["kernel"] == "selective_scan" and math.isclose(roof["frac"], scan / sfu)


@pytest.mark.parametrize("name", ["mamba_layer_b1_l2048", "sambay_mlp_b1_l2048"])
def test_layer_workload_config(name):
    assert name in bench.LAYER_WORKLOADS
    d, _, layers, decode = bench.workload_dims(name)
    assert (d.batch, d.seqlen, d.d_model, d.d_inner) == (1, 2048, 2560, 5120) and not decode
    cfg = bench.config_of(name, d, layers, decode)
    assert cfg["batch"] == 1 and cfg["seq_len"] == 2048 and cfg["d_model"] == 2560
    assert cfg.get("d_inner", cfg.get("d_ff")) == 5120


@pytest.mark.parametrize("name", bench.WORKLOADS)
def test_oracle_baseline_of_every_workload(name):
    """The reference arm's unit of work (one bounded oracle sample) runs for
    every workload and describes itself."""
    base = bench.cpu_baseline(name, budget_s=0.0, reps_max=1)
    assert base["kind"] == "oracle" and base["unit"] == bench.UNIT
    assert base["value"] > 0 and base["cores"] >= 1 and base["sample"]

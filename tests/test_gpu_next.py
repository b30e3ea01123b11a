"""GPU parity of the rows next to the scan + GMU path, through the C ABI.

* The whole Mamba layer whose readout is M: in_proj's scan branch
  (sambay_in_proj), the scan, and the gated out_proj (gmu_forward with
  W1 = W_z, W2 = W_out); prefill, and decode step by step.  The tiny float32
  workload runs as stated: one Mamba layer producing M from X, then one GMU
  layer reusing M.
* SambaY-MLP: the SwiGLU hidden activation as the memory
  (sambay_mlp_memory), then the GMU on it; prefill rows and decode rows.

Every expected value comes from the float64 oracle on the seeded inputs.
"""

import numpy as np
import pytest
import torch

from gated_memory_sharing_b200 import abi, synth
from gated_memory_sharing_b200.layers import GMULayer, MLPMemory, MambaLayer, to_device
from oracle import sambay_ref as ref
from tests.gpu_util import TOL_BF16, TOL_F32, assert_close, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from gated_memory_sharing_b200 import build
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    abi.load()
    torch.cuda.set_device(0)
    yield
    assert abi.sambay_device_status() == 0


def _io(d):
    return (abi.BF16, TOL_BF16) if d.io == synth.BF16 else (abi.F32, TOL_F32)


def test_tiny_workload_mamba_layer_then_gmu_f32():
    """The tiny float32 workload as stated: one Mamba layer producing M from X
    (in_proj, conv, scan), then one GMU layer (W1: 64 -> 128, W2: 128 -> 64)."""
    d, seed = synth.workload("tiny_f32")
    w = synth.scan_weights(d, seed)
    bw = synth.mamba_block_weights(d, seed)
    gw = synth.gmu_weights(d, seed)
    X = synth.gmu_inputs(d, seed).reshape(d.batch, d.seqlen, d.d_model)
    Xc = synth.gmu_inputs(d, seed, tag="X_cross")
    layer = MambaLayer(w, bw, d.d_model, abi.F32)
    gmu = GMULayer(gw["W1"], gw["W2"], abi.F32)
    out, M, h, cs = layer.prefill(to_device(X, abi.F32))
    Y = gmu.forward(to_device(Xc, abi.F32), M.reshape(-1, d.d_inner))
    r = ref.mamba_layer_ref(X, w, bw["W_in"], bw["W_z"], bw["W_out"])
    Yr, _, _ = ref.gmu_ref(Xc, r["M"].reshape(-1, d.d_inner), gw["W1"], gw["W2"])
    assert_close(host(M), r["M"], TOL_F32, "tiny Mamba layer M")
    assert_close(host(out), r["out"], TOL_F32, "tiny Mamba layer out")
    assert_close(host(h), r["ssm_state"], TOL_F32, "tiny Mamba layer h")
    assert_close(host(Y), Yr, TOL_F32, "tiny GMU on the Mamba layer's M")


@pytest.mark.parametrize("d", [
    synth.Dims(2, 77, 128, 256, 16, 4, 16, synth.BF16),
    synth.Dims(3, 45, 64, 128, 16, 4, 8, synth.F32),
], ids=["bf16", "f32"])
def test_mamba_layer_prefill_then_decode(d):
    io, tol = _io(d)
    seed = 61
    w = synth.scan_weights(d, seed)
    bw = synth.mamba_block_weights(d, seed)
    X = synth.gmu_inputs(d, seed).reshape(d.batch, d.seqlen, d.d_model)
    L0 = d.seqlen - 5
    layer = MambaLayer(w, bw, d.d_model, io)
    out, M, h, cs = layer.prefill(to_device(np.ascontiguousarray(X[:, :L0]), io))
    r = ref.mamba_layer_ref(X, w, bw["W_in"], bw["W_z"], bw["W_out"], io_round=io == abi.BF16)
    assert_close(host(M), r["M"][:, :L0], tol, "Mamba layer M (prefill)")
    assert_close(host(out), r["out"][:, :L0], tol, "Mamba layer out (prefill)")
    for i in range(L0, d.seqlen):
        o_t, m_t = layer.step(to_device(np.ascontiguousarray(X[:, i]), io), h, cs)
        assert_close(host(m_t), r["M"][:, i], tol, f"Mamba layer m_t step {i}")
        assert_close(host(o_t), r["out"][:, i], tol, f"Mamba layer out step {i}")
    assert_close(host(h), r["ssm_state"], tol, "Mamba layer h after decoding")
    # the window holds u = X W_in^T as in_proj wrote it (io-typed)
    assert_close(host(cs), r["conv_state"], tol, "Mamba layer conv window")


def test_mamba_layer_full_width_b1_l2048():
    """The Mamba layer at the prefill workload's width (d_model 2560, d_inner
    5120, 2048 tokens): M in full, the layer output on sampled rows."""
    d, seed = synth.workload("prefill_b1_l2048")
    w = synth.scan_weights(d, seed)
    bw = synth.mamba_block_weights(d, seed)
    X = synth.gmu_inputs(d, seed).reshape(d.batch, d.seqlen, d.d_model)
    layer = MambaLayer(w, bw, d.d_model, abi.BF16)
    out, M, h, _ = layer.prefill(to_device(X, abi.BF16))
    # u (in_proj -> scan) and M (scan -> gated output) cross the ABI as bf16
    r = ref.mamba_layer_ref(X, w, bw["W_in"], bw["W_z"], bw["W_out"], io_round=True)
    assert_close(host(M), r["M"], TOL_BF16, "full-width Mamba layer M")
    assert_close(host(h), r["ssm_state"], TOL_BF16, "full-width Mamba layer h")
    rows = np.unique(np.concatenate([np.random.default_rng(5).choice(d.tokens, 48, replace=False),
                                     [0, d.tokens - 1]]))
    assert_close(host(out).reshape(-1, d.d_model)[rows], r["out"].reshape(-1, d.d_model)[rows], TOL_BF16,
                 "full-width Mamba layer out (sampled rows)")


@pytest.mark.parametrize("rows,io_name", [(300, "bf16"), (1, "bf16"), (16, "bf16"), (64, "bf16"), (200, "bf16"),
                                          (77, "f32")])
def test_sambay_mlp_memory_and_gmu(rows, io_name):
    if io_name == "bf16":
        d = synth.Dims(1, 1, 256, 512, 16, 4, 16, synth.BF16)
    else:
        d = synth.Dims(1, 1, 64, 128, 16, 4, 8, synth.F32)
    io, tol = _io(d)
    seed = 70 + rows
    mw = synth.mlp_weights(d, seed)
    gw = synth.gmu_weights(d, seed)
    Xs = synth.gmu_inputs(d, seed, rows=rows, tag="X_self")
    Xc = synth.gmu_inputs(d, seed, rows=rows, tag="X_cross")
    mem = MLPMemory(mw["W_g"], mw["W_u"], io)
    gmu = GMULayer(gw["W1"], gw["W2"], io)
    M = mem.forward(to_device(Xs, io))
    Xcd = to_device(Xc, io)
    Y = gmu.forward(Xcd, M) if rows > 256 or rows % 2 == 0 else gmu.step(Xcd, M)
    Yr, Mr = ref.sambay_mlp_gmu_ref(Xc, Xs, mw["W_g"], mw["W_u"], gw["W1"], gw["W2"])
    assert_close(host(M), Mr, tol, f"MLP memory rows={rows}")
    assert_close(host(Y), Yr, tol, f"SambaY-MLP GMU rows={rows}")


def test_sambay_mlp_full_width_rows():
    """SambaY-MLP at the model width (d_model 2560, MLP width 5120): 2048
    prefill rows (sampled) and 64 decode rows (all)."""
    d, seed = synth.workload("prefill_b1_l2048")
    mw = synth.mlp_weights(d, seed)
    gw = synth.gmu_weights(d, seed)
    mem = MLPMemory(mw["W_g"], mw["W_u"], abi.BF16)
    gmu = GMULayer(gw["W1"], gw["W2"], abi.BF16)
    for rows, sample in ((2048, 40), (64, 64)):
        Xs = synth.gmu_inputs(d, seed, rows=rows, tag="X_self")
        Xc = synth.gmu_inputs(d, seed, rows=rows, tag="X_cross")
        M = mem.forward(to_device(Xs, abi.BF16))
        Xcd = to_device(Xc, abi.BF16)
        Y = gmu.forward(Xcd, M, residual=True) if rows > 256 else gmu.step(Xcd, M, residual=True)
        idx = np.unique(np.random.default_rng(rows).choice(rows, sample, replace=False))
        Yr, Mr = ref.sambay_mlp_gmu_ref(Xc[idx], Xs[idx], mw["W_g"], mw["W_u"], gw["W1"], gw["W2"], residual=True)
        assert_close(host(M)[idx], Mr, TOL_BF16, f"MLP memory rows={rows}")
        assert_close(host(Y)[idx], Yr, TOL_BF16, f"SambaY-MLP GMU rows={rows}")

"""GPU parity: the CUDA path through the C ABI against the float64 oracle.

Small cases span several tiles with ragged tails (rows not a multiple of 128,
sequence lengths not a multiple of the 32-token scan chunk) and the edge cases
(L = 1, one sequence, one decode row); the full-size prefill workload
(batch 1 x 2048 tokens, d_model 2560, d_inner 5120) is checked in the launch
configuration the benchmark times, the scan readout in full and the GMU on
sampled rows (GMU rows are independent, so a sampled row is an exact check).
"""

import numpy as np
import pytest
import torch

from gated_memory_sharing_b200 import abi, synth
from gated_memory_sharing_b200.layers import GMULayer, ScanLayer, to_device, to_device_f32
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


def _io(io_name):
    return (abi.BF16, TOL_BF16) if io_name == synth.BF16 else (abi.F32, TOL_F32)


SMALL = {
    "f32": synth.Dims(2, 77, 64, 128, 16, 4, 8, synth.F32),
    "bf16": synth.Dims(3, 100, 128, 256, 16, 4, 16, synth.BF16),
}


# ------------------------------------------------------------------ GMU

@pytest.mark.parametrize("name", ["f32", "bf16"])
@pytest.mark.parametrize("residual", [False, True])
def test_gmu_forward_small(name, residual):
    d = SMALL[name]
    io, tol = _io(d.io)
    seed = 11
    gw = synth.gmu_weights(d, seed)
    rows = 300                                   # 2 full 128-row tiles + a ragged one
    X = synth.gmu_inputs(d, seed, rows=rows)
    M = synth.memory_input(d, seed, rows=rows)
    g = GMULayer(gw["W1"], gw["W2"], io)
    Y = g.forward(to_device(X, io), to_device(M, io), residual=residual)
    Yr, _, _ = ref.gmu_ref(X, M, gw["W1"], gw["W2"], residual=residual)
    assert_close(host(Y), Yr, tol, f"gmu_forward {name}")


def test_gmu_forward_multi_tile_bf16():
    # several 128 x 256 tiles of GEMM1 and 128 x 128 tiles of GEMM2, K over
    # several 64-blocks, rows ragged
    d = synth.Dims(1, 1, 384, 640, 16, 4, 16, synth.BF16)
    seed = 12
    gw = synth.gmu_weights(d, seed)
    rows = 333
    X = synth.gmu_inputs(d, seed, rows=rows)
    M = synth.memory_input(d, seed, rows=rows)
    g = GMULayer(gw["W1"], gw["W2"], abi.BF16)
    Y = g.forward(to_device(X, abi.BF16), to_device(M, abi.BF16), residual=True)
    Yr, _, _ = ref.gmu_ref(X, M, gw["W1"], gw["W2"], residual=True)
    assert_close(host(Y), Yr, TOL_BF16, "gmu_forward multi-tile")


@pytest.mark.parametrize("rows,d_model,d_inner", [
    (1900, 2560, 1024),     # GEMM2: 8 x 10 tiles of 256 x 256 on 74 CTA pairs, the last 6 cut along K
    (500, 768, 12032),      # GEMM1: 2 x 47 tiles, the last 20 cut along K into 3
])
def test_gmu_forward_k_split_tail_bf16(rows, d_model, d_inner):
    # more 256-row tiles than CTA pairs: the partial last round runs as K
    # ranges (first, one per CTA pair) whose fp32 partial tiles the same
    # kernel's CTAs sum in a fixed order after their last whole tile
    d = synth.Dims(1, 1, d_model, d_inner, 16, 4, 16, synth.BF16)
    seed = 15
    gw = synth.gmu_weights(d, seed)
    X = synth.gmu_inputs(d, seed, rows=rows)
    M = synth.memory_input(d, seed, rows=rows)
    g = GMULayer(gw["W1"], gw["W2"], abi.BF16)
    Y = g.forward(to_device(X, abi.BF16), to_device(M, abi.BF16), residual=True)
    Yr, _, _ = ref.gmu_ref(X, M, gw["W1"], gw["W2"], residual=True)
    assert_close(host(Y), Yr, TOL_BF16, f"gmu_forward K-split tail rows={rows}")
    # deterministic: the same bits on a second call, whatever the scratch holds
    # on entry (the tail's arrival word included: random bytes here)
    ws = g._ws[("fwd", rows)]
    gen = torch.Generator(device=ws.device)
    gen.manual_seed(rows)
    ws.copy_(torch.randint(0, 256, ws.shape, generator=gen, device=ws.device, dtype=torch.int32).to(ws.dtype))
    assert torch.equal(Y, g.forward(to_device(X, abi.BF16), to_device(M, abi.BF16), residual=True))


def test_gmu_forward_in_place_residual_bf16():
    d = SMALL["bf16"]
    seed = 13
    gw = synth.gmu_weights(d, seed)
    X = synth.gmu_inputs(d, seed, rows=130)
    M = synth.memory_input(d, seed, rows=130)
    g = GMULayer(gw["W1"], gw["W2"], abi.BF16)
    Xd = to_device(X, abi.BF16)
    g.forward(Xd, to_device(M, abi.BF16), residual=True, Y=Xd)      # X <- X + GMU(X, M)
    Yr, _, _ = ref.gmu_ref(X, M, gw["W1"], gw["W2"], residual=True)
    assert_close(host(Xd), Yr, TOL_BF16, "gmu_forward in place")


@pytest.mark.parametrize("name", ["f32", "bf16"])
@pytest.mark.parametrize("rows", [1, 16, 64, 100, 256])
def test_gmu_step(name, rows):
    d = SMALL[name] if name == "f32" else synth.Dims(1, 1, 256, 512, 16, 4, 16, synth.BF16)
    io, tol = _io(d.io)
    seed = 14 + rows
    gw = synth.gmu_weights(d, seed)
    X = synth.gmu_inputs(d, seed, rows=rows)
    M = synth.memory_input(d, seed, rows=rows)
    g = GMULayer(gw["W1"], gw["W2"], io)
    Xd, Md = to_device(X, io), to_device(M, io)
    for residual in (False, True):
        Y = g.step(Xd, Md, residual=residual)
        Yr, _, _ = ref.gmu_ref(X, M, gw["W1"], gw["W2"], residual=residual)
        assert_close(host(Y), Yr, tol, f"gmu_step {name} rows={rows} residual={residual}")
    # a second call reuses the self-cleaned split-K buffers
    Y2 = g.step(Xd, Md, residual=True)
    assert torch.equal(Y2, g.step(Xd, Md, residual=True))


# ------------------------------------------------------------------ scan

@pytest.mark.parametrize("name", ["f32", "bf16"])
def test_scan_prefill_small(name):
    d = SMALL[name]
    io, tol = _io(d.io)
    seed = 21
    w = synth.scan_weights(d, seed)
    u = synth.scan_inputs(d, seed)
    layer = ScanLayer(w, d.d_model, io)
    M, h, cs = layer.prefill(to_device(u, io))
    r = ref.scan_prefill_ref(u, w)
    assert_close(host(M), r["M"], tol, f"scan M {name}")
    assert_close(host(h), r["ssm_state"], tol, f"scan h {name}")
    np.testing.assert_array_equal(host(cs), r["conv_state"])


@pytest.mark.parametrize("L", [1, 3, 31, 32, 33])
def test_scan_prefill_short_and_ragged(L):
    d = synth.Dims(1, L, 64, 128, 16, 4, 8, synth.BF16)
    seed = 22 + L
    w = synth.scan_weights(d, seed)
    u = synth.scan_inputs(d, seed)
    layer = ScanLayer(w, d.d_model, abi.BF16)
    M, h, cs = layer.prefill(to_device(u, abi.BF16))
    r = ref.scan_prefill_ref(u, w)
    assert_close(host(M), r["M"], TOL_BF16, f"scan L={L}")
    assert_close(host(h), r["ssm_state"], TOL_BF16, f"state L={L}")
    np.testing.assert_array_equal(host(cs), r["conv_state"])


@pytest.mark.parametrize("B,L,Di,R", [
    (2, 150, 320, 72),    # 300 tokens: 4 whole 64-token tiles + 44; 2.5 channel tiles; R < its 128 pad
    (1, 129, 192, 160),   # one token past a tile; R = 160 padded to 192
    (2, 200, 256, 128),   # x_proj (R + 32 = 160 columns) on CTA pairs: a 256-row tile and a 144-row one
])
def test_scan_prefill_ragged_projection_tiles(B, L, Di, R):
    """Prefill whose x_proj / dt projection tiles are ragged in tokens,
    channels and rank."""
    d = synth.Dims(B, L, 128, Di, 16, 4, R, synth.BF16)
    seed = 25 + L + R
    w = synth.scan_weights(d, seed)
    u = synth.scan_inputs(d, seed)
    layer = ScanLayer(w, d.d_model, abi.BF16)
    M, h, cs = layer.prefill(to_device(u, abi.BF16))
    r = ref.scan_prefill_ref(u, w)
    assert_close(host(M), r["M"], TOL_BF16, f"scan B{B} L{L} Di{Di} R{R}")
    assert_close(host(h), r["ssm_state"], TOL_BF16, "state")
    np.testing.assert_array_equal(host(cs), r["conv_state"])


@pytest.mark.parametrize("io", [synth.BF16, synth.F32])
def test_scan_prefill_mixed_cta_widths(io):
    """8 sequences x 640 channels: the partition makes 18 CTAs per sequence,
    16 of nine 4-channel quads and 2 of eight (the narrower CTAs' spare lanes
    run on unused tile columns), over 70 tokens (a ragged third chunk), from
    a given state."""
    d = synth.Dims(8, 70, 128, 640, 16, 4, 16, io)
    aio, tol = _io(io)
    seed = 29
    w = synth.scan_weights(d, seed)
    u = synth.scan_inputs(d, seed)
    rng = np.random.default_rng(3)
    h0 = rng.standard_normal((d.batch, d.d_inner, 16)).astype(np.float32)
    cs0 = synth.round_bf16(rng.standard_normal((d.batch, d.d_inner, 4)).astype(np.float32)) \
        if io == synth.BF16 else rng.standard_normal((d.batch, d.d_inner, 4)).astype(np.float32)
    layer = ScanLayer(w, d.d_model, aio)
    h, cs = to_device_f32(h0), to_device(cs0, aio)
    M, h, cs = layer.prefill(to_device(u, aio), h, cs, fresh=False)
    r = ref.scan_prefill_ref(u, w, h0, cs0)
    assert_close(host(M), r["M"], tol, f"scan M mixed CTA widths {io}")
    assert_close(host(h), r["ssm_state"], tol, "state")
    np.testing.assert_array_equal(host(cs), r["conv_state"])


@pytest.mark.parametrize("name", ["f32", "bf16"])
def test_scan_prefill_continues_state(name):
    d = SMALL[name]
    io, tol = _io(d.io)
    seed = 23
    w = synth.scan_weights(d, seed)
    u = synth.scan_inputs(d, seed)
    layer = ScanLayer(w, d.d_model, io)
    L1 = 2    # shorter than the conv window: the new conv state mixes old and new inputs
    Ma, h, cs = layer.prefill(to_device(u[:, :L1], io))
    Mb, h, cs = layer.prefill(to_device(u[:, L1:], io), h, cs)
    r = ref.scan_prefill_ref(u, w)
    assert_close(np.concatenate([host(Ma), host(Mb)], axis=1), r["M"], tol, f"chunked {name}")
    assert_close(host(h), r["ssm_state"], tol, "state")
    np.testing.assert_array_equal(host(cs), r["conv_state"])


@pytest.mark.parametrize("name", ["f32", "bf16"])
def test_decode_steps_equal_oracle_prefill(name):
    d = SMALL[name]
    io, tol = _io(d.io)
    seed = 24
    w = synth.scan_weights(d, seed)
    u = synth.scan_inputs(d, seed)
    L0 = d.seqlen - 6
    layer = ScanLayer(w, d.d_model, io)
    _, h, cs = layer.prefill(to_device(u[:, :L0], io))
    r = ref.scan_prefill_ref(u, w)
    for i in range(L0, d.seqlen):
        m = layer.step(to_device(np.ascontiguousarray(u[:, i]), io), h, cs)
        assert_close(host(m), r["M"][:, i], tol, f"step {i}")
    assert_close(host(h), r["ssm_state"], tol, "state after steps")
    np.testing.assert_array_equal(host(cs), r["conv_state"])


@pytest.mark.parametrize("B", [1, 5, 64, 65, 130])
def test_decode_step_batches(B):
    """bf16 decode steps at batches on both sides of 64 sequences (one kernel
    over all slices up to 64; three kernels with sequence groups beyond):
    every step's readout and the final state against the oracle's prefill
    over the same tokens."""
    d = synth.Dims(B, 12, 128, 256, 16, 4, 16, synth.BF16)
    seed = 26 + B
    w = synth.scan_weights(d, seed)
    u = synth.scan_inputs(d, seed)
    L0 = 8
    layer = ScanLayer(w, d.d_model, abi.BF16)
    _, h, cs = layer.prefill(to_device(u[:, :L0], abi.BF16))
    r = ref.scan_prefill_ref(u, w)
    for i in range(L0, d.seqlen):
        m = layer.step(to_device(np.ascontiguousarray(u[:, i]), abi.BF16), h, cs)
        assert_close(host(m), r["M"][:, i], TOL_BF16, f"B={B} step {i}")
    assert_close(host(h), r["ssm_state"], TOL_BF16, f"B={B} state after steps")
    np.testing.assert_array_equal(host(cs), r["conv_state"])


def test_decode_state_save_restore_is_bit_identical():
    d = SMALL["bf16"]
    seed = 25
    w = synth.scan_weights(d, seed)
    u = synth.scan_inputs(d, seed)
    layer = ScanLayer(w, d.d_model, abi.BF16)
    _, h, cs = layer.prefill(to_device(u[:, :50], abi.BF16))
    h0, cs0 = h.clone(), cs.clone()
    outs_a = [layer.step(to_device(np.ascontiguousarray(u[:, i]), abi.BF16), h, cs).clone() for i in range(50, 60)]
    h.copy_(h0); cs.copy_(cs0)
    outs_b = [layer.step(to_device(np.ascontiguousarray(u[:, i]), abi.BF16), h, cs).clone() for i in range(50, 60)]
    for a, b in zip(outs_a, outs_b):
        assert torch.equal(a, b)


def test_tiny_workload_end_to_end_f32():
    """The tiny float32 workload: one Mamba scan producing M, then one GMU."""
    d, seed = synth.workload("tiny_f32")
    w = synth.scan_weights(d, seed)
    gw = synth.gmu_weights(d, seed)
    u = synth.scan_inputs(d, seed)
    X = synth.gmu_inputs(d, seed)
    layer = ScanLayer(w, d.d_model, abi.F32)
    gmu = GMULayer(gw["W1"], gw["W2"], abi.F32)
    M, _, _ = layer.prefill(to_device(u, abi.F32))
    Y = gmu.forward(to_device(X, abi.F32), M.reshape(-1, d.d_inner))
    r = ref.scan_prefill_ref(u, w)
    Yr, _, _ = ref.gmu_ref(X, r["M"].reshape(-1, d.d_inner), gw["W1"], gw["W2"])
    assert_close(host(M), r["M"], TOL_F32, "tiny M")
    assert_close(host(Y), Yr, TOL_F32, "tiny Y")


# ------------------------------------------------------------------ full size

def test_prefill_b1_l2048_full_size():
    """The benchmarked workload at full size: scan M in full, GMU rows sampled."""
    d, seed = synth.workload("prefill_b1_l2048")
    w = synth.scan_weights(d, seed)
    gw = synth.gmu_weights(d, seed)
    u = synth.scan_inputs(d, seed)
    X = synth.gmu_inputs(d, seed)
    layer = ScanLayer(w, d.d_model, abi.BF16)
    gmu = GMULayer(gw["W1"], gw["W2"], abi.BF16)
    M, h, _ = layer.prefill(to_device(u, abi.BF16))
    Xd = to_device(X, abi.BF16)
    Y = gmu.forward(Xd, M.reshape(-1, d.d_inner))
    r = ref.scan_prefill_ref(u, w)
    assert_close(host(M), r["M"], TOL_BF16, "full-size M")
    assert_close(host(h), r["ssm_state"], TOL_BF16, "full-size h")
    rows = np.random.default_rng(0).choice(d.tokens, 48, replace=False)
    rows = np.unique(np.concatenate([rows, [0, d.tokens - 1]]))
    Yr, _, _ = ref.gmu_ref(X[rows], r["M"].reshape(-1, d.d_inner)[rows], gw["W1"], gw["W2"])
    assert_close(host(Y)[rows], Yr, TOL_BF16, "full-size Y (sampled rows)")


def test_decode_b64_full_width_steps():
    """The decode workload's batch (64 sequences, d_inner 5120): scan steps and
    GMU steps after a short prompt, every sequence checked."""
    d, seed = synth.workload("decode_b64")
    L0, steps = 24, 4
    w = synth.scan_weights(d, seed)
    gw = synth.gmu_weights(d, seed)
    u = synth.scan_inputs(d, seed, seqlen=L0 + steps)
    X = synth.gmu_inputs(d, seed, rows=d.batch * steps).reshape(steps, d.batch, d.d_model)
    layer = ScanLayer(w, d.d_model, abi.BF16)
    gmu = GMULayer(gw["W1"], gw["W2"], abi.BF16)
    _, h, cs = layer.prefill(to_device(u[:, :L0], abi.BF16))
    r = ref.scan_prefill_ref(u, w)
    for i in range(steps):
        m = layer.step(to_device(np.ascontiguousarray(u[:, L0 + i]), abi.BF16), h, cs)
        assert_close(host(m), r["M"][:, L0 + i], TOL_BF16, f"decode m step {i}")
        Y = gmu.step(to_device(X[i], abi.BF16), m, residual=True)
        Yr, _, _ = ref.gmu_ref(X[i], r["M"][:, L0 + i], gw["W1"], gw["W2"], residual=True)
        assert_close(host(Y), Yr, TOL_BF16, f"decode Y step {i}")


def test_back_to_back_calls_are_bit_identical():
    """Each entry point's kernels start while the one before them finishes
    (programmatic dependent launch) and wait for it before touching memory;
    repeated calls queued without a host sync must give the same bits."""
    d, seed = synth.workload("prefill_b1_l2048")
    w = synth.scan_weights(d, seed)
    gw = synth.gmu_weights(d, seed)
    scan = ScanLayer(w, d.d_model, abi.BF16)
    gmu = GMULayer(gw["W1"], gw["W2"], abi.BF16)
    u = to_device(synth.scan_inputs(d, seed), abi.BF16)
    X = to_device(synth.gmu_inputs(d, seed), abi.BF16)
    h, cs = scan.new_state(1)
    Ms, Ys = [], []
    for _ in range(8):
        M = torch.empty_like(u)
        Y = torch.empty_like(X)
        scan.prefill(u, h, cs, M=M, fresh=True)
        gmu.forward(X, M.view(-1, d.d_inner), residual=True, Y=Y)
        Ms.append(M)
        Ys.append(Y)
    torch.cuda.synchronize()
    for M, Y in zip(Ms[1:], Ys[1:]):
        assert torch.equal(M, Ms[0]) and torch.equal(Y, Ys[0])
    # decode: the same step from copies of one state
    B = 64
    dd = synth.Dims(B, 16, d.d_model, d.d_inner, 16, 4, d.dt_rank, synth.BF16)
    _, h0, cs0 = scan.prefill(to_device(synth.scan_inputs(dd, seed + 1), abi.BF16))
    ut = to_device(synth.scan_inputs(dd, seed + 2, seqlen=1)[:, 0].copy(), abi.BF16)
    xt = to_device(synth.gmu_inputs(dd, seed + 3, rows=B), abi.BF16)
    outs = []
    for _ in range(8):
        h1, c1 = h0.clone(), cs0.clone()
        m = scan.step(ut, h1, c1)
        outs.append((h1, c1, m, gmu.step(xt, m, residual=True)))
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert all(torch.equal(a, b) for a, b in zip(o, outs[0]))

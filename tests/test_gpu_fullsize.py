"""Full-size GPU parity for the long-prefill and cross-decoder-sharing workloads.

Outputs the oracle cannot afford in full are checked on samples it computes
exactly: the scan is independent per channel once x_proj (which mixes all
channels) is known, so sampled channels are checked over the whole sequence;
GMU rows are independent, so sampled rows are exact checks.  Every oracle
input is the seeded synthetic input, never a GPU result.
"""

import numpy as np
import pytest
import torch

from gated_memory_sharing_b200 import abi, synth
from gated_memory_sharing_b200.layers import GMULayer, ScanLayer, to_device
from oracle import sambay_ref as ref
from tests.gpu_util import TOL_BF16, assert_close, assert_close_chain, assert_layers_per_layer, host

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


def _oracle_scan_channels(u, w, chans):
    """Oracle readout M[:, :, chans] over the whole sequence, batch by batch.

    x_proj needs every channel's conv output, so the conv runs on all channels;
    dt_proj and the recurrence only on the sampled ones (their rows of W_dt, A,
    D and bias)."""
    out = []
    for b in range(u.shape[0]):
        uc, _ = ref.causal_conv1d_silu(u[b:b + 1], w["conv_w"], w["conv_b"])
        delta, Bm, Cm = ref.x_proj(uc, w["x_proj_w"], w["dt_rank"], w["d_state"])
        dt = ref.dt_softplus(delta, w["dt_proj_w"][chans], w["dt_bias"][chans])
        M, _ = ref.selective_scan(uc[:, :, chans], dt, w["A"][chans], Bm, Cm, w["D"][chans])
        out.append(M)
        del uc
    return np.concatenate(out, axis=0)


def test_long_prefill_b4_l32768():
    """Batch 4 x 32768 tokens: the scan carries its fp32 state through the whole
    sequence (sampled channels checked at every token), then one GMU layer over
    all 131072 rows (sampled rows checked)."""
    d, seed = synth.workload("long_prefill_b4_l32768")
    w = synth.scan_weights(d, seed)
    u = synth.scan_inputs(d, seed)
    layer = ScanLayer(w, d.d_model, abi.BF16)
    M, h, _ = layer.prefill(to_device(u, abi.BF16))
    torch.cuda.synchronize()
    chans = np.sort(np.random.default_rng(1).choice(d.d_inner, 24, replace=False))
    chans = np.unique(np.concatenate([chans, [0, d.d_inner - 1]]))
    Mg = host(M[:, :, torch.as_tensor(chans, device=M.device)])
    Mr = _oracle_scan_channels(u, w, chans)
    assert_close(Mg, Mr, TOL_BF16, "long prefill M (sampled channels)")
    del M
    # the GMU at this size, on a seeded memory readout
    gw = synth.gmu_weights(d, seed)
    X = synth.gmu_inputs(d, seed)
    Mx = synth.memory_input(d, seed)
    gmu = GMULayer(gw["W1"], gw["W2"], abi.BF16)
    Y = gmu.forward(to_device(X, abi.BF16), to_device(Mx, abi.BF16), residual=True)
    rows = np.unique(np.concatenate([np.random.default_rng(2).choice(d.tokens, 40, replace=False),
                                     [0, d.tokens - 1]]))
    Yr, _, _ = ref.gmu_ref(X[rows], Mx[rows], gw["W1"], gw["W2"], residual=True)
    assert_close(host(Y)[rows], Yr, TOL_BF16, "long prefill GMU (sampled rows)")


def test_sharing_slice_prefill_b2_l8192_eight_layers():
    """One scan's M feeds 8 GMU layers with distinct weights and a residual
    between layers (X <- X + GMU_l(X, M), in place)."""
    d, seed = synth.workload("sharing_b2_l8192")
    w = synth.scan_weights(d, seed)
    u = synth.scan_inputs(d, seed)
    X = synth.gmu_inputs(d, seed)
    layer = ScanLayer(w, d.d_model, abi.BF16)
    M, _, _ = layer.prefill(to_device(u, abi.BF16))
    Mflat = M.view(-1, d.d_inner)
    Xd = to_device(X, abi.BF16)
    W1s, W2s = [], []
    for l in range(synth.SHARING_LAYERS):
        gw = synth.gmu_weights(d, seed, layer=l)
        W1s.append(gw["W1"]); W2s.append(gw["W2"])
        GMULayer(gw["W1"], gw["W2"], abi.BF16).forward(Xd, Mflat, residual=True, Y=Xd)
    torch.cuda.synchronize()
    # scan: sampled channels over both full sequences
    chans = np.unique(np.concatenate([np.random.default_rng(3).choice(d.d_inner, 24, replace=False),
                                      [0, d.d_inner - 1]]))
    Mg = host(M[:, :, torch.as_tensor(chans, device=M.device)])
    assert_close(Mg, _oracle_scan_channels(u, w, chans), TOL_BF16, "sharing M (sampled channels)")
    # 8-layer chain on sampled rows whose tokens lie in the first 192 of each sequence
    L0 = 192
    r0 = ref.scan_prefill_ref(u[:, :L0], w)["M"]                  # [B, L0, Di], all channels
    rng = np.random.default_rng(4)
    toks = rng.choice(L0, 12, replace=False)
    rows = np.concatenate([toks, d.seqlen + toks])               # both sequences
    Mrows = np.concatenate([r0[0, toks], r0[1, toks]])
    Xr = ref.gmu_layers_ref(X[rows], Mrows, W1s, W2s)
    assert_close_chain(host(Xd)[rows], Xr, len(W1s), "8-layer sharing chain (sampled rows)")
    # every layer on its own at full size, on the oracle's chain state
    gmus = [GMULayer(W1s[l], W2s[l], abi.BF16) for l in range(len(W1s))]
    assert_layers_per_layer(lambda l, x, m: gmus[l].forward(x, m, residual=True), to_device(X, abi.BF16), Mflat,
                            rows, X[rows], Mrows, W1s, W2s, "8-layer sharing chain")


def test_sharing_slice_decode_b16_eight_layers():
    """Decode at batch 16: each step's m_t feeds the 8 GMU layers."""
    d, seed = synth.workload("sharing_b2_l8192")
    B, L0, steps = synth.SHARING_DECODE_BATCH, 16, 3
    dd = synth.Dims(B, L0, d.d_model, d.d_inner, d.d_state, d.d_conv, d.dt_rank, synth.BF16)
    w = synth.scan_weights(dd, seed)
    u = synth.scan_inputs(dd, seed + 1, seqlen=L0 + steps)
    X0 = synth.gmu_inputs(dd, seed + 2, rows=B * steps).reshape(steps, B, d.d_model)
    layer = ScanLayer(w, d.d_model, abi.BF16)
    gws = [synth.gmu_weights(d, seed, layer=l) for l in range(synth.SHARING_LAYERS)]
    gmus = [GMULayer(g["W1"], g["W2"], abi.BF16) for g in gws]
    _, h, cs = layer.prefill(to_device(u[:, :L0], abi.BF16))
    r = ref.scan_prefill_ref(u, w)
    for i in range(steps):
        m = layer.step(to_device(np.ascontiguousarray(u[:, L0 + i]), abi.BF16), h, cs)
        x = to_device(X0[i], abi.BF16)
        for g in gmus:
            g.step(x, m, residual=True, Y=x)
        W1s, W2s = [g["W1"] for g in gws], [g["W2"] for g in gws]
        xr = ref.gmu_layers_ref(X0[i], r["M"][:, L0 + i], W1s, W2s)
        assert_close_chain(host(x), xr, len(gws), f"decode step {i}: 8-layer chain")
        assert_layers_per_layer(lambda l, xx, mm: gmus[l].step(xx, mm, residual=True), to_device(X0[i], abi.BF16), m,
                                np.arange(B), X0[i], r["M"][:, L0 + i], W1s, W2s, f"decode step {i}")

"""GPU parity of the decode path through the C ABI.

* sambay_decode_step (the scan step and a stack of GMU layers issued as one
  chain of kernels) gives the same bits as the separate sambay_scan_step and
  gmu_step calls;
* the decode workloads over their whole stated horizons against the float64
  oracle: 64 sequences decoding 32768 tokens after a 2048-token prompt, and 16
  sequences decoding 4096 tokens through 8 GMU layers;
* the fault detector: a kernel whose bounded wait runs out reports it through
  sambay_device_status, and the device stays usable.

The long-horizon cases check two of the sequences against the oracle (the
sequences are independent, so a sequence is an exact check); the other
sequences' inputs are seeded draws made on the device, since no oracle reads
them.  Per sequence the oracle runs the decoded tokens as prompt chunks that
carry the state, which the oracle's own pins equate with token-by-token
decoding.
"""

import numpy as np
import pytest
import torch

from gated_memory_sharing_b200 import abi, synth
from gated_memory_sharing_b200.layers import DecodeChain, GMULayer, ScanLayer, to_device, workspace
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


def _dev_normal(shape, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    return torch.randn(shape, generator=g, device="cuda", dtype=torch.float32).to(torch.bfloat16)


# ------------------------------------------------------------------ chain == separate calls

@pytest.mark.parametrize("B,layers,Dm,Di,R", [
    (64, 1, 2560, 5120, 160),     # the decode workload's width
    (16, 8, 2560, 5120, 160),     # the sharing slice's decode batch and depth
    (3, 2, 128, 256, 16),         # a ragged batch on a small model
])
def test_decode_chain_equals_separate_calls(B, layers, Dm, Di, R):
    d = synth.Dims(B, 24, Dm, Di, 16, 4, R, synth.BF16)
    seed = 31 + B
    w = synth.scan_weights(d, seed)
    scan = ScanLayer(w, Dm, abi.BF16)
    gws = [synth.gmu_weights(d, seed, layer=l) for l in range(layers)]
    gmus = [GMULayer(g["W1"], g["W2"], abi.BF16) for g in gws]
    chain = DecodeChain(scan, gmus)
    _, h0, c0 = scan.prefill(to_device(synth.scan_inputs(d, seed), abi.BF16))
    ut = [to_device(np.ascontiguousarray(synth.scan_inputs(d, seed + 1 + i, seqlen=1)[:, 0]), abi.BF16)
          for i in range(3)]
    xt = [to_device(synth.gmu_inputs(d, seed + 5 + i, rows=B), abi.BF16) for i in range(3)]
    ha, ca, hb, cb = h0.clone(), c0.clone(), h0.clone(), c0.clone()
    for i in range(3):
        xa, xb = xt[i].clone(), xt[i].clone()
        ma = scan.step(ut[i], ha, ca)
        for g in gmus:
            g.step(xa, ma, residual=True, Y=xa)
        mb = chain.step(ut[i], hb, cb, xb)
        torch.cuda.synchronize()
        for a, b, what in ((ma, mb, "m_t"), (xa, xb, "X"), (ha, hb, "h"), (ca, cb, "conv state")):
            assert torch.equal(a, b), f"step {i}: {what} differs between the chain and separate calls"


# ------------------------------------------------------------------ fault detector

def test_bounded_wait_timeout_is_reported_and_device_stays_usable():
    d = synth.Dims(1, 1, 256, 512, 16, 4, 16, synth.BF16)
    rows = 64
    seed = 41
    gw = synth.gmu_weights(d, seed)
    X = synth.gmu_inputs(d, seed, rows=rows)
    M = synth.memory_input(d, seed, rows=rows)
    g = GMULayer(gw["W1"], gw["W2"], abi.BF16)
    Xd, Md = to_device(X, abi.BF16), to_device(M, abi.BF16)
    dims = g.dims(rows)
    ws = workspace(abi.gmu_step_workspace(dims, rows))
    Y = torch.empty_like(Xd)
    assert abi.sambay_device_status() == 0
    # each epilogue waits on a barrier nothing arrives at, limited to 2^16 cycles
    abi.sambay_gmu_step_stall_test(dims, rows, Xd, Md, g.W1, g.W2, None, Y, ws, 1 << 16)
    assert abi.sambay_device_status() == 5          # SAMBAY_ERR_TIMEOUT, then cleared
    assert abi.sambay_device_status() == 0
    # the context is intact: an ordinary call afterwards is correct
    Y2 = g.step(Xd, Md, residual=True)
    Yr, _, _ = ref.gmu_ref(X, M, gw["W1"], gw["W2"], residual=True)
    assert_close(host(Y2), Yr, TOL_BF16, "gmu_step after a timed-out call")
    assert abi.sambay_device_status() == 0


# ------------------------------------------------------------------ long horizons

def _oracle_decode_chunks(u_prompt, u_ring, steps, w, chunk, on_chunk):
    """The oracle's readout for `steps` decoded tokens after `u_prompt`, with the
    step-i input u_ring[:, i % ring]; on_chunk(first_step, M_chunk, h, conv) per
    chunk of tokens."""
    r = ref.scan_prefill_ref(u_prompt, w)
    h, cs = r["ssm_state"], r["conv_state"]
    ring = u_ring.shape[1]
    for s0 in range(0, steps, chunk):
        idx = np.arange(s0, min(steps, s0 + chunk)) % ring
        rr = ref.scan_prefill_ref(u_ring[:, idx], w, h, cs)
        h, cs = rr["ssm_state"], rr["conv_state"]
        on_chunk(s0, rr["M"], h, cs)


def _long_decode(workload, B, prompt, steps, n_layers, checked, ring=256, chunk=1024, y_every=64,
                 h_every=4096):
    d0, seed = synth.workload(workload)
    d = synth.Dims(B, prompt, d0.d_model, d0.d_inner, d0.d_state, d0.d_conv, d0.dt_rank, synth.BF16)
    Di, Dm = d.d_inner, d.d_model
    w = synth.scan_weights(d, seed)
    gws = [synth.gmu_weights(d, seed, layer=l) for l in range(n_layers)]
    nc = len(checked)
    ck = torch.as_tensor(checked, device="cuda")
    # the checked sequences' inputs from the seeded generator module (shared
    # with the oracle); every other sequence from seeded device draws
    u_p = synth.scan_inputs(d, seed, batch=nc, seqlen=prompt, tag="u_prompt")        # [nc, prompt, Di]
    u_r = synth.scan_inputs(d, seed, batch=nc, seqlen=ring, tag="u_ring")            # [nc, ring, Di]
    x_r = synth.gmu_inputs(d, seed, rows=nc * ring, tag="x_ring").reshape(nc, ring, Dm)
    U0 = _dev_normal((B, prompt, Di), seed + 1)
    U0[ck] = to_device(u_p, abi.BF16)
    UR = _dev_normal((ring, B, Di), seed + 2)
    UR[:, ck] = to_device(u_r, abi.BF16).transpose(0, 1)
    XR = _dev_normal((ring, B, Dm), seed + 3)
    XR[:, ck] = to_device(x_r, abi.BF16).transpose(0, 1)

    scan = ScanLayer(w, Dm, abi.BF16)
    chain = DecodeChain(scan, [GMULayer(g["W1"], g["W2"], abi.BF16) for g in gws])
    _, h, cs = scan.prefill(U0)
    del U0
    m = torch.empty(B, Di, dtype=torch.bfloat16, device="cuda")
    x = torch.empty(B, Dm, dtype=torch.bfloat16, device="cuda")
    m_hist = torch.empty(steps, nc, Di, dtype=torch.bfloat16, device="cuda")
    y_rows = list(range(y_every - 1, steps, y_every))
    y_hist = torch.empty(len(y_rows), nc, Dm, dtype=torch.bfloat16, device="cuda")
    h_snap = {}
    yi = 0
    for i in range(steps):
        x.copy_(XR[i % ring])
        chain.step(UR[i % ring], h, cs, x, m_t=m)
        m_hist[i] = m[ck]
        if yi < len(y_rows) and y_rows[yi] == i:
            y_hist[yi] = x[ck]
            yi += 1
        if (i + 1) % h_every == 0 or i + 1 == steps:
            h_snap[i + 1] = host(h[ck])
    torch.cuda.synchronize()
    assert abi.sambay_device_status() == 0
    m_hist = host(m_hist)                                      # [steps, nc, Di]
    y_hist = host(y_hist)
    worst = {"m": 0.0, "h": 0.0}
    M_or = {}

    def on_chunk(s0, Mc, hh, _cs):
        n = Mc.shape[1]
        worst["m"] = max(worst["m"], assert_close(m_hist[s0:s0 + n].transpose(1, 0, 2), Mc, TOL_BF16,
                                                  f"m_t, steps {s0}..{s0 + n - 1}"))
        if s0 + n in h_snap:
            worst["h"] = max(worst["h"], assert_close(h_snap[s0 + n], hh, TOL_BF16, f"h after {s0 + n} steps"))
        for j, i in enumerate(y_rows):
            if s0 <= i < s0 + n:
                M_or[i] = Mc[:, i - s0]

    _oracle_decode_chunks(u_p, u_r, steps, w, chunk, on_chunk)
    # the layers' output on the sampled steps (GMU rows are independent)
    X0 = np.concatenate([x_r[:, i % ring] for i in y_rows])        # [len * nc, Dm], step-major
    Mr = np.concatenate([M_or[i] for i in y_rows])
    W1s, W2s = [g["W1"] for g in gws], [g["W2"] for g in gws]
    Xr = ref.gmu_layers_ref(X0, Mr, W1s, W2s)
    what = f"X after {n_layers} GMU layer(s), sampled steps"
    if n_layers == 1:
        ey = assert_close(y_hist.reshape(-1, Dm), Xr, TOL_BF16, what)
    else:
        ey = assert_close_chain(y_hist.reshape(-1, Dm), Xr, n_layers, what)
        # each layer on its own (decode kernels, the workload's batch), on the
        # oracle's chain state of a few sampled steps
        gm = chain.gmus
        for i in y_rows[:: max(1, len(y_rows) // 4)]:
            assert_layers_per_layer(lambda l, xx, mm: gm[l].step(xx, mm, residual=True), XR[i % ring], m, checked,
                                    x_r[:, i % ring], M_or[i], W1s, W2s, f"decode step {i}")
    return worst["m"], worst["h"], ey


def test_decode_b64_prompt2048_32768_steps():
    """The decode workload over its whole stated horizon: 64 sequences, a
    2048-token prompt, then 32768 decode steps (scan step + one GMU layer with
    residual); m_t checked at every step, h every 4096 steps, the GMU output
    every 64th step, for the first and last sequence."""
    em, eh, ey = _long_decode("decode_b64", 64, 2048, synth.DECODE_STEPS["decode_b64"], 1, [0, 63])
    print(f"decode_b64 32768 steps: max rel err m_t {em:.3g}, h {eh:.3g}, Y {ey:.3g}")


def test_sharing_decode_b16_4096_steps_eight_layers():
    """The sharing slice's decode over its whole horizon: 16 sequences, 4096
    steps, each step's m_t feeding 8 GMU layers (X <- X + GMU_l(X, m_t))."""
    em, eh, ey = _long_decode("sharing_b2_l8192", synth.SHARING_DECODE_BATCH, 1024,
                              synth.DECODE_STEPS["sharing_b2_l8192"], synth.SHARING_LAYERS, [0, 15],
                              y_every=32, h_every=1024)
    print(f"sharing decode 4096 steps x 8 layers: max rel err m_t {em:.3g}, h {eh:.3g}, X {ey:.3g}")

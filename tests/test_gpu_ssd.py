"""GPU parity of the SambaY-2 memory readout (Mamba-2 SSD scan, chunked on
the tensor cores) against the float64 oracle (oracle/ssd_ref.py)."""

import numpy as np
import pytest
import torch

from gated_memory_sharing_b200 import abi, synth
from gated_memory_sharing_b200.layers import Mamba2Scan, to_device, to_device_f32
from oracle import ssd_ref
from tests.gpu_util import TOL_BF16, assert_close, host

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _status_clean():
    yield
    assert abi.sambay_device_status() == 0


def _run(d, seed, seqlen=None):
    w = synth.ssd_weights(d, seed)
    xbc, dt_raw = synth.ssd_inputs(d, seed, seqlen)
    layer = Mamba2Scan(w)
    M, h, cs = layer.prefill(to_device(xbc, abi.BF16), to_device(dt_raw, abi.BF16))
    torch.cuda.synchronize()
    return w, xbc, dt_raw, layer, M, h, cs


@pytest.mark.parametrize("B,L,H,N", [
    (2, 77, 2, 64),       # two partial chunks, ragged tail
    (1, 64, 3, 128),      # exactly one chunk
    (3, 200, 2, 128),     # several chunks, a 8-token tail
    (1, 5, 4, 64),        # shorter than a chunk, one token past the conv window
])
def test_ssd_prefill_matches_oracle(B, L, H, N):
    d = synth.SsdDims(B, L, H, 64, N)
    w, xbc, dt_raw, layer, M, h, cs = _run(d, 40 + L + N)
    r = ssd_ref.mamba2_scan_ref(xbc, dt_raw, w)
    assert_close(host(M), r["M"], TOL_BF16, f"M B{B} L{L} H{H} N{N}")
    assert_close(host(h), r["ssm_state"], TOL_BF16, "final state")
    np.testing.assert_array_equal(host(cs), r["conv_state"])


def test_ssd_prefill_continues_state():
    """A prompt in two calls (the second from the first's states, its first
    chunk shorter than the conv window) equals the whole prompt."""
    d = synth.SsdDims(2, 150, 2, 64, 128)
    seed = 51
    w = synth.ssd_weights(d, seed)
    xbc, dt_raw = synth.ssd_inputs(d, seed)
    layer = Mamba2Scan(w)
    L1 = 3
    Ma, h, cs = layer.prefill(to_device(xbc[:, :L1], abi.BF16), to_device(dt_raw[:, :L1], abi.BF16))
    Mb, h, cs = layer.prefill(to_device(xbc[:, L1:], abi.BF16), to_device(dt_raw[:, L1:], abi.BF16), h, cs)
    torch.cuda.synchronize()
    r = ssd_ref.mamba2_scan_ref(xbc, dt_raw, w)
    assert_close(np.concatenate([host(Ma), host(Mb)], axis=1), r["M"], TOL_BF16, "chunked prompt M")
    assert_close(host(h), r["ssm_state"], TOL_BF16, "state")
    np.testing.assert_array_equal(host(cs), r["conv_state"])


def test_ssd_prefill_from_given_state():
    d = synth.SsdDims(2, 90, 3, 64, 64)
    seed = 52
    w = synth.ssd_weights(d, seed)
    xbc, dt_raw = synth.ssd_inputs(d, seed)
    rng = np.random.default_rng(0)
    h0 = rng.standard_normal((2, 3, 64, 64)).astype(np.float32)
    cs0 = synth.round_bf16(rng.standard_normal((2, d.channels, 4)).astype(np.float32))
    layer = Mamba2Scan(w)
    h, cs = to_device_f32(h0), to_device(cs0, abi.BF16)
    M, h, cs = layer.prefill(to_device(xbc, abi.BF16), to_device(dt_raw, abi.BF16), h, cs, fresh=False)
    torch.cuda.synchronize()
    r = ssd_ref.mamba2_scan_ref(xbc, dt_raw, w, h0, cs0)
    assert_close(host(M), r["M"], TOL_BF16, "M from a given state")
    assert_close(host(h), r["ssm_state"], TOL_BF16, "state")
    np.testing.assert_array_equal(host(cs), r["conv_state"])


def test_ssd_prefill_full_size_sampled_heads():
    """The SambaY-2 variant of the prefill workload (batch 1, 2048 tokens,
    80 heads of 64, d_state 128): every token of three heads against the
    oracle (heads are independent given the shared B, C)."""
    d, seed = synth.SSD_WORKLOAD, synth.SSD_WORKLOAD_SEED
    w, xbc, dt_raw, layer, M, h, cs = _run(d, seed)
    P, N, H = d.headdim, d.d_state, d.nheads
    heads = [0, 37, H - 1]
    cols = np.concatenate([np.arange(k * P, (k + 1) * P) for k in heads]
                          + [np.arange(H * P, H * P + 2 * N)])
    ws = dict(w)
    ws["conv_w"], ws["conv_b"] = w["conv_w"][cols], w["conv_b"][cols]
    for k in ("dt_bias", "A", "D"):
        ws[k] = w[k][heads]
    r = ssd_ref.mamba2_scan_ref(xbc[..., cols], dt_raw[..., heads], ws)
    Mg = host(M).reshape(1, d.seqlen, H, P)[:, :, heads].reshape(1, d.seqlen, -1)
    assert_close(Mg, r["M"], TOL_BF16, "full-size M (sampled heads)")
    assert_close(host(h)[:, heads], r["ssm_state"], TOL_BF16, "full-size state (sampled heads)")


def test_ssd_prefill_repeatable():
    d = synth.SsdDims(1, 130, 2, 64, 128)
    w, xbc, dt_raw, layer, M, h, cs = _run(d, 53)
    M2, h2, _ = layer.prefill(to_device(xbc, abi.BF16), to_device(dt_raw, abi.BF16))
    torch.cuda.synchronize()
    assert torch.equal(M, M2) and torch.equal(h, h2)


@pytest.mark.parametrize("B,H,N", [(3, 2, 128), (2, 3, 64)])
def test_ssd_decode_steps_equal_oracle_prefill(B, H, N):
    """Decode steps after a prompt (states updated in place) against the
    oracle's readout of the whole token sequence."""
    d = synth.SsdDims(B, 40, H, 64, N)
    seed = 60 + B + N
    w = synth.ssd_weights(d, seed)
    xbc, dt_raw = synth.ssd_inputs(d, seed)
    layer = Mamba2Scan(w)
    L0 = 33
    _, h, cs = layer.prefill(to_device(xbc[:, :L0], abi.BF16), to_device(dt_raw[:, :L0], abi.BF16))
    r = ssd_ref.mamba2_scan_ref(xbc, dt_raw, w)
    for t in range(L0, d.seqlen):
        m = layer.step(to_device(np.ascontiguousarray(xbc[:, t]), abi.BF16),
                       to_device(np.ascontiguousarray(dt_raw[:, t]), abi.BF16), h, cs)
        torch.cuda.synchronize()
        assert_close(host(m), r["M"][:, t], TOL_BF16, f"step {t}")
    assert_close(host(h), r["ssm_state"], TOL_BF16, "state after steps")
    np.testing.assert_array_equal(host(cs), r["conv_state"])


def test_ssd_decode_b64_full_width_sampled_heads():
    """64 sequences at 80 heads of 64, d_state 128: a short prompt, then decode
    steps; three heads of every sequence against the oracle."""
    d = synth.SsdDims(64, 20, 80, 64, 128)
    seed = 70
    w = synth.ssd_weights(d, seed)
    xbc, dt_raw = synth.ssd_inputs(d, seed)
    layer = Mamba2Scan(w)
    L0 = 16
    _, h, cs = layer.prefill(to_device(xbc[:, :L0], abi.BF16), to_device(dt_raw[:, :L0], abi.BF16))
    ms = []
    for t in range(L0, d.seqlen):
        ms.append(host(layer.step(to_device(np.ascontiguousarray(xbc[:, t]), abi.BF16),
                                  to_device(np.ascontiguousarray(dt_raw[:, t]), abi.BF16), h, cs)))
    torch.cuda.synchronize()
    P, N, H = d.headdim, d.d_state, d.nheads
    heads = [1, 40, H - 1]
    cols = np.concatenate([np.arange(k * P, (k + 1) * P) for k in heads] + [np.arange(H * P, H * P + 2 * N)])
    ws = dict(w)
    ws["conv_w"], ws["conv_b"] = w["conv_w"][cols], w["conv_b"][cols]
    for k in ("dt_bias", "A", "D"):
        ws[k] = w[k][heads]
    r = ssd_ref.mamba2_scan_ref(xbc[..., cols], dt_raw[..., heads], ws)
    got = np.stack(ms, axis=1).reshape(64, d.seqlen - L0, H, P)[:, :, heads].reshape(64, d.seqlen - L0, -1)
    assert_close(got, r["M"][:, L0:], TOL_BF16, "decode m_t (sampled heads)")
    assert_close(host(h)[:, heads], r["ssm_state"], TOL_BF16, "state (sampled heads)")

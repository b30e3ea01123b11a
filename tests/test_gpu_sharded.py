"""GPU parity of the channel-sharded prefill's calls (sambay_scan_prefill_xproj
/ _finish, gmu_forward_partial / gmu_finish).

One GPU here, so the ranks of a sharded run go one after another in this
process, with the all-reduce done as a device-side sum of the ranks' buffers
between the phases (no kernel waits on another rank).
"""

import numpy as np
import pytest
import torch

from gated_memory_sharing_b200 import abi, sharded, synth
from gated_memory_sharing_b200.layers import ScanLayer, to_device
from oracle import sambay_ref as ref
from tests.gpu_util import TOL_BF16, TOL_F32, assert_close, host

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _status_clean():
    yield
    assert abi.sambay_device_status() == 0


def _io(io):
    return (abi.BF16, TOL_BF16) if io == synth.BF16 else (abi.F32, TOL_F32)


def _run_sharded(d, w, gw, u, X, world, residual=True):
    """All ranks' phases in order; returns (M [B, L, Di], Y, h, cs) assembled."""
    io, _ = _io(d.io)
    rows = d.batch * d.seqlen
    ranks = []
    for k in range(world):
        lo, hi = sharded.shard_bounds(d.d_inner, world, k)
        ops = sharded.DeviceOps(sharded.shard_scan_weights(w, lo, hi),
                                *sharded.shard_gmu_weights(gw["W1"], gw["W2"], lo, hi), d.d_model, io)
        uk = to_device(np.ascontiguousarray(u[..., lo:hi]), io)
        h, cs = ops.new_state(d.batch)
        ranks.append(dict(ops=ops, u=uk, h=h, cs=cs, M=torch.empty_like(uk), xdbl=ops.xdbl_buffer(rows),
                          yp=ops.y_buffer(rows)))
    Xd = to_device(X, io)
    for r in ranks:
        r["ops"].xproj(r["u"], r["cs"], True, r["xdbl"])
    xsum = sum(r["xdbl"] for r in ranks)                      # the all-reduce
    for r in ranks:
        r["ops"].finish(r["u"], xsum, r["M"], r["h"], r["cs"], True)
        r["ops"].gmu_partial(Xd, r["M"].reshape(rows, -1), r["yp"])
    ysum = sum(r["yp"] for r in ranks)                        # the second all-reduce
    Y = torch.empty_like(Xd)
    ranks[0]["ops"].gmu_finish(ysum, Xd if residual else None, Y)
    torch.cuda.synchronize()
    cat = lambda key: torch.cat([r[key] for r in ranks], dim=1 if key != "M" else 2)
    return cat("M"), Y, cat("h"), cat("cs")


@pytest.mark.parametrize("io", [synth.BF16, synth.F32])
def test_one_shard_phases_equal_the_unsharded_prefill_bitwise(io):
    """With one shard, x_proj's split sums land in xdbl and the finish phase
    takes them as its single split: the same arithmetic in the same order."""
    d = synth.Dims(2, 150, 128, 320, 16, 4, 72, io) if io == synth.BF16 else synth.Dims(2, 77, 64, 128, 16, 4, 8, io)
    w = synth.scan_weights(d, 31)
    u = synth.scan_inputs(d, 31)
    aio, _ = _io(io)
    ud = to_device(u, aio)
    layer = ScanLayer(w, d.d_model, aio)
    M0, h0, cs0 = layer.prefill(ud)
    ops = sharded.DeviceOps(w, np.zeros((d.d_inner, d.d_model), np.float32),
                            np.zeros((d.d_inner, d.d_model), np.float32), d.d_model, aio)
    h, cs = ops.new_state(d.batch)
    xdbl = ops.xdbl_buffer(d.batch * d.seqlen)
    M = torch.empty_like(ud)
    ops.xproj(ud, cs, True, xdbl)
    ops.finish(ud, xdbl, M, h, cs, True)
    torch.cuda.synchronize()
    assert torch.equal(M, M0) and torch.equal(h, h0) and torch.equal(cs, cs0)


@pytest.mark.parametrize("io,world", [(synth.BF16, 2), (synth.BF16, 4), (synth.F32, 2)])
def test_sharded_prefill_matches_oracle(io, world):
    d = synth.Dims(2, 100, 128, 256 * world // 2, 16, 4, 16, io)
    w = synth.scan_weights(d, 40 + world)
    gw = synth.gmu_weights(d, 41)
    u = synth.scan_inputs(d, 42)
    X = synth.gmu_inputs(d, 43, rows=d.batch * d.seqlen)
    M, Y, h, cs = _run_sharded(d, w, gw, u, X, world)
    r = ref.scan_prefill_ref(u, w)
    Yr, _, _ = ref.gmu_ref(X, r["M"].reshape(d.batch * d.seqlen, -1), gw["W1"], gw["W2"], residual=True)
    _, tol = _io(io)
    assert_close(host(M), r["M"], tol, f"sharded M world {world}")
    assert_close(host(h), r["ssm_state"], tol, "sharded state")
    np.testing.assert_array_equal(host(cs), r["conv_state"])
    assert_close(host(Y), Yr, tol, f"sharded Y world {world}")


def test_sharded_full_width_equals_unsharded():
    """2048 tokens at d_inner 5120 in two shards of 2560 against the unsharded
    prefill + GMU on the same GPU (sharding changes only the order of the
    x_proj and out-projection sums)."""
    d, seed = synth.WORKLOADS["prefill_b1_l2048"], 1000
    w = synth.scan_weights(d, seed)
    gw = synth.gmu_weights(d, seed)
    u = synth.scan_inputs(d, seed)
    X = synth.gmu_inputs(d, seed, rows=d.seqlen)
    M, Y, h, _ = _run_sharded(d, w, gw, u, X, 2)
    from gated_memory_sharing_b200.layers import GMULayer
    layer = ScanLayer(w, d.d_model, abi.BF16)
    M0, h0, _ = layer.prefill(to_device(u, abi.BF16))
    Y0 = GMULayer(gw["W1"], gw["W2"], abi.BF16).forward(to_device(X, abi.BF16), M0.reshape(d.seqlen, -1),
                                                        residual=True)
    torch.cuda.synchronize()
    assert_close(host(M), host(M0), TOL_BF16, "sharded vs unsharded M")
    assert_close(host(h), host(h0), TOL_BF16, "sharded vs unsharded state")
    assert_close(host(Y), host(Y0), TOL_BF16, "sharded vs unsharded Y")


def test_gmu_finish_without_residual_and_argument_errors():
    d = synth.Dims(64, 1, 128, 256, 16, 4, 16, synth.BF16)
    rows = 64
    ysum = torch.randn(rows, d.d_model, device="cuda")
    Y = torch.empty(rows, d.d_model, dtype=torch.bfloat16, device="cuda")
    dims = abi.make_dims(rows, 1, d.d_model, d.d_inner, 16, 4, 4, abi.BF16)
    abi.gmu_finish(dims, rows, ysum, None, Y)
    torch.cuda.synchronize()
    assert torch.equal(Y, ysum.to(torch.bfloat16))
    with pytest.raises(abi.SambayError):
        abi.gmu_finish(dims, 0, ysum, None, Y)

"""The channel-sharded prefill (gated_memory_sharing_b200.sharded) on the host:
world size 2 over gloo, no GPU.

ShardedPrefill runs with stand-in compute built from the float64 oracle on
each rank's shard (conv, x_proj partial sums, then after the all-reduce the
dt projection and the scan; the GMU's partial out projection, then after the
second all-reduce the residual).  The concatenated M shards and the
replicated Y must equal the unsharded oracle: this pins the shard bounds, the
weight slicing, where the two all-reduces sit and what they sum.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from gated_memory_sharing_b200 import sharded, synth

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """A shard's compute on the CPU from the oracle's steps (test stand-in)."""

    def __init__(self, w_shard, W1s, W2s):
        self.w, self.W1, self.W2 = w_shard, W1s, W2s
        self.uc = None

    def new_state(self, batch):
        Di, N = self.w["A"].shape
        return (torch.zeros(batch, Di, N, dtype=torch.float64),
                torch.zeros(batch, Di, self.w["conv_w"].shape[1], dtype=torch.float64))

    def xdbl_buffer(self, rows):
        return torch.empty(rows, self.w["dt_rank"] + 2 * self.w["A"].shape[1], dtype=torch.float64)

    def y_buffer(self, rows):
        return torch.empty(rows, self.W1.shape[1], dtype=torch.float64)

    def xproj(self, u, conv_state, fresh, xdbl, stream=None):
        from oracle import sambay_ref as ref
        uc, self.new_cs = ref.causal_conv1d_silu(u.numpy(), self.w["conv_w"], self.w["conv_b"],
                                                 None if fresh else conv_state.numpy())
        self.uc = uc
        delta, Bm, Cm = ref.x_proj(uc, self.w["x_proj_w"], self.w["dt_rank"], self.w["A"].shape[1])
        xdbl.copy_(torch.from_numpy(np.concatenate([delta, Bm, Cm], axis=-1).reshape(xdbl.shape)))

    def finish(self, u, xdbl, M, ssm_state, conv_state, fresh, stream=None):
        from oracle import sambay_ref as ref
        B, L, _ = u.shape
        R, N = self.w["dt_rank"], self.w["A"].shape[1]
        x = xdbl.numpy().reshape(B, L, -1)
        dt = ref.dt_softplus(x[..., :R], self.w["dt_proj_w"], self.w["dt_bias"])
        y, h = ref.selective_scan(self.uc, dt, self.w["A"], x[..., R:R + N], x[..., R + N:], self.w["D"],
                                  None if fresh else ssm_state.numpy())
        M.copy_(torch.from_numpy(y))
        ssm_state.copy_(torch.from_numpy(h))
        conv_state.copy_(torch.from_numpy(self.new_cs))

    def gmu_partial(self, X, M2, Y_part, stream=None):
        from oracle import sambay_ref as ref
        Y, _, _ = ref.gmu_ref(X.numpy(), M2.numpy(), self.W1, self.W2, residual=False)
        Y_part.copy_(torch.from_numpy(Y))

    def gmu_finish(self, Y_sum, residual, Y, stream=None):
        Y.copy_(Y_sum if residual is None else Y_sum + residual)


def _problem():
    d = synth.Dims(2, 37, 64, 256, 16, 4, 8, synth.F32)
    w = synth.scan_weights(d, 5)
    gw = synth.gmu_weights(d, 6)
    u = synth.scan_inputs(d, 7).astype(np.float64)
    X = np.random.default_rng(8).standard_normal((d.batch * d.seqlen, d.d_model))
    return d, w, gw, u, X


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        d, w, gw, u, X = _problem()
        lo, hi = sharded.shard_bounds(d.d_inner, world, rank)
        ops = OracleOps(sharded.shard_scan_weights(w, lo, hi), *sharded.shard_gmu_weights(gw["W1"], gw["W2"], lo, hi))
        run = sharded.ShardedPrefill(ops, all_reduce=dist.all_reduce)
        M, Y, h, cs = run.forward(torch.from_numpy(np.ascontiguousarray(u[..., lo:hi])), torch.from_numpy(X))
        out[rank] = (lo, hi, M.numpy(), Y.numpy(), h.numpy(), cs.numpy())
    finally:
        dist.destroy_process_group()


def test_two_rank_sharded_prefill_equals_unsharded_oracle():
    from oracle import sambay_ref as ref
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    d, w, gw, u, X = _problem()
    r = ref.scan_prefill_ref(u, w)
    Yr, _, _ = ref.gmu_ref(X, r["M"].reshape(d.batch * d.seqlen, -1), gw["W1"], gw["W2"], residual=True)
    M = np.concatenate([res[k][2] for k in range(world)], axis=-1)
    assert [res[k][:2] for k in range(world)] == [(0, 128), (128, 256)]
    np.testing.assert_allclose(M, r["M"], rtol=1e-10, atol=1e-12)
    for k in range(world):
        np.testing.assert_allclose(res[k][3], Yr, rtol=1e-10, atol=1e-10)   # Y is replicated
        lo, hi = res[k][:2]
        np.testing.assert_allclose(res[k][4], r["ssm_state"][:, lo:hi], rtol=1e-10, atol=1e-12)
        np.testing.assert_array_equal(res[k][5], r["conv_state"][:, lo:hi])


def test_shard_bounds():
    assert sharded.shard_bounds(5120, 4, 3) == (3840, 5120)
    assert sharded.shard_bounds(5120, 1, 0) == (0, 5120)
    with pytest.raises(ValueError):
        sharded.shard_bounds(5120, 3, 0)          # 1706.67 channels
    with pytest.raises(ValueError):
        sharded.shard_bounds(128, 4, 0)           # 32 < 64
    with pytest.raises(ValueError):
        sharded.shard_bounds(5120, 2, 2)


def test_shard_weights_tile_the_full_weights():
    d, w, gw, _, _ = _problem()
    parts = [sharded.shard_scan_weights(w, *sharded.shard_bounds(d.d_inner, 4, k)) for k in range(4)]
    for key in ("conv_w", "conv_b", "dt_proj_w", "dt_bias", "A", "D"):
        np.testing.assert_array_equal(np.concatenate([p[key] for p in parts], axis=0), w[key])
    np.testing.assert_array_equal(np.concatenate([p["x_proj_w"] for p in parts], axis=1), w["x_proj_w"])
    W1s, W2s = zip(*(sharded.shard_gmu_weights(gw["W1"], gw["W2"], *sharded.shard_bounds(d.d_inner, 4, k))
                     for k in range(4)))
    np.testing.assert_array_equal(np.concatenate(W1s), gw["W1"])
    np.testing.assert_array_equal(np.concatenate(W2s), gw["W2"])

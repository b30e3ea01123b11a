"""Channel-sharded prefill of the scan and the GMU: one d_inner shard per rank.

The selective scan is independent per channel except for x_proj, whose
[delta | B | C] are sums over all channels (Gu & Dao 2023, "Mamba", section
3.2, the selection projections s_Delta, s_B, s_C), and the GMU's output
projection Y = H W2, a sum over the channels of H ("Decoder-Hybrid-Decoder
Architecture for Efficient Reasoning with Long Generation", Paper-Notes page,
方法详解 > 关键设计: the GMU's gate and product are element-wise per channel).
So each rank keeps d_inner / world channels of the scan (its slice of u, M,
the conv and SSM states, and the weights of those channels), the matching
rows of W1 and of W2, and two all-reduces carry the cross-channel sums:

  1. xdbl [B*L, R + 2N] float32, after this rank's x_proj partial sums;
  2. Y [B*L, d_model] float32, after this rank's out-projection partial.

X (the GMU input) is replicated; the residual is added once, after the sum.

`ShardedPrefill` holds the order of those steps; `DeviceOps` is its compute,
the C ABI calls of this package on the rank's GPU.  The all-reduce is
`torch.distributed.all_reduce` on the rank's process group by default (NCCL
between GPUs).
"""

from __future__ import annotations

import contextlib

import numpy as np
import torch

from . import abi
from .layers import GMULayer, ScanLayer


def shard_bounds(d_inner: int, world: int, rank: int, align: int = 64) -> tuple[int, int]:
    """Channels [lo, hi) of `rank`: equal contiguous shards whose width is a
    multiple of `align` (the bfloat16 kernels' d_inner granularity)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    if d_inner % (world * align) != 0:
        raise ValueError(f"d_inner {d_inner} does not split into {world} shards of a multiple of {align}")
    width = d_inner // world
    return rank * width, (rank + 1) * width


def shard_scan_weights(w: dict, lo: int, hi: int) -> dict:
    """The scan weights of channels [lo, hi): per-channel rows of the conv,
    dt_proj, A and D; the matching columns of W_x [R + 2N, d_inner]."""
    return {
        "conv_w": np.ascontiguousarray(w["conv_w"][lo:hi]),
        "conv_b": np.ascontiguousarray(w["conv_b"][lo:hi]),
        "x_proj_w": np.ascontiguousarray(w["x_proj_w"][:, lo:hi]),
        "dt_proj_w": np.ascontiguousarray(w["dt_proj_w"][lo:hi]),
        "dt_bias": np.ascontiguousarray(w["dt_bias"][lo:hi]),
        "A": np.ascontiguousarray(w["A"][lo:hi]),
        "D": np.ascontiguousarray(w["D"][lo:hi]),
        "dt_rank": w["dt_rank"],
    }


def shard_gmu_weights(W1: np.ndarray, W2: np.ndarray, lo: int, hi: int):
    """Rows [lo, hi) of W1 [d_inner, d_model] and of W2 [d_inner, d_model]."""
    return np.ascontiguousarray(W1[lo:hi]), np.ascontiguousarray(W2[lo:hi])


class DeviceOps:
    """One shard's compute on its GPU, through the C ABI."""

    def __init__(self, w_shard: dict, W1_shard, W2_shard, d_model: int, io: int, device="cuda"):
        self.scan = ScanLayer(w_shard, d_model, io, device)
        self.gmu = GMULayer(W1_shard, W2_shard, io, device)
        self.io = io
        self.device = device

    def new_state(self, batch: int):
        return self.scan.new_state(batch)

    def xdbl_buffer(self, rows: int) -> torch.Tensor:
        return torch.empty(rows, self.scan.dt_rank + 2 * self.scan.d_state, dtype=torch.float32,
                           device=self.device)

    def y_buffer(self, rows: int) -> torch.Tensor:
        return torch.empty(rows, self.gmu.d_model, dtype=torch.float32, device=self.device)

    def _scan_ws(self, B: int, L: int):
        d = self.scan.dims(B, L)
        return d, self.scan._workspace(("sharded", B, L), abi.sambay_scan_prefill_workspace(d))

    def xproj(self, u, conv_state, fresh: bool, xdbl, stream=None):
        B, L, _ = u.shape
        d, ws = self._scan_ws(B, L)
        abi.sambay_scan_prefill_xproj(self.scan.abi_w, d, u, conv_state, fresh, xdbl, ws, stream)

    def finish(self, u, xdbl, M, ssm_state, conv_state, fresh: bool, stream=None):
        B, L, _ = u.shape
        d, ws = self._scan_ws(B, L)
        abi.sambay_scan_prefill_finish(self.scan.abi_w, d, u, xdbl, M, ssm_state, conv_state, fresh, ws,
                                       stream)

    def gmu_partial(self, X, M2, Y_part, stream=None):
        rows = X.shape[0]
        d = self.gmu.dims(rows)
        ws = self.gmu._workspace(("partial", rows), abi.gmu_forward_workspace(d, rows))
        abi.gmu_forward_partial(d, rows, X, M2, self.gmu.W1, self.gmu.W2, Y_part, ws, stream)

    def gmu_finish(self, Y_sum, residual, Y, stream=None):
        rows = Y.shape[0]
        abi.gmu_finish(self.gmu.dims(rows), rows, Y_sum, residual, Y, stream)


def _on(stream):
    """Make `stream` torch's current stream for the block (no-op for None)."""
    return torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()


def _dist_all_reduce(t: torch.Tensor) -> None:
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t)


class ShardedPrefill:
    """One rank's part of the channel-sharded prefill: M for the rank's
    channels and the full GMU output Y.

    ops: the shard's compute (DeviceOps); all_reduce: in-place sum of a
    tensor over the ranks (every rank calls it in the same order)."""

    def __init__(self, ops, all_reduce=_dist_all_reduce):
        self.ops = ops
        self.all_reduce = all_reduce

    def forward(self, u, X, ssm_state=None, conv_state=None, fresh=None, residual=True, M=None, Y=None,
                stream=None):
        """u [B, L, Di_shard] (this rank's channels), X [B*L, d_model]
        (replicated) -> M [B, L, Di_shard], Y [B*L, d_model].  States are
        this rank's channels, updated in place.  With `stream` given, the
        all-reduces are issued on it too, between the calls they join."""
        B, L, _ = u.shape
        rows = B * L
        if fresh is None:
            fresh = ssm_state is None
        if ssm_state is None:
            ssm_state, conv_state = self.ops.new_state(B)
        if M is None:
            M = torch.empty_like(u)
        if Y is None:
            Y = torch.empty_like(X)
        xdbl = self.ops.xdbl_buffer(rows)
        self.ops.xproj(u, conv_state, fresh, xdbl, stream)
        with _on(stream):
            self.all_reduce(xdbl)                   # [delta | B | C] summed over all channels
        self.ops.finish(u, xdbl, M, ssm_state, conv_state, fresh, stream)
        y_part = self.ops.y_buffer(rows)
        self.ops.gmu_partial(X, M.reshape(rows, -1), y_part, stream)
        with _on(stream):
            self.all_reduce(y_part)                 # H W2 summed over all channels
        self.ops.gmu_finish(y_part, X if residual else None, Y, stream)
        return M, Y, ssm_state, conv_state

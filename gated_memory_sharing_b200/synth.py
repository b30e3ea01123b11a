"""Seeded synthetic inputs shared by the oracle tests, the GPU parity tests and
the benchmark.

This module holds no arithmetic of the method: only the workload shapes,
seeded random draws with the stated distributions, and rounding of the draws
to the I/O storage format (bfloat16 round-to-nearest-even, or float32).

Recipe (one NumPy ``Generator(PCG64)`` per tensor name, seeded from
``(seed, crc32(name))``; ``seed`` defaults to ``1000 + workload id``):

    X, u             ~ N(0, 1)
    conv_w [Di, K]   ~ N(0, 1/K)          conv_b ~ U(-1/sqrt(K), 1/sqrt(K))
    x_proj_w         ~ N(0, 1/Di)         dt_proj_w ~ N(0, 1/R)
    W1 [Di, Dm]      ~ N(0, 1/Dm)         W2 [Di, Dm] ~ N(0, 1/Di)
    A [Di, N]        = -exp(U[log 1, log 16])                  (float32)
    dt_bias [Di]     = softplus^-1(dt0), dt0 = exp(U[log 1e-3, log 1e-1])
                       so that softplus(dt_bias) lies in [1e-3, 1e-1] (float32)
    D [Di]           ~ U(0.5, 1.5)                              (float32)
    M (GMU-only)     ~ N(0, 1)
    Mamba block      W_in, W_z [Di, Dm] ~ N(0, 1/Dm), W_out [Di, Dm] ~ N(0, 1/Di)
    SwiGLU MLP       W_g, W_u [Dff, Dm] ~ N(0, 1/Dm)

Tensors of the I/O type are rounded to it once here; the same rounded values
feed both the oracle (widened to float64) and the CUDA path.
"""

from __future__ import annotations

import dataclasses
import zlib

import numpy as np

F32 = "f32"
BF16 = "bf16"


@dataclasses.dataclass(frozen=True)
class Dims:
    batch: int
    seqlen: int
    d_model: int
    d_inner: int
    d_state: int = 16
    d_conv: int = 4
    dt_rank: int = 160
    io: str = BF16

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen


# The five workloads (name -> dims).  Decode workloads list the prefill dims;
# the decode step count is separate.
WORKLOADS = {
    "tiny_f32": Dims(1, 64, 64, 128, 16, 4, 4, F32),
    "prefill_b1_l2048": Dims(1, 2048, 2560, 5120, 16, 4, 160, BF16),
    "decode_b64": Dims(64, 2048, 2560, 5120, 16, 4, 160, BF16),
    "long_prefill_b4_l32768": Dims(4, 32768, 2560, 5120, 16, 4, 160, BF16),
    "sharing_b2_l8192": Dims(2, 8192, 2560, 5120, 16, 4, 160, BF16),
}
WORKLOAD_IDS = {name: i for i, name in enumerate(WORKLOADS)}
DECODE_STEPS = {"decode_b64": 32768, "sharing_b2_l8192": 4096}
SHARING_LAYERS = 8
# cross-attention beside the GMU at d_model 2560: 40 query heads of 64, sharing
# 20 key/value heads (grouped-query attention)
ATTN_Q_HEADS, ATTN_KV_HEADS, ATTN_HEAD_DIM = 40, 20, 64
SHARING_DECODE_BATCH = 16
LONG_PREFILL_CHUNK = 256


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round float values to the nearest bfloat16 (ties to even); float32 out."""
    x = np.ascontiguousarray(a, dtype=np.float32)
    bits = x.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    bits = (bits + 0x7FFF + lsb) & 0xFFFF0000
    return bits.astype(np.uint32).view(np.float32).reshape(x.shape)


def to_io(a: np.ndarray, io: str) -> np.ndarray:
    return round_bf16(a) if io == BF16 else np.ascontiguousarray(a, dtype=np.float32)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """The upper 16 bits of float32 values that are already bfloat16-exact."""
    x = np.ascontiguousarray(a, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


class Draws:
    """Named, independent, reproducible random streams."""

    def __init__(self, seed: int):
        self.seed = int(seed)

    def gen(self, name: str) -> np.random.Generator:
        return np.random.Generator(
            np.random.PCG64([self.seed, zlib.crc32(name.encode())]))

    def normal(self, name, shape, std=1.0):
        return self.gen(name).standard_normal(size=shape, dtype=np.float32) * np.float32(std)

    def uniform(self, name, shape, lo, hi):
        return self.gen(name).uniform(lo, hi, size=shape)


def scan_weights(d: Dims, seed: int) -> dict:
    """Mamba scan parameters for dims ``d`` (I/O-typed weights rounded)."""
    r = Draws(seed)
    Di, N, K, R = d.d_inner, d.d_state, d.d_conv, d.dt_rank
    dt0 = np.exp(r.uniform("dt0", (Di,), np.log(1e-3), np.log(1e-1)))
    # inverse of softplus: x = log(expm1(dt0)), written stably for small dt0
    dt_bias = dt0 + np.log(-np.expm1(-dt0))
    return dict(
        conv_w=to_io(r.normal("conv_w", (Di, K), 1.0 / np.sqrt(K)), d.io),
        conv_b=to_io(r.uniform("conv_b", (Di,), -1.0 / np.sqrt(K), 1.0 / np.sqrt(K)), d.io),
        x_proj_w=to_io(r.normal("x_proj_w", (R + 2 * N, Di), 1.0 / np.sqrt(Di)), d.io),
        dt_proj_w=to_io(r.normal("dt_proj_w", (Di, R), 1.0 / np.sqrt(R)), d.io),
        dt_bias=dt_bias.astype(np.float32),
        A=(-np.exp(r.uniform("A", (Di, N), np.log(1.0), np.log(16.0)))).astype(np.float32),
        D=r.uniform("D", (Di,), 0.5, 1.5).astype(np.float32),
        dt_rank=R,
        d_state=N,
    )


def gmu_weights(d: Dims, seed: int, layer: int = 0) -> dict:
    r = Draws(seed)
    Di, Dm = d.d_inner, d.d_model
    return dict(
        W1=to_io(r.normal(f"W1_{layer}", (Di, Dm), 1.0 / np.sqrt(Dm)), d.io),
        W2=to_io(r.normal(f"W2_{layer}", (Di, Dm), 1.0 / np.sqrt(Di)), d.io),
    )


def mamba_block_weights(d: Dims, seed: int) -> dict:
    """in_proj's x and z halves and out_proj (stored [Di, Dm], used on the right)."""
    r = Draws(seed)
    Di, Dm = d.d_inner, d.d_model
    return dict(
        W_in=to_io(r.normal("W_in", (Di, Dm), 1.0 / np.sqrt(Dm)), d.io),
        W_z=to_io(r.normal("W_z", (Di, Dm), 1.0 / np.sqrt(Dm)), d.io),
        W_out=to_io(r.normal("W_out", (Di, Dm), 1.0 / np.sqrt(Di)), d.io),
    )


def mlp_weights(d: Dims, seed: int, d_ff=None) -> dict:
    """A SwiGLU MLP's gate and up projections, [Dff, Dm] each."""
    r = Draws(seed)
    Df = d.d_inner if d_ff is None else d_ff
    return dict(
        W_g=to_io(r.normal("W_g", (Df, d.d_model), 1.0 / np.sqrt(d.d_model)), d.io),
        W_u=to_io(r.normal("W_u", (Df, d.d_model), 1.0 / np.sqrt(d.d_model)), d.io),
    )


def scan_inputs(d: Dims, seed: int, batch=None, seqlen=None, tag="u") -> np.ndarray:
    b = d.batch if batch is None else batch
    L = d.seqlen if seqlen is None else seqlen
    return to_io(Draws(seed).normal(tag, (b, L, d.d_inner)), d.io)


def gmu_inputs(d: Dims, seed: int, rows=None, tag="X") -> np.ndarray:
    T = d.tokens if rows is None else rows
    return to_io(Draws(seed).normal(tag, (T, d.d_model)), d.io)


def memory_input(d: Dims, seed: int, rows=None, tag="M") -> np.ndarray:
    T = d.tokens if rows is None else rows
    return to_io(Draws(seed).normal(tag, (T, d.d_inner)), d.io)


def attention_inputs(batch: int, kv_len: int, q_heads: int, kv_heads: int, head_dim: int, seed: int):
    """q [B, Hq, dh] and the KV cache K, V [B, N, Hkv, dh], N(0, 1), bf16-rounded."""
    r = Draws(seed)
    return (round_bf16(r.normal("q", (batch, q_heads, head_dim))),
            round_bf16(r.normal("K", (batch, kv_len, kv_heads, head_dim))),
            round_bf16(r.normal("V", (batch, kv_len, kv_heads, head_dim))))


@dataclasses.dataclass(frozen=True)
class SsdDims:
    """The SambaY-2 (Mamba-2) layer: d_inner = nheads * headdim, one group of
    B and C (d_state each), conv over C = d_inner + 2 d_state channels."""
    batch: int
    seqlen: int
    nheads: int
    headdim: int = 64
    d_state: int = 128
    d_conv: int = 4
    io: str = BF16

    @property
    def channels(self) -> int:
        return self.nheads * self.headdim + 2 * self.d_state


# The SambaY-2 variant of the prefill workload: d_inner 5120 as 80 heads of 64,
# d_state 128 (Mamba-2's defaults; the pages give no sizes for the variant).
SSD_WORKLOAD = SsdDims(1, 2048, 80, 64, 128, 4, BF16)
SSD_WORKLOAD_SEED = 1000 + 17


def ssd_weights(d: SsdDims, seed: int) -> dict:
    """Mamba-2 layer parameters for the readout: conv over [x | B | C], dt bias
    with softplus(dt_bias) in [1e-3, 1e-1], A = -exp(U[log 1, log 16]) per head,
    D ~ U(0.5, 1.5) per head (the Mamba-1 recipe per head)."""
    r = Draws(seed)
    C, H, K = d.channels, d.nheads, d.d_conv
    dt0 = np.exp(r.uniform("ssd_dt0", (H,), np.log(1e-3), np.log(1e-1)))
    return dict(
        conv_w=to_io(r.normal("ssd_conv_w", (C, K), 1.0 / np.sqrt(K)), d.io),
        conv_b=to_io(r.uniform("ssd_conv_b", (C,), -1.0 / np.sqrt(K), 1.0 / np.sqrt(K)), d.io),
        dt_bias=(dt0 + np.log(-np.expm1(-dt0))).astype(np.float32),
        A=(-np.exp(r.uniform("ssd_A", (H,), np.log(1.0), np.log(16.0)))).astype(np.float32),
        D=r.uniform("ssd_D", (H,), 0.5, 1.5).astype(np.float32),
        P=d.headdim,
        N=d.d_state,
    )


def ssd_inputs(d: SsdDims, seed: int, seqlen=None):
    """(xbc [Bt, L, C], dt_raw [Bt, L, H]): the in_proj slices, N(0, 1) and
    N(0, 0.5^2) (dt_raw around the bias), I/O-rounded."""
    r = Draws(seed)
    L = d.seqlen if seqlen is None else seqlen
    return (to_io(r.normal("xbc", (d.batch, L, d.channels)), d.io),
            to_io(r.normal("dt_raw", (d.batch, L, d.nheads), 0.5), d.io))


def workload(name: str):
    """(dims, default seed) of a named workload."""
    return WORKLOADS[name], 1000 + WORKLOAD_IDS[name]

"""GPU parity of the cross-attention decode over the single KV cache
(sambay_cross_attn_decode) against the float64 oracle: grouped heads, both
head sizes, a single cached token, KV ranges split over several CTAs, and the
decode workload's shape (64 sequences, 2048 cached tokens, 40 query heads on
20 key/value heads of 64) on sampled sequences."""

import numpy as np
import pytest
import torch

from gated_memory_sharing_b200 import abi, synth
from gated_memory_sharing_b200.layers import workspace
from oracle import sambay_ref as ref
from tests.gpu_util import TOL_BF16, assert_close, host

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


def _run(q, K, V, scale=0.0):
    B, Hq, dh = q.shape
    N, Hkv = K.shape[1], K.shape[2]
    dims = abi.AttnDims(B, N, Hq, Hkv, dh)
    dev = lambda a: torch.from_numpy(a).to("cuda").to(torch.bfloat16).contiguous()
    out = torch.empty(B, Hq, dh, dtype=torch.bfloat16, device="cuda")
    ws = workspace(abi.sambay_cross_attn_decode_workspace(dims))
    abi.sambay_cross_attn_decode(dims, dev(q), dev(K), dev(V), out, scale, ws)
    torch.cuda.synchronize()
    return host(out), abi.sambay_cross_attn_decode_workspace(dims)


@pytest.mark.parametrize("B,N,Hq,Hkv,dh", [
    (2, 77, 4, 2, 64),       # ragged last tile, groups of 2
    (3, 1, 8, 8, 64),        # one cached token, no grouping
    (4, 33, 6, 3, 64),
    (2, 300, 32, 2, 128),    # groups of 16, head size 128
    (1, 5000, 16, 2, 64),    # few sequences: the KV range splits over CTAs
    (1, 3000, 8, 1, 128),
])
def test_cross_attn_decode_small(B, N, Hq, Hkv, dh):
    q, K, V = synth.attention_inputs(B, N, Hq, Hkv, dh, seed=90 + N)
    got, ws = _run(q, K, V)
    if B * Hkv < 64 and N > 1000:
        assert ws > 0                     # the split path ran
    assert_close(got, ref.cross_attention_decode_ref(q, K, V), TOL_BF16, f"attention B{B} N{N} Hq{Hq} Hkv{Hkv} dh{dh}")


def test_cross_attn_decode_explicit_scale():
    q, K, V = synth.attention_inputs(2, 129, 4, 2, 64, seed=97)
    got, _ = _run(q, K, V, scale=0.3)
    assert_close(got, ref.cross_attention_decode_ref(q, K, V, scale=0.3), TOL_BF16, "attention scale 0.3")


def test_cross_attn_decode_workload_shape():
    """64 sequences, 2048 cached tokens, 40 query heads on 20 KV heads of 64;
    sequences are independent, so 4 sampled ones are exact checks."""
    B, N = 64, 2048
    Hq, Hkv, dh = synth.ATTN_Q_HEADS, synth.ATTN_KV_HEADS, synth.ATTN_HEAD_DIM
    q, K, V = synth.attention_inputs(B, N, Hq, Hkv, dh, seed=98)
    got, ws = _run(q, K, V)
    assert ws == 0                        # one CTA per (sequence, KV head) fills the GPU
    seqs = [0, 17, 40, 63]
    assert_close(got[seqs], ref.cross_attention_decode_ref(q[seqs], K[seqs], V[seqs]), TOL_BF16,
                 "attention at the decode workload's shape (sampled sequences)")

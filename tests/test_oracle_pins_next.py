"""Pins for the oracle functions around the scan + GMU path: the bf16 I/O
rounding of chained layers, the Mamba layer that produces M, the SwiGLU MLP
representation of SambaY-MLP, and single-query cross-attention over the KV
cache.  Each is fixed against a library routine, brute force, a hand-derived
value or a special case that reduces to another pinned function.  CPU only.
"""

import math

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as F

from oracle import sambay_ref as ref


# ---------------------------------------------------------------- bf16 rounding

def test_round_bf16_matches_torch_conversion():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(2000) * 1e-30).astype(np.float32),
        (rng.standard_normal(2000) * 1e30).astype(np.float32),
        np.float32([0.0, -0.0, 1.0, -1.0, 3.0, 1e-38, -2e-38]),
    ])
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(ref.round_bf16(x.astype(np.float64)), want)


def test_round_bf16_ties_to_even_by_hand():
    # bf16 spacing at 1 is 2^-7: 1 + 2^-8 is a tie between 1 (even) and
    # 1 + 2^-7 (odd); 1 + 3 * 2^-8 a tie between 1 + 2^-7 (odd) and 1 + 2^-6 (even)
    assert ref.round_bf16(1.0 + 2.0 ** -8) == 1.0
    assert ref.round_bf16(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6
    assert ref.round_bf16(-(1.0 + 3 * 2.0 ** -8)) == -(1.0 + 2.0 ** -6)
    assert ref.round_bf16(1.0 + 2.0 ** -8 + 2.0 ** -20) == 1.0 + 2.0 ** -7
    assert ref.round_bf16(2.0 ** -130) == 2.0 ** -130          # a bf16 subnormal, exact


def test_gmu_layers_io_round_rounds_between_layers():
    rng = np.random.default_rng(1)
    T, Dm, Di = 6, 8, 12
    X = rng.standard_normal((T, Dm))
    M = rng.standard_normal((T, Di))
    W1s = [rng.standard_normal((Di, Dm)) * 0.3 for _ in range(3)]
    W2s = [rng.standard_normal((Di, Dm)) * 0.3 for _ in range(3)]

    def bf(a):
        return torch.from_numpy(np.asarray(a, np.float64)).to(torch.bfloat16).to(torch.float64).numpy()

    x, m = X, bf(M)
    for W1, W2 in zip(W1s, W2s):
        z = x @ W1.T
        x = bf(x + (m * z * scipy.special.expit(z)) @ W2)
    np.testing.assert_allclose(ref.gmu_layers_ref(X, M, W1s, W2s, io_round=True), x, rtol=1e-12, atol=1e-14)
    # and without rounding the chain differs from the rounded one
    assert not np.allclose(ref.gmu_layers_ref(X, M, W1s, W2s), x, rtol=1e-6)


# ---------------------------------------------------------------- Mamba layer

def _scan_weights(rng, Di, N=3, K=4, R=2):
    return dict(
        conv_w=rng.standard_normal((Di, K)) * 0.5,
        conv_b=rng.standard_normal(Di) * 0.3,
        x_proj_w=rng.standard_normal((R + 2 * N, Di)) * 0.4,
        dt_proj_w=rng.standard_normal((Di, R)) * 0.5,
        dt_bias=rng.uniform(-4.0, -1.0, Di),
        A=-np.exp(rng.uniform(0.0, np.log(16.0), (Di, N))),
        D=rng.uniform(0.5, 1.5, Di),
        dt_rank=R,
        d_state=N,
    )


def test_mamba_layer_matches_torch_linear_composition():
    rng = np.random.default_rng(2)
    B, L, Dm, Di = 2, 9, 5, 6
    w = _scan_weights(rng, Di)
    X = rng.standard_normal((B, L, Dm))
    W_in, W_z, W_out = (rng.standard_normal((Di, Dm)) * 0.5 for _ in range(3))
    r = ref.mamba_layer_ref(X, w, W_in, W_z, W_out)
    Xt = torch.from_numpy(X)
    u = F.linear(Xt, torch.from_numpy(W_in))            # the x branch, X W_in^T
    z = F.linear(Xt, torch.from_numpy(W_z))             # the gate branch
    y = ref.scan_prefill_ref(u.numpy(), w)["M"]
    out = F.linear(torch.from_numpy(y) * F.silu(z), torch.from_numpy(W_out).T) + Xt
    np.testing.assert_allclose(r["out"], out.numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(r["M"], y, rtol=1e-13)


def test_mamba_layer_io_round_rounds_u_and_M():
    rng = np.random.default_rng(8)
    B, L, Dm, Di = 1, 11, 5, 6
    w = _scan_weights(rng, Di)
    X = rng.standard_normal((B, L, Dm))
    W_in, W_z, W_out = (rng.standard_normal((Di, Dm)) * 0.5 for _ in range(3))
    r = ref.mamba_layer_ref(X, w, W_in, W_z, W_out, io_round=True)
    bf = lambda t: t.to(torch.bfloat16).to(torch.float64)
    Xt = torch.from_numpy(X)
    u = bf(F.linear(Xt, torch.from_numpy(W_in)))
    z = F.linear(Xt, torch.from_numpy(W_z))
    y = ref.scan_prefill_ref(u.numpy(), w)["M"]
    out = F.linear(bf(torch.from_numpy(y)) * F.silu(z), torch.from_numpy(W_out).T) + Xt
    np.testing.assert_allclose(r["M"], y, rtol=1e-13)
    np.testing.assert_allclose(r["out"], out.numpy(), rtol=1e-12, atol=1e-13)
    assert not np.allclose(r["M"], ref.mamba_layer_ref(X, w, W_in, W_z, W_out)["M"], rtol=1e-6)


def test_mamba_layer_special_cases():
    rng = np.random.default_rng(3)
    B, L, Di = 1, 7, 6
    w = _scan_weights(rng, Di)
    X = rng.standard_normal((B, L, Di))
    W_z, W_out = (rng.standard_normal((Di, Di)) for _ in range(2))
    # identity x branch: M is the scan of X itself
    r = ref.mamba_layer_ref(X, w, np.eye(Di), W_z, W_out)
    np.testing.assert_allclose(r["M"], ref.scan_prefill_ref(X, w)["M"], rtol=1e-13)
    # zero gate branch: SiLU(0) = 0 closes the layer, only the residual passes
    r0 = ref.mamba_layer_ref(X, w, np.eye(Di), np.zeros((Di, Di)), W_out)
    np.testing.assert_array_equal(r0["out"], X)
    # the gate multiplies y, not u: with a large positive gate SiLU(z) ~ z
    r1 = ref.mamba_layer_ref(X, w, np.eye(Di), np.eye(Di) * 50.0, np.eye(Di), residual=False)
    np.testing.assert_allclose(r1["out"], r1["M"] * (50.0 * X) * scipy.special.expit(50.0 * X), rtol=1e-12)


# ---------------------------------------------------------------- MLP representation

def test_mlp_representation_bruteforce_and_branch_order():
    rng = np.random.default_rng(4)
    T, Dm, Dff = 3, 4, 5
    X = rng.standard_normal((T, Dm))
    W_g = rng.standard_normal((Dff, Dm))
    W_u = rng.standard_normal((Dff, Dm))
    M = ref.mlp_representation_ref(X, W_g, W_u)
    for t in range(T):
        for f in range(Dff):
            g = sum(X[t, k] * W_g[f, k] for k in range(Dm))
            u = sum(X[t, k] * W_u[f, k] for k in range(Dm))
            assert M[t, f] == pytest.approx(g / (1.0 + math.exp(-g)) * u, rel=1e-12, abs=1e-14)
    # SiLU acts on the W_g branch: with W_g = 0 everything is 0, with W_u = 0 too,
    # and swapping the branches changes the result
    assert not ref.mlp_representation_ref(X, np.zeros_like(W_g), W_u).any()
    assert not np.allclose(ref.mlp_representation_ref(X, W_u, W_g), M)


def test_sambay_mlp_gmu_reduces_to_gmu_on_the_mlp_memory():
    rng = np.random.default_rng(5)
    T, Dm, Dff = 4, 6, 8
    Xs, Xc = rng.standard_normal((T, Dm)), rng.standard_normal((T, Dm))
    W_g, W_u, W1, W2 = (rng.standard_normal((Dff, Dm)) * 0.4 for _ in range(4))
    Y, M = ref.sambay_mlp_gmu_ref(Xc, Xs, W_g, W_u, W1, W2)
    Mt = F.silu(torch.from_numpy(Xs) @ torch.from_numpy(W_g).T) * (torch.from_numpy(Xs) @ torch.from_numpy(W_u).T)
    Yt = (Mt * F.silu(torch.from_numpy(Xc) @ torch.from_numpy(W1).T)) @ torch.from_numpy(W2)
    np.testing.assert_allclose(M, Mt.numpy(), rtol=1e-12)
    np.testing.assert_allclose(Y, Yt.numpy(), rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- cross-attention decode

def test_cross_attention_bruteforce_loops():
    rng = np.random.default_rng(6)
    B, N, Hq, Hkv, dh = 2, 5, 4, 2, 3
    q = rng.standard_normal((B, Hq, dh))
    K = rng.standard_normal((B, N, Hkv, dh))
    V = rng.standard_normal((B, N, Hkv, dh))
    out = ref.cross_attention_decode_ref(q, K, V)
    for b in range(B):
        for h in range(Hq):
            kv = h // (Hq // Hkv)                  # consecutive query heads share a KV head
            s = [sum(q[b, h, d] * K[b, j, kv, d] for d in range(dh)) / math.sqrt(dh) for j in range(N)]
            m = max(s)
            e = [math.exp(x - m) for x in s]
            for d in range(dh):
                want = sum(e[j] * V[b, j, kv, d] for j in range(N)) / sum(e)
                assert out[b, h, d] == pytest.approx(want, rel=1e-12, abs=1e-14)


def test_cross_attention_special_cases():
    rng = np.random.default_rng(7)
    B, N, Hq, Hkv, dh = 2, 7, 6, 3, 4
    K = rng.standard_normal((B, N, Hkv, dh))
    V = rng.standard_normal((B, N, Hkv, dh))
    # one cached token: the output is its value
    q = rng.standard_normal((B, Hq, dh))
    np.testing.assert_allclose(ref.cross_attention_decode_ref(q, K[:, :1], V[:, :1]),
                               np.repeat(V[:, 0], Hq // Hkv, axis=1), rtol=1e-13)
    # a zero query weighs every token equally: the mean of the values
    np.testing.assert_allclose(ref.cross_attention_decode_ref(np.zeros((B, Hq, dh)), K, V),
                               np.repeat(V.mean(axis=1), Hq // Hkv, axis=1), rtol=1e-12, atol=1e-14)
    # grouped heads equal ungrouped attention over explicitly repeated KV heads
    Kr, Vr = np.repeat(K, Hq // Hkv, axis=2), np.repeat(V, Hq // Hkv, axis=2)
    np.testing.assert_allclose(ref.cross_attention_decode_ref(q, K, V),
                               ref.cross_attention_decode_ref(q, Kr, Vr), rtol=1e-13)
    # scipy's softmax on the scaled logits
    logits = np.einsum("bhd,bnhd->bhn", q, Kr) / math.sqrt(dh)
    want = np.einsum("bhn,bnhd->bhd", scipy.special.softmax(logits, axis=-1), Vr)
    np.testing.assert_allclose(ref.cross_attention_decode_ref(q, K, V), want, rtol=1e-12)
    # a dominant key takes all the weight
    Kd = K.copy()
    Kd[:, 3] = 0.0
    qd = np.zeros((B, Hq, dh))
    qd[:, :, 0] = 1.0
    Kd[:, 3, :, 0] = 1e4
    np.testing.assert_allclose(ref.cross_attention_decode_ref(qd, Kd, V),
                               np.repeat(V[:, 3], Hq // Hkv, axis=1), rtol=1e-12)

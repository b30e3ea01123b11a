"""Pins for the float64 oracle against things other than itself.

Each test fixes a part of the oracle with a hand-derived value, a closed form,
a brute-force evaluation, a library routine or an invariant of the method, so
that a dropped term, a wrong sign or index, or a transposed operand anywhere in
the oracle fails at least one of them.  CPU only.
"""

import json
import math
import os

import numpy as np
import pytest
import scipy.special

from oracle import sambay_ref as ref
from gated_memory_sharing_b200 import synth


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def _tiny_weights(rng, Di=6, N=3, K=4, R=2):
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


# ---------------------------------------------------------------- elementwise

def test_silu_known_values():
    s = 1.0 / (1.0 + math.exp(-1.0))
    assert ref.silu(0.0) == 0.0
    assert ref.silu(1.0) == pytest.approx(s, rel=1e-15)
    assert ref.silu(-1.0) == pytest.approx(-(1.0 - s), rel=1e-15)
    x = np.linspace(-30, 30, 121)
    np.testing.assert_allclose(ref.silu(x), x * scipy.special.expit(x), rtol=1e-14, atol=1e-300)
    # saturation: SiLU(x) -> x for large x, -> 0 (from below) for very negative x
    assert ref.silu(50.0) == pytest.approx(50.0, rel=1e-15)
    assert -1e-300 < ref.silu(-800.0) <= 0.0


def test_softplus_closed_forms():
    assert ref.softplus(0.0) == pytest.approx(math.log(2.0), rel=1e-15)
    x = np.linspace(-20, 20, 81)
    # softplus(x) - softplus(-x) = x ;  softplus is the integral of the logistic
    np.testing.assert_allclose(ref.softplus(x) - ref.softplus(-x), x, atol=1e-13)
    np.testing.assert_allclose(ref.softplus(x), np.log1p(np.exp(x)), rtol=1e-14)
    assert ref.softplus(800.0) == pytest.approx(800.0, rel=1e-15)
    # the dt bias recipe inverts softplus: softplus(bias) = dt0 in [1e-3, 1e-1]
    w = synth.scan_weights(synth.WORKLOADS["tiny_f32"], 1000)
    dt0 = ref.softplus(w["dt_bias"].astype(np.float64))
    assert dt0.min() >= 1e-3 * (1 - 1e-5) and dt0.max() <= 1e-1 * (1 + 1e-5)


# ----------------------------------------------------------------------- conv

def test_conv_impulse_golden(golden_dir):
    g = _load(golden_dir, "conv_impulse.json")
    w = np.array(g["w"])[None, :]
    u = np.array(g["u"])[None, :, None]
    uc, state = ref.causal_conv1d_silu(u, w, np.zeros(1))
    np.testing.assert_allclose(uc[0, :, 0], ref.silu(np.array(g["pre"])), rtol=1e-15)
    np.testing.assert_array_equal(state[0, 0], np.array(g["state_after"]))


def test_conv_matches_numpy_convolve():
    rng = np.random.default_rng(1)
    Bsz, L, Di, K = 2, 11, 5, 4
    u = rng.standard_normal((Bsz, L, Di))
    w = rng.standard_normal((Di, K))
    bias = rng.standard_normal(Di)
    uc, state = ref.causal_conv1d_silu(u, w, bias)
    for b in range(Bsz):
        for c in range(Di):
            padded = np.concatenate([np.zeros(K - 1), u[b, :, c]])
            # np.convolve flips its kernel: correlating with w = convolving with w[::-1]
            pre = np.convolve(padded, w[c, ::-1], mode="valid") + bias[c]
            np.testing.assert_allclose(uc[b, :, c], scipy.special.expit(pre) * pre, rtol=1e-12)
            np.testing.assert_array_equal(state[b, c], u[b, -K:, c])


def test_conv_state_continuation_and_short_prompt():
    rng = np.random.default_rng(2)
    u = rng.standard_normal((1, 9, 3))
    w = rng.standard_normal((3, 4))
    bias = rng.standard_normal(3)
    full, st_full = ref.causal_conv1d_silu(u, w, bias)
    a, st_a = ref.causal_conv1d_silu(u[:, :2], w, bias)     # L < K
    np.testing.assert_array_equal(st_a[0, :, :2], 0.0)      # zero-padded history
    np.testing.assert_array_equal(st_a[0, :, 2:], u[0, :2].T)
    b, st_b = ref.causal_conv1d_silu(u[:, 2:], w, bias, st_a)
    np.testing.assert_allclose(np.concatenate([a, b], axis=1), full, rtol=1e-14)
    np.testing.assert_array_equal(st_b, st_full)


# --------------------------------------------------------------------- x_proj

def test_x_proj_split_order():
    # x_proj_w rows pick single channels, so each output slice is identifiable
    Di, R, N = 10, 2, 3
    uc = np.arange(1, Di + 1, dtype=np.float64)[None, None, :] * np.array([1.0, -2.0])[:, None, None]
    W = np.zeros((R + 2 * N, Di))
    for j in range(R + 2 * N):
        W[j, j] = 1.0
    delta, Bm, Cm = ref.x_proj(uc, W, R, N)
    np.testing.assert_array_equal(delta[0, 0], [1, 2])
    np.testing.assert_array_equal(Bm[0, 0], [3, 4, 5])
    np.testing.assert_array_equal(Cm[1, 0], [-12, -14, -16])


def test_dt_softplus_bruteforce():
    rng = np.random.default_rng(3)
    delta = rng.standard_normal((1, 4, 3))
    Wdt = rng.standard_normal((5, 3))
    bias = rng.standard_normal(5)
    got = ref.dt_softplus(delta, Wdt, bias)
    for t in range(4):
        for c in range(5):
            z = bias[c] + sum(delta[0, t, r] * Wdt[c, r] for r in range(3))
            assert got[0, t, c] == pytest.approx(math.log1p(math.exp(z)), rel=1e-13)


# ----------------------------------------------------------------------- scan

def test_scan_half_decay_golden(golden_dir):
    g = _load(golden_dir, "scan_half_decay.json")
    L = len(g["u"])
    ln2 = math.log(2.0)
    uc = np.array(g["u"])[None, :, None]
    dt = np.full((1, L, 1), ln2)
    A = np.array([[g["A"]]])
    Bm = np.array(g["B"])[None, :, None]
    Cm = np.array(g["C"])[None, :, None]
    y, h = ref.selective_scan(uc, dt, A, Bm, Cm, np.array([g["D"]]))
    want = np.array(g["y_coef_ln2"]) * ln2 + np.array(g["y_const"])
    np.testing.assert_allclose(y[0, :, 0], want, rtol=1e-14, atol=1e-15)
    assert h[0, 0, 0] == pytest.approx(g["h_coef_ln2"][-1] * ln2, rel=1e-14)


def test_scan_geometric_closed_form():
    # N = 1, constant dt, B = C = 1, constant input v:
    # y_t = dt*v*(1 - a^(t+1))/(1 - a) + D*v with a = exp(dt*A)
    L, dt0, A0, v, D0 = 40, 0.07, -3.0, 1.7, 0.9
    a = math.exp(dt0 * A0)
    y, _ = ref.selective_scan(np.full((1, L, 1), v), np.full((1, L, 1), dt0), np.array([[A0]]),
                              np.ones((1, L, 1)), np.ones((1, L, 1)), np.array([D0]))
    t = np.arange(L)
    want = dt0 * v * (1.0 - a ** (t + 1)) / (1.0 - a) + D0 * v
    np.testing.assert_allclose(y[0, :, 0], want, rtol=1e-13)


def test_scan_single_token_and_limits():
    rng = np.random.default_rng(4)
    Bsz, Di, N = 2, 5, 16
    uc = rng.standard_normal((Bsz, 1, Di))
    dt = rng.uniform(1e-3, 0.1, (Bsz, 1, Di))
    A = -np.exp(rng.uniform(0, np.log(16), (Di, N)))
    Bm = rng.standard_normal((Bsz, 1, N))
    Cm = rng.standard_normal((Bsz, 1, N))
    D = rng.uniform(0.5, 1.5, Di)
    # L = 1 from a zero state: y = dt*uc*(C.B) + D*uc
    y, _ = ref.selective_scan(uc, dt, A, Bm, Cm, D)
    cb = np.sum(Cm[:, 0] * Bm[:, 0], axis=-1)
    np.testing.assert_allclose(y[:, 0], dt[:, 0] * uc[:, 0] * cb[:, None] + D * uc[:, 0], rtol=1e-13)
    # A -> -inf: exp(dt*A) = 0, the scan forgets everything: memoryless readout
    L = 6
    uc = rng.standard_normal((Bsz, L, Di))
    dt = rng.uniform(1e-3, 0.1, (Bsz, L, Di))
    Bm = rng.standard_normal((Bsz, L, N))
    Cm = rng.standard_normal((Bsz, L, N))
    y, _ = ref.selective_scan(uc, dt, np.full((Di, N), -1e300), Bm, Cm, D)
    cb = np.sum(Cm * Bm, axis=-1)
    np.testing.assert_allclose(y, dt * uc * cb[:, :, None] + D * uc, rtol=1e-13)
    # dt = 0: nothing enters the state, only the skip term remains
    y, h = ref.selective_scan(uc, np.zeros_like(dt), A, Bm, Cm, D)
    np.testing.assert_allclose(y, D * uc, rtol=1e-15)
    assert not h.any()


def test_scan_bruteforce_scalar_loops():
    rng = np.random.default_rng(5)
    Bsz, L, Di, N = 2, 5, 3, 4
    uc = rng.standard_normal((Bsz, L, Di))
    dt = rng.uniform(0.01, 0.5, (Bsz, L, Di))
    A = -rng.uniform(0.5, 4.0, (Di, N))
    Bm = rng.standard_normal((Bsz, L, N))
    Cm = rng.standard_normal((Bsz, L, N))
    D = rng.standard_normal(Di)
    h0 = rng.standard_normal((Bsz, Di, N))
    y, h = ref.selective_scan(uc, dt, A, Bm, Cm, D, h0)
    for b in range(Bsz):
        for c in range(Di):
            hs = [h0[b, c, n] for n in range(N)]
            for t in range(L):
                acc = 0.0
                for n in range(N):
                    hs[n] = math.exp(dt[b, t, c] * A[c, n]) * hs[n] + dt[b, t, c] * Bm[b, t, n] * uc[b, t, c]
                    acc += Cm[b, t, n] * hs[n]
                assert y[b, t, c] == pytest.approx(acc + D[c] * uc[b, t, c], rel=1e-12, abs=1e-14)
            np.testing.assert_allclose(h[b, c], hs, rtol=1e-12)


def test_scan_recurrent_equals_parallel_form():
    rng = np.random.default_rng(6)
    L, Di, N = 12, 4, 16
    uc = rng.standard_normal((1, L, Di))
    dt = rng.uniform(1e-3, 0.3, (1, L, Di))
    A = -np.exp(rng.uniform(0, np.log(16), (Di, N)))
    Bm = rng.standard_normal((1, L, N))
    Cm = rng.standard_normal((1, L, N))
    D = rng.uniform(0.5, 1.5, Di)
    y, _ = ref.selective_scan(uc, dt, A, Bm, Cm, D)
    mix = ref.mixing_matrix_ref(dt[0], A, Bm[0], Cm[0], D)
    assert np.all(np.triu(mix[0], 1) == 0.0)                  # causal
    par = np.stack([mix[c] @ uc[0, :, c] for c in range(Di)], axis=1)
    np.testing.assert_allclose(y[0], par, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("chunk", [1, 7, 256])
def test_scan_chunked_equals_unchunked(chunk):
    rng = np.random.default_rng(7)
    L, Di, N = 300, 3, 16
    uc = rng.standard_normal((2, L, Di))
    dt = rng.uniform(1e-3, 0.1, (2, L, Di))
    A = -np.exp(rng.uniform(0, np.log(16), (Di, N)))
    Bm = rng.standard_normal((2, L, N))
    Cm = rng.standard_normal((2, L, N))
    D = rng.uniform(0.5, 1.5, Di)
    y, h = ref.selective_scan(uc, dt, A, Bm, Cm, D)
    ys, hc = [], None
    for s in range(0, L, chunk):
        e = min(L, s + chunk)
        yc, hc = ref.selective_scan(uc[:, s:e], dt[:, s:e], A, Bm[:, s:e], Cm[:, s:e], D, hc)
        ys.append(yc)
    np.testing.assert_allclose(np.concatenate(ys, axis=1), y, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(hc, h, rtol=1e-13)


def test_scan_linear_in_input():
    rng = np.random.default_rng(8)
    L, Di, N = 9, 4, 16
    dt = rng.uniform(1e-3, 0.2, (1, L, Di))
    A = -np.exp(rng.uniform(0, np.log(16), (Di, N)))
    Bm = rng.standard_normal((1, L, N))
    Cm = rng.standard_normal((1, L, N))
    D = rng.uniform(0.5, 1.5, Di)
    u1 = rng.standard_normal((1, L, Di))
    u2 = rng.standard_normal((1, L, Di))
    f = lambda u: ref.selective_scan(u, dt, A, Bm, Cm, D)[0]
    np.testing.assert_allclose(f(2.0 * u1 - 3.0 * u2), 2.0 * f(u1) - 3.0 * f(u2), rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------- prefill / decode

def test_decode_steps_equal_prefill():
    rng = np.random.default_rng(9)
    w = _tiny_weights(rng)
    L0, k = 7, 5
    u = rng.standard_normal((2, L0 + k, 6))
    full = ref.scan_prefill_ref(u, w)
    r = ref.scan_prefill_ref(u[:, :L0], w)
    h, cs = r["ssm_state"], r["conv_state"]
    for i in range(k):
        m, h, cs = ref.scan_step_ref(u[:, L0 + i], w, h, cs)
        np.testing.assert_allclose(m, full["M"][:, L0 + i], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(h, full["ssm_state"], rtol=1e-12)
    np.testing.assert_array_equal(cs, full["conv_state"])
    # the decode state has a fixed size, whatever the position
    assert h.shape == (2, 6, 3) and cs.shape == (2, 6, 4)


def test_prefill_chunked_with_state_equals_whole():
    rng = np.random.default_rng(10)
    w = _tiny_weights(rng)
    u = rng.standard_normal((1, 20, 6))
    full = ref.scan_prefill_ref(u, w)
    a = ref.scan_prefill_ref(u[:, :8], w)
    b = ref.scan_prefill_ref(u[:, 8:], w, a["ssm_state"], a["conv_state"])
    np.testing.assert_allclose(np.concatenate([a["M"], b["M"]], axis=1), full["M"], rtol=1e-12, atol=1e-14)


# ------------------------------------------------------------------------ GMU

def test_gmu_golden(golden_dir):
    g = _load(golden_dir, "gmu_tiny.json")
    X, W1, M, W2 = (np.array(g[k]) for k in ("X", "W1", "M", "W2"))
    Y, G, H = ref.gmu_ref(X, M, W1, W2)
    np.testing.assert_allclose(G, g["G"], rtol=1e-15)
    np.testing.assert_allclose(Y, g["Y"], rtol=1e-15)
    Yr, _, _ = ref.gmu_ref(X, M, W1, W2, residual=True)
    np.testing.assert_allclose(Yr, g["Y_residual"], rtol=1e-15)


def test_gmu_bruteforce_loops():
    rng = np.random.default_rng(11)
    T, Dm, Di = 3, 4, 5
    X = rng.standard_normal((T, Dm))
    M = rng.standard_normal((T, Di))
    W1 = rng.standard_normal((Di, Dm))
    W2 = rng.standard_normal((Di, Dm))
    Y, _, _ = ref.gmu_ref(X, M, W1, W2)
    for t in range(T):
        for o in range(Dm):
            acc = 0.0
            for i in range(Di):
                z = sum(X[t, k] * W1[i, k] for k in range(Dm))
                acc += M[t, i] * (z / (1.0 + math.exp(-z))) * W2[i, o]
            assert Y[t, o] == pytest.approx(acc, rel=1e-12, abs=1e-14)


def test_gmu_special_cases():
    rng = np.random.default_rng(12)
    T, Dm, Di = 4, 3, 6
    X = rng.standard_normal((T, Dm))
    M = rng.standard_normal((T, Di))
    W2 = rng.standard_normal((Di, Dm))
    # W1 = 0: the gate is SiLU(0) = 0, nothing passes
    Y, _, _ = ref.gmu_ref(X, M, np.zeros((Di, Dm)), W2)
    assert not Y.any()
    Yr, _, _ = ref.gmu_ref(X, M, np.zeros((Di, Dm)), W2, residual=True)
    np.testing.assert_array_equal(Yr, X)
    # constant gate input c: Y = SiLU(c) * M W2
    c = 0.8
    Xc = np.zeros((T, Dm)); Xc[:, 0] = 1.0
    W1 = np.zeros((Di, Dm)); W1[:, 0] = c
    Y, _, _ = ref.gmu_ref(Xc, M, W1, W2)
    np.testing.assert_allclose(Y, scipy.special.expit(c) * c * (M @ W2), rtol=1e-13)


def test_gmu_layers_compose():
    rng = np.random.default_rng(13)
    T, Dm, Di = 5, 3, 4
    X = rng.standard_normal((T, Dm))
    M = rng.standard_normal((T, Di))
    W1s = [rng.standard_normal((Di, Dm)) for _ in range(3)]
    W2s = [rng.standard_normal((Di, Dm)) for _ in range(3)]
    x = X
    for W1, W2 in zip(W1s, W2s):
        z = x @ W1.T
        x = x + (M * (z * scipy.special.expit(z))) @ W2
    np.testing.assert_allclose(ref.gmu_layers_ref(X, M, W1s, W2s), x, rtol=1e-13)


def test_lifted_tensor_identity_tiny_workload():
    """GMU(X, M) equals token mixing through the lifted tensor Ã_ijk = G_ik A_ij.

    Materialises every channel's mixing matrix by brute force on the tiny
    float32 workload (L = 64, d_inner = 128) and checks the two routes to Y
    agree to float64 round-off.
    """
    d, seed = synth.workload("tiny_f32")
    w = synth.scan_weights(d, seed)
    u = synth.scan_inputs(d, seed)
    gw = synth.gmu_weights(d, seed)
    X = synth.gmu_inputs(d, seed)
    r = ref.scan_prefill_ref(u, w)
    Y, G, _ = ref.gmu_ref(X, r["M"][0], gw["W1"], gw["W2"])
    mix = ref.mixing_matrix_ref(r["dt"][0], w["A"], r["Bm"][0], r["Cm"][0], w["D"])
    Y_lift = ref.lifted_gmu_ref(r["uc"][0], G, mix, gw["W2"])
    np.testing.assert_allclose(Y_lift, Y, rtol=1e-10, atol=1e-12)
    assert np.abs(Y - Y_lift).max() <= 1e-12 * np.abs(Y).max()

"""Pins of the SambaY-2 (Mamba-2 SSD) oracle against things other than itself.

The SSD recurrence (Dao & Gu 2024, "Transformers are SSMs"; the SambaY-2 row
of the ablation table, Paper-Notes page, 实验关键数据 > 消融实验) is checked
against a hand-derived golden case, a scalar brute force, its matrix form,
the chunked form, and closed forms of its special cases.
"""

import json
import os

import numpy as np
import pytest

from oracle import sambay_ref as ref
from oracle import ssd_ref as ssd

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "ssd_tiny.json")


def _rand(shape, rng, scale=1.0):
    return rng.standard_normal(shape) * scale


def _inputs(rng, Bt=2, L=13, H=3, P=4, N=5):
    x = _rand((Bt, L, H, P), rng)
    dt = rng.uniform(0.01, 0.4, (Bt, L, H))
    A = -np.exp(rng.uniform(0.0, np.log(8.0), H))
    Bm = _rand((Bt, L, N), rng)
    Cm = _rand((Bt, L, N), rng)
    D = rng.uniform(0.5, 1.5, H)
    return x, dt, A, Bm, Cm, D


def test_golden_hand_derived():
    g = json.load(open(GOLDEN))
    x = np.array(g["x"]).reshape(1, 3, 1, 1)
    dt = np.array(g["dt"]).reshape(1, 3, 1)
    Bm = np.array(g["B"]).reshape(1, 3, 1)
    Cm = np.array(g["C"]).reshape(1, 3, 1)
    y, h = ssd.ssd_recurrent(x, dt, np.array([g["A"]]), Bm, Cm, np.array([g["D"]]))
    np.testing.assert_allclose(y.ravel(), g["y"], rtol=1e-14)
    np.testing.assert_allclose(h.ravel(), [g["final_state"]], rtol=1e-14)


def test_scalar_brute_force():
    rng = np.random.default_rng(1)
    x, dt, A, Bm, Cm, D = _inputs(rng, Bt=1, L=6, H=2, P=2, N=3)
    h0 = _rand((1, 2, 2, 3), rng)
    y, h = ssd.ssd_recurrent(x, dt, A, Bm, Cm, D, h0)
    for hh in range(2):
        for p in range(2):
            st = [float(h0[0, hh, p, n]) for n in range(3)]
            for t in range(6):
                a = float(np.exp(dt[0, t, hh] * A[hh]))
                acc = 0.0
                for n in range(3):
                    st[n] = a * st[n] + float(dt[0, t, hh]) * float(x[0, t, hh, p]) * float(Bm[0, t, n])
                    acc += st[n] * float(Cm[0, t, n])
                assert abs(y[0, t, hh, p] - (acc + D[hh] * x[0, t, hh, p])) < 1e-12
            np.testing.assert_allclose(h[0, hh, p], st, rtol=1e-12)


@pytest.mark.parametrize("chunk", [1, 3, 8, 13, 64])
def test_chunked_equals_recurrent(chunk):
    rng = np.random.default_rng(2)
    x, dt, A, Bm, Cm, D = _inputs(rng)
    h0 = _rand((2, 3, 4, 5), rng)
    y1, h1 = ssd.ssd_recurrent(x, dt, A, Bm, Cm, D, h0)
    y2, h2 = ssd.ssd_chunked(x, dt, A, Bm, Cm, D, h0, chunk=chunk)
    np.testing.assert_allclose(y2, y1, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(h2, h1, rtol=1e-11, atol=1e-12)


def test_matrix_form():
    """From a zero state y = Mix x + D x, Mix the 2-D mixing matrix per head."""
    rng = np.random.default_rng(3)
    x, dt, A, Bm, Cm, D = _inputs(rng)
    y, _ = ssd.ssd_recurrent(x, dt, A, Bm, Cm, D)
    mix = ssd.ssd_matrix(dt, A, Bm, Cm)
    assert np.all(np.triu(mix[0, 0], 1) == 0.0)
    y2 = np.einsum("bhts,bshp->bthp", mix, x) + D[None, None, :, None] * x
    np.testing.assert_allclose(y2, y, rtol=1e-11, atol=1e-12)


def test_lifted_tensor_identity_exact_2d():
    """GMU over the SSD readout: Y = (M ⊙ G) W2 with G = SiLU(X W1^T) equals
    the token mixing with the lifted tensor Ã[t, s, k] = G[t, k] Mix_h(k)[t, s]
    (Paper-Notes page, 方法详解 > 关键设计), with the 2-D Mix exact."""
    rng = np.random.default_rng(4)
    Bt, L, H, P, N, Dm = 1, 7, 2, 3, 4, 5
    x, dt, A, Bm, Cm, D = _inputs(rng, Bt, L, H, P, N)
    D = np.zeros(H)
    y, _ = ssd.ssd_recurrent(x, dt, A, Bm, Cm, D)
    M = y.reshape(L, H * P)
    X = _rand((L, Dm), rng)
    W1 = _rand((H * P, Dm), rng)
    W2 = _rand((H * P, Dm), rng)
    Y, _, _ = ref.gmu_ref(X, M, W1, W2)
    G = ref.silu(X @ W1.T)                                       # [L, H*P]
    mix = ssd.ssd_matrix(dt, A, Bm, Cm)[0]                       # [H, L, L]
    head = np.arange(H * P) // P
    lifted = G[:, None, :] * mix[head].transpose(1, 2, 0)        # [t, s, k]
    xk = x.reshape(L, H * P)
    Y2 = np.einsum("tsk,sk->tk", lifted, xk) @ W2
    np.testing.assert_allclose(Y2, Y, rtol=1e-10, atol=1e-11)


def test_zero_dt_keeps_state_and_reads_skip():
    rng = np.random.default_rng(5)
    x, dt, A, Bm, Cm, D = _inputs(rng)
    h0 = _rand((2, 3, 4, 5), rng)
    y, h = ssd.ssd_recurrent(x, np.zeros_like(dt), A, Bm, Cm, D, h0)
    np.testing.assert_allclose(h, h0, rtol=0, atol=0)
    carry = np.einsum("bhpn,btn->bthp", h0, Cm)
    np.testing.assert_allclose(y, carry + D[None, None, :, None] * x, rtol=1e-13)


def test_no_memory_limit():
    """A -> -inf: nothing is carried; y_t = dt_t (C_t . B_t) x_t + D x_t."""
    rng = np.random.default_rng(6)
    x, dt, A, Bm, Cm, D = _inputs(rng)
    y, h = ssd.ssd_recurrent(x, dt, np.full(3, -1e9), Bm, Cm, D, _rand((2, 3, 4, 5), rng))
    cb = np.einsum("btn,btn->bt", Cm, Bm)
    want = (dt * cb[..., None])[..., None] * x + D[None, None, :, None] * x
    np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-12)
    last = dt[:, -1, :, None, None] * x[:, -1, :, :, None] * Bm[:, -1, None, None, :]
    np.testing.assert_allclose(h, last, rtol=1e-12, atol=1e-12)


def _weights(rng, H=3, P=4, N=5, K=4):
    C = H * P + 2 * N
    return {"conv_w": _rand((C, K), rng, 0.5), "conv_b": rng.uniform(-0.5, 0.5, C),
            "dt_bias": rng.uniform(-4.0, -1.0, H), "A": -np.exp(rng.uniform(0.0, np.log(8.0), H)),
            "D": rng.uniform(0.5, 1.5, H), "P": P, "N": N}


def test_split_order_of_xbc():
    """[x | B | C]: with the B slice zero after the conv nothing enters the
    state (y = D x); with the C slice zero the readout sees only the skip."""
    rng = np.random.default_rng(7)
    H, P, N = 3, 4, 5
    w = _weights(rng, H, P, N)
    xbc = _rand((2, 9, H * P + 2 * N), rng)
    for lo, hi in ((H * P, H * P + N), (H * P + N, H * P + 2 * N)):
        w2 = dict(w)
        w2["conv_b"] = w["conv_b"].copy()
        w2["conv_b"][lo:hi] = 0.0
        z = xbc.copy()
        z[..., lo:hi] = 0.0
        r = ssd_ref_run(z, rng, w2)
        xc, _ = ref.causal_conv1d_silu(z, w2["conv_w"], w2["conv_b"])
        xs = xc[..., : H * P].reshape(2, 9, H, P)
        np.testing.assert_allclose(r["M"].reshape(2, 9, H, P), w2["D"][None, None, :, None] * xs, rtol=1e-12,
                                   atol=1e-12)


def ssd_ref_run(xbc, rng, w):
    dt_raw = _rand(xbc.shape[:2] + (w["dt_bias"].shape[0],), np.random.default_rng(8))
    return ssd.mamba2_scan_ref(xbc, dt_raw, w)


def test_decode_equals_prefill_and_chunked_prompt():
    rng = np.random.default_rng(9)
    H, P, N = 3, 4, 5
    w = _weights(rng, H, P, N)
    xbc = _rand((2, 11, H * P + 2 * N), rng)
    dt_raw = _rand((2, 11, H), rng)
    whole = ssd.mamba2_scan_ref(xbc, dt_raw, w)
    a = ssd.mamba2_scan_ref(xbc[:, :2], dt_raw[:, :2], w)       # shorter than the conv window
    b = ssd.mamba2_scan_ref(xbc[:, 2:6], dt_raw[:, 2:6], w, a["ssm_state"], a["conv_state"])
    h, cs = b["ssm_state"], b["conv_state"]
    ms = [a["M"], b["M"]]
    for t in range(6, 11):
        m, h, cs = ssd.mamba2_step_ref(xbc[:, t], dt_raw[:, t], w, h, cs)
        ms.append(m[:, None])
    np.testing.assert_allclose(np.concatenate(ms, axis=1), whole["M"], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(h, whole["ssm_state"], rtol=1e-11, atol=1e-12)
    np.testing.assert_array_equal(cs, whole["conv_state"])


def test_dt_is_softplus_of_raw_plus_bias():
    """One token from a zero state with the conv reduced to the current tap:
    y = dt (C . B) x + D x with dt = softplus(dt_raw + dt_bias)."""
    rng = np.random.default_rng(10)
    H, P, N = 2, 3, 4
    w = _weights(rng, H, P, N)
    C = H * P + 2 * N
    w["conv_w"] = np.zeros((C, 4))
    w["conv_w"][:, 3] = 1.0
    w["conv_b"] = np.zeros(C)
    xbc = _rand((1, 1, C), rng)
    dt_raw = _rand((1, 1, H), rng)
    r = ssd.mamba2_scan_ref(xbc, dt_raw, w)
    xc = ref.silu(xbc[0, 0])
    x, Bv, Cv = xc[: H * P].reshape(H, P), xc[H * P: H * P + N], xc[H * P + N:]
    dt = np.log1p(np.exp(dt_raw[0, 0] + w["dt_bias"]))
    want = (dt * (Cv @ Bv))[:, None] * x + w["D"][:, None] * x
    np.testing.assert_allclose(r["M"][0, 0], want.ravel(), rtol=1e-12)

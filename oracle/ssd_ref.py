"""Plain float64 CPU oracle for the SambaY-2 memory readout: the Mamba-2 scan.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The ablation table of "Decoder-Hybrid-Decoder Architecture for Efficient
Reasoning with Long Generation" (Paper-Notes page, 实验关键数据 > 消融实验,
row "SambaY-2 (Mamba→Mamba-2)") swaps the self-decoder's Mamba layers for
Mamba-2, whose forget gate is one scalar per head.  The pages print none of
Mamba-2's steps; they are taken from the Mamba-2 paper (Dao & Gu 2024,
"Transformers are SSMs", the SSD layer), used as mathematics only:

    per head h (P channels), one scalar decay a_t = exp(dt_t A_h), A_h < 0,
    state H in R^{P x N}, B_t, C_t in R^N shared by the heads (one group):
        H_t = a_t H_{t-1} + dt_t x_t B_t^T          (x_t in R^P)
        y_t = H_t C_t + D_h x_t
    with dt_t = softplus(dt_raw_t + dt_bias_h), and the causal depthwise conv
    + SiLU applied to the concatenation [x | B | C] before the split.

As for Mamba-1, the memory M is the readout y before the layer's gate, norm
and out_proj.

Shapes (ngroups = 1):
    xbc     [Bt, L, H*P + 2N]   the in_proj slice [x | B | C] before the conv
    dt_raw  [Bt, L, H]          the in_proj dt slice
    x       [Bt, L, H, P]   dt [Bt, L, H]   Bm, Cm [Bt, L, N]
    A, D, dt_bias [H]       conv_w [H*P + 2N, K]   conv_b [H*P + 2N]
    ssm_state [Bt, H, P, N]     conv_state [Bt, H*P + 2N, K]
"""

from __future__ import annotations

import numpy as np

from .sambay_ref import causal_conv1d_silu, softplus

__all__ = [
    "ssd_recurrent",
    "ssd_chunked",
    "ssd_matrix",
    "mamba2_scan_ref",
    "mamba2_step_ref",
]


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def ssd_recurrent(x, dt, A, Bm, Cm, D, h0=None):
    """The SSD recurrence token by token (definition above): returns
    (y [Bt, L, H, P], final state [Bt, H, P, N])."""
    x, dt, A, Bm, Cm, D = map(_f64, (x, dt, A, Bm, Cm, D))
    Bt, L, H, P = x.shape
    N = Bm.shape[-1]
    h = np.zeros((Bt, H, P, N)) if h0 is None else _f64(h0).copy()
    y = np.empty((Bt, L, H, P))
    for t in range(L):
        a = np.exp(dt[:, t] * A)                                    # [Bt, H]
        u = dt[:, t, :, None] * x[:, t]                             # [Bt, H, P]
        h = a[:, :, None, None] * h + u[..., None] * Bm[:, t, None, None, :]
        y[:, t] = np.einsum("bhpn,bn->bhp", h, Cm[:, t]) + D[None, :, None] * x[:, t]
    return y, h


def ssd_matrix(dt, A, Bm, Cm):
    """The SSD mixing matrices, one per (sequence, head): for s <= t
        Mix[b, h, t, s] = (C_t . B_s) exp(A_h sum_{s < k <= t} dt_k) dt_s
    and 0 above the diagonal, so that y = Mix x + D x from a zero state.
    This is the 2-D A_ij of the lifted-tensor identity (Paper-Notes page,
    方法详解 > 关键设计) in its exact form: one matrix shared by the head's P
    channels."""
    dt, A, Bm, Cm = map(_f64, (dt, A, Bm, Cm))
    Bt, L, H = dt.shape
    cs = np.cumsum(dt, axis=1)                                      # [Bt, L, H]
    CB = np.einsum("btn,bsn->bts", Cm, Bm)                          # [Bt, L, L]
    mix = np.zeros((Bt, H, L, L))
    for t in range(L):
        for s in range(t + 1):
            decay = np.exp(A * (cs[:, t] - cs[:, s]))               # [Bt, H]
            mix[:, :, t, s] = CB[:, t, s][:, None] * decay * dt[:, s]
    return mix


def ssd_chunked(x, dt, A, Bm, Cm, D, h0=None, chunk=64):
    """The same readout computed chunk by chunk, the form a tensor-core
    kernel uses.  Within a chunk with cumulative log-decays
    c_t = A sum_{k <= t, k in chunk} dt_k:
        intra   y_t += sum_{s <= t} (C_t . B_s) exp(c_t - c_s) dt_s x_s
        carry   y_t += exp(c_t) H_in C_t
        state   H_out = exp(c_end) H_in + sum_s exp(c_end - c_s) dt_s x_s B_s^T
    Returns (y, final state) like ssd_recurrent."""
    x, dt, A, Bm, Cm, D = map(_f64, (x, dt, A, Bm, Cm, D))
    Bt, L, H, P = x.shape
    N = Bm.shape[-1]
    h = np.zeros((Bt, H, P, N)) if h0 is None else _f64(h0).copy()
    y = np.empty((Bt, L, H, P))
    for c0 in range(0, L, chunk):
        c1 = min(L, c0 + chunk)
        xc, dtc, Bc, Cc = x[:, c0:c1], dt[:, c0:c1], Bm[:, c0:c1], Cm[:, c0:c1]
        cl = np.cumsum(dtc, axis=1) * A                              # [Bt, Q, H]
        CB = np.einsum("btn,bsn->bts", Cc, Bc)                       # [Bt, Q, Q]
        Q = c1 - c0
        seg = cl[:, :, None, :] - cl[:, None, :, :]                  # [Bt, t, s, H]
        causal = np.tril(np.ones((Q, Q), dtype=bool))
        W = np.where(causal[None, :, :, None], CB[..., None] * np.exp(np.where(causal[None, :, :, None], seg, 0.0)),
                     0.0) * dtc[:, None, :, :]                       # [Bt, t, s, H]
        intra = np.einsum("btsh,bshp->bthp", W, xc)
        carry = np.exp(cl)[..., None] * np.einsum("bhpn,btn->bthp", h, Cc)
        y[:, c0:c1] = intra + carry + D[None, None, :, None] * xc
        wend = np.exp(cl[:, -1:, :] - cl) * dtc                      # [Bt, Q, H]
        h = np.exp(cl[:, -1])[:, :, None, None] * h + np.einsum("bsh,bshp,bsn->bhpn", wend, xc, Bc)
    return y, h


def _split_xbc(xc, H, P, N):
    Bt, L, _ = xc.shape
    x = xc[..., : H * P].reshape(Bt, L, H, P)
    return x, xc[..., H * P: H * P + N], xc[..., H * P + N: H * P + 2 * N]


def mamba2_scan_ref(xbc, dt_raw, w, ssm_state=None, conv_state=None):
    """The SambaY-2 memory readout over a prompt: the causal conv + SiLU of
    [x | B | C] (left context = the conv state, zeros for a fresh prompt),
    dt = softplus(dt_raw + dt_bias), then the SSD recurrence.

    w: conv_w [C, K], conv_b [C], dt_bias [H], A [H], D [H]; headdim P and
    d_state N from w["P"], w["N"].
    Returns dict(M [Bt, L, H*P], ssm_state [Bt, H, P, N], conv_state [Bt, C, K])."""
    xbc, dt_raw = _f64(xbc), _f64(dt_raw)
    H, P, N = int(w["dt_bias"].shape[0]), int(w["P"]), int(w["N"])
    xc, cs = causal_conv1d_silu(xbc, w["conv_w"], w["conv_b"], conv_state)
    x, Bm, Cm = _split_xbc(xc, H, P, N)
    dt = softplus(dt_raw + _f64(w["dt_bias"])[None, None, :])
    y, h = ssd_recurrent(x, dt, w["A"], Bm, Cm, w["D"], ssm_state)
    Bt, L = xbc.shape[:2]
    return {"M": y.reshape(Bt, L, H * P), "ssm_state": h, "conv_state": cs}


def mamba2_step_ref(xbc_t, dt_raw_t, w, ssm_state, conv_state):
    """One decode token per sequence: the prompt readout with L = 1 on the
    carried state.  xbc_t [Bt, C], dt_raw_t [Bt, H].  Returns (m_t [Bt, H*P],
    ssm_state, conv_state)."""
    r = mamba2_scan_ref(_f64(xbc_t)[:, None], _f64(dt_raw_t)[:, None], w, ssm_state, conv_state)
    return r["M"][:, 0], r["ssm_state"], r["conv_state"]

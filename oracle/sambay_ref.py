"""Plain float64 CPU oracle for the SambaY scan -> memory readout -> GMU path.

TEST INFRASTRUCTURE ONLY (see the package docstring).  Every function takes
NumPy arrays (any float dtype; they are widened to float64 first) and returns
float64 arrays.  Shapes follow the C-ABI:

    u, M      [B, L, Di]   token-major, channel fastest
    conv_w    [Di, K]      conv_b [Di]
    x_proj_w  [R + 2N, Di] rows [0,R) -> delta, [R,R+N) -> B, [R+N,R+2N) -> C
    dt_proj_w [Di, R]      dt_bias [Di]
    A         [Di, N]      (negative)   D [Di]
    ssm_state [B, Di, N]   conv_state [B, Di, K] (last K inputs, oldest first)
    X, Y      [T, Dm]      W1, W2 [Di, Dm]

Readings of points the sources leave open are stated where they are used
(conv tap order, B discretisation, what M is, ...).
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "silu",
    "softplus",
    "causal_conv1d_silu",
    "x_proj",
    "dt_softplus",
    "selective_scan",
    "scan_prefill_ref",
    "scan_step_ref",
    "gmu_ref",
    "gmu_layers_ref",
    "mixing_matrix_ref",
    "lifted_gmu_ref",
]


def _f64(a):
    return np.asarray(a, dtype=np.float64)


# --------------------------------------------------------------------------
# Elementwise functions
# --------------------------------------------------------------------------

def silu(x):
    """SiLU(x) = x * sigmoid(x) = x / (1 + e^-x).

    The activation the Paper-Notes page names for sigma in the GMU equation
    (方法详解 > 关键设计, Gated Memory Unit), also Mamba's post-conv activation.
    Written via the logistic function so large |x| neither overflows nor
    loses the sign.
    """
    x = _f64(x)
    with np.errstate(over="ignore"):
        return x / (1.0 + np.exp(-x))


def softplus(x):
    """softplus(x) = log(1 + e^x), exactly (no linear cut-over).

    Mamba section 3.2 / Algorithm 2: Δ = softplus(parameter + s_Δ(x)).
    ``np.logaddexp(0, x)`` is log(e^0 + e^x) evaluated without overflow.
    """
    return np.logaddexp(0.0, _f64(x))


# --------------------------------------------------------------------------
# Mamba selective SSM, step by step (Gu & Dao 2023, section 3.2, Algorithm 2)
# --------------------------------------------------------------------------

def causal_conv1d_silu(u, conv_w, conv_b, conv_state=None):
    """Causal depthwise conv over time, then SiLU (Mamba block, section 3.4).

    uc[b, t, c] = SiLU(conv_b[c] + sum_k conv_w[c, k] * ucat[b, t + k, c])

    where ucat is the input with K-1 steps of left context prepended: the last
    K-1 entries of ``conv_state`` (time order, oldest first), or zeros for a
    fresh prompt.  Reading: cross-correlation order, so conv_w[c, K-1]
    multiplies the current token (the PyTorch conv1d convention Mamba uses).

    Returns (uc [B, L, Di], new_conv_state [B, Di, K]) where the new state is
    the last K inputs seen (zeros where fewer than K were ever seen).
    """
    u = _f64(u)
    w = _f64(conv_w)
    bias = _f64(conv_b)
    Bsz, L, Di = u.shape
    K = w.shape[1]
    if conv_state is None:
        left = np.zeros((Bsz, K - 1, Di))
        hist = np.zeros((Bsz, K, Di))
    else:
        cs = _f64(conv_state)                      # [B, Di, K]
        left = np.transpose(cs[:, :, 1:], (0, 2, 1))   # last K-1 inputs
        hist = np.transpose(cs, (0, 2, 1))
    ucat = np.concatenate([left, u], axis=1)       # [B, L + K - 1, Di]
    pre = np.empty((Bsz, L, Di))
    for t in range(L):
        window = ucat[:, t:t + K, :]               # [B, K, Di], oldest first
        pre[:, t, :] = bias[None, :] + np.einsum("bkc,ck->bc", window, w)
    uc = silu(pre)
    full = np.concatenate([hist, u], axis=1)       # everything seen, in order
    new_state = np.transpose(full[:, -K:, :], (0, 2, 1)).copy()
    return uc, new_state


def x_proj(uc, x_proj_w, dt_rank, d_state):
    """Input-dependent projections s_B(x), s_C(x) and the low-rank s_Δ input.

    [delta | Bm | Cm] = uc @ x_proj_w^T  (Mamba section 3.2, Algorithm 2 steps
    2-4; the shared low-rank Δ projection of section 3.6).  B and C are shared
    by all channels of a token; delta feeds dt_proj.
    """
    xdbl = _f64(uc) @ _f64(x_proj_w).T
    R, N = dt_rank, d_state
    return xdbl[..., :R], xdbl[..., R:R + N], xdbl[..., R + N:R + 2 * N]


def dt_softplus(delta, dt_proj_w, dt_bias):
    """Δ = softplus(delta @ dt_proj_w^T + dt_bias) (Mamba Algorithm 2 step 4)."""
    return softplus(_f64(delta) @ _f64(dt_proj_w).T + _f64(dt_bias))


def selective_scan(uc, dt, A, Bm, Cm, D, h0=None):
    """The selective SSM recurrence and its readout, one token at a time.

    h_t[c, n] = exp(Δ_t[c] A[c, n]) h_{t-1}[c, n] + Δ_t[c] Bm_t[n] uc_t[c]
    y_t[c]    = sum_n Cm_t[n] h_t[c, n] + D[c] uc_t[c]

    Discretisation: Ā = exp(ΔA) (zero-order hold) with the simplified
    B̄ = ΔB (Mamba section 3.2 / Algorithm 2, the form its reference kernels
    use).  h0 is zero for a fresh prompt.  The readout y is the token-mixing
    output M^(l') that the GMU reuses (Paper-Notes, 关键设计; "memory readout
    states" in the abstract): it is taken before Mamba's own SiLU(z) output
    gate and before out_proj, with the D skip term included.

    uc, dt: [B, L, Di];  A: [Di, N];  Bm, Cm: [B, L, N];  D: [Di].
    Returns (y [B, L, Di], h_last [B, Di, N]).
    """
    uc, dt, A, Bm, Cm, D = map(_f64, (uc, dt, A, Bm, Cm, D))
    Bsz, L, Di = uc.shape
    N = A.shape[1]
    h = np.zeros((Bsz, Di, N)) if h0 is None else _f64(h0).copy()
    y = np.empty((Bsz, L, Di))
    for t in range(L):
        dA = np.exp(dt[:, t, :, None] * A[None, :, :])                  # [B,Di,N]
        dBu = (dt[:, t, :] * uc[:, t, :])[:, :, None] * Bm[:, t, None, :]
        h = dA * h + dBu
        y[:, t, :] = np.einsum("bcn,bn->bc", h, Cm[:, t, :]) + D[None, :] * uc[:, t, :]
    return y, h


def scan_prefill_ref(u, w, ssm_state=None, conv_state=None):
    """One Mamba scan over a prompt: conv -> x_proj -> Δ -> scan -> M.

    ``w`` is a dict with conv_w, conv_b, x_proj_w, dt_proj_w, dt_bias, A, D,
    dt_rank, d_state.  ``ssm_state``/``conv_state`` None means a fresh prompt
    (zero state); otherwise the prompt continues the given state.

    Returns dict(M, ssm_state, conv_state, uc, dt, Bm, Cm, delta).
    """
    uc, cs = causal_conv1d_silu(u, w["conv_w"], w["conv_b"], conv_state)
    delta, Bm, Cm = x_proj(uc, w["x_proj_w"], w["dt_rank"], w["d_state"])
    dt = dt_softplus(delta, w["dt_proj_w"], w["dt_bias"])
    M, h = selective_scan(uc, dt, w["A"], Bm, Cm, w["D"], ssm_state)
    return dict(M=M, ssm_state=h, conv_state=cs, uc=uc, dt=dt, Bm=Bm, Cm=Cm,
                delta=delta)


def scan_step_ref(u_t, w, ssm_state, conv_state):
    """One decode step: the prefill with L = 1 on the carried state.

    The decode state is the fixed-size pair (h [B, Di, N], conv window
    [B, Di, K]), independent of position (Paper-Notes, 关键设计 design
    motivation: decoding keeps a constant-size state instead of a KV cache).

    u_t [B, Di] -> (m_t [B, Di], new ssm_state, new conv_state).
    """
    r = scan_prefill_ref(_f64(u_t)[:, None, :], w, ssm_state, conv_state)
    return r["M"][:, 0, :], r["ssm_state"], r["conv_state"]


# --------------------------------------------------------------------------
# Gated Memory Unit (Paper-Notes, 方法详解 > 关键设计)
# --------------------------------------------------------------------------

def gmu_ref(X, M, W1, W2, residual=False):
    """Y = (M ⊙ SiLU(X W1^T)) W2, plus X when ``residual``.

    X [T, Dm], M [T, Di], W1 [Di, Dm], W2 [Di, Dm] (the equation multiplies
    by W2 on the right, so W2 maps Di -> Dm).  Returns (Y, G, H) with the
    gate G = SiLU(X W1^T) and H = M ⊙ G.
    """
    X, M, W1, W2 = map(_f64, (X, M, W1, W2))
    G = silu(X @ W1.T)
    H = M * G
    Y = H @ W2
    if residual:
        Y = Y + X
    return Y, G, H


def gmu_layers_ref(X, M, W1s, W2s):
    """Cross-decoder sharing: one memory readout M feeds a stack of GMUs.

    X_{l+1} = X_l + GMU_l(X_l, M) for each (W1_l, W2_l); every layer reads the
    same M (Paper-Notes, 整体框架: the cross-decoder's GMU layers reuse the
    last SSM layer's token-mixing output).  Returns the final X.
    """
    X = _f64(X)
    for W1, W2 in zip(W1s, W2s):
        X, _, _ = gmu_ref(X, M, W1, W2, residual=True)
    return X


# --------------------------------------------------------------------------
# The mixing-matrix view (Paper-Notes, 关键设计 and 亮点与洞察)
# --------------------------------------------------------------------------

def mixing_matrix_ref(dt, A, Bm, Cm, D):
    """Materialise the scan's lower-triangular token-mixing matrices.

    For one sequence (dt [L, Di], Bm/Cm [L, N]) and each channel c:

        A^(c)[i, j] = sum_n Cm_i[n] exp(A[c, n] sum_{s=j+1..i} Δ_s[c]) Δ_j[c] Bm_j[n]
                      for j <= i, else 0;  plus D[c] on the diagonal,

    so that y[:, c] = A^(c) @ uc[:, c] for a zero initial state (unrolling the
    recurrence of :func:`selective_scan`).  Mamba-1 mixes per channel, so the
    page's 2-D A_ij carries a channel index here.  Brute force: O(L^2 Di N).
    Returns an array [Di, L, L].
    """
    dt, A, Bm, Cm, D = map(_f64, (dt, A, Bm, Cm, D))
    L, Di = dt.shape
    out = np.zeros((Di, L, L))
    for c in range(Di):
        for i in range(L):
            for j in range(i + 1):
                decay = np.exp(A[c, :] * dt[j + 1:i + 1, c].sum())   # [N]
                out[c, i, j] = np.sum(Cm[i, :] * decay * dt[j, c] * Bm[j, :])
            out[c, i, i] += D[c]
    return out


def lifted_gmu_ref(uc, G, mix, W2):
    """GMU output through the lifted 3-D mixing tensor Ã_ijk = G_ik A_ij.

    Paper-Notes (关键设计): gating by G lifts the token-mixing matrix to a
    3-D tensor that re-weights each channel's mixing.  With the per-channel
    matrices of :func:`mixing_matrix_ref` (mix [Di, L, L]):

        Ã[i, j, k] = G[i, k] * mix[k, i, j]
        Y          = (sum_j Ã[:, j, :] * uc[j, :]) @ W2

    for one sequence (uc [L, Di], G [L, Di]).  Returns Y [L, Dm].
    """
    uc, G, mix, W2 = map(_f64, (uc, G, mix, W2))
    L, Di = uc.shape
    At = np.einsum("ik,kij->ijk", G, mix)          # [L, L, Di]
    H = np.einsum("ijk,jk->ik", At, uc)            # [L, Di]
    return H @ W2

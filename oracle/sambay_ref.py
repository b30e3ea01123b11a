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
    "round_bf16",
    "mamba_layer_ref",
    "mlp_representation_ref",
    "sambay_mlp_gmu_ref",
    "cross_attention_decode_ref",
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
# The bf16 I/O type
# --------------------------------------------------------------------------

def round_bf16(x):
    """Round to the nearest bfloat16 value, ties to even; float64 out.

    bfloat16 keeps 8 significant bits: for |x| in [2^(e-1), 2^e) the spacing
    is 2^(e-8), and below the smallest normal 2^-126 it stays 2^-133.  Only
    used where a caller-visible tensor of a bf16 workload passes between two
    calls (the I/O of the cross-decoder's layers); finite inputs only.
    """
    x = _f64(x)
    _, e = np.frexp(x)                      # x = m 2^e, 0.5 <= |m| < 1
    e = np.maximum(e, -125)                 # normal range of bf16: 2^-126 and up
    ulp = np.ldexp(1.0, e - 8)
    return np.rint(x / ulp) * ulp           # np.rint rounds half to even


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


def gmu_layers_ref(X, M, W1s, W2s, io_round=False):
    """Cross-decoder sharing: one memory readout M feeds a stack of GMUs.

    X_{l+1} = X_l + GMU_l(X_l, M) for each (W1_l, W2_l); every layer reads the
    same M (Paper-Notes, 整体框架: the cross-decoder's GMU layers reuse the
    last SSM layer's token-mixing output).  Returns the final X.

    ``io_round``: the layers exchange X (and read M) as bfloat16 tensors, the
    I/O type of the bf16 workloads, so each layer's input is the bf16 rounding
    of the previous layer's exact output (:func:`round_bf16`); the arithmetic
    inside a layer stays exact.  Without it, X is carried exactly from layer
    to layer.
    """
    X = _f64(X)
    M = round_bf16(M) if io_round else _f64(M)
    for W1, W2 in zip(W1s, W2s):
        X, _, _ = gmu_ref(X, M, W1, W2, residual=True)
        if io_round:
            X = round_bf16(X)
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


# --------------------------------------------------------------------------
# Around the path: the Mamba layer that produces M, and the two neighbours of
# the GMU in the cross-decoder
# --------------------------------------------------------------------------

def mamba_layer_ref(X, w, W_in, W_z, W_out, ssm_state=None, conv_state=None, residual=True, io_round=False):
    """The whole Mamba layer whose scan readout is the shared memory M.

    Mamba block (Gu & Dao 2023, section 3.4): the input is projected into two
    branches, x = X W_in^T (the scan input u) and z = X W_z^T (the gate); the
    scan of u gives y, the layer output is (y ⊙ SiLU(z)) W_out.  The Samba
    self-decoder stacks such layers (Paper-Notes, 方法详解 > 整体框架), and M is
    the last one's y before its own gate (reading: the GMU's gate takes the
    place of SiLU(z), so M is the pre-gate readout).

    X [B, L, Dm]; W_in, W_z [Di, Dm] (the x and z halves of in_proj, used
    transposed); W_out [Di, Dm], multiplying on the right (out_proj's weight
    transposed).  Returns dict(out [B, L, Dm] (+X when ``residual``), M = y,
    z, u, ssm_state, conv_state).

    ``io_round``: the layer's steps exchange u (projection -> scan) and M
    (scan -> gated output projection) as bfloat16 tensors, the I/O type of the
    bf16 workloads; the scan then runs on the bf16 rounding of the exact u,
    and the output projection reads the bf16 rounding of the exact M.  The
    arithmetic inside each step stays float64.
    """
    X = _f64(X)
    u = X @ _f64(W_in).T
    z = X @ _f64(W_z).T
    if io_round:
        u = round_bf16(u)
    r = scan_prefill_ref(u, w, ssm_state, conv_state)
    out = ((round_bf16(r["M"]) if io_round else r["M"]) * silu(z)) @ _f64(W_out)
    if residual:
        out = out + X
    return dict(out=out, M=r["M"], z=z, u=u, ssm_state=r["ssm_state"], conv_state=r["conv_state"])


def mlp_representation_ref(X, W_g, W_u):
    """The intermediate representation of a SwiGLU MLP: SiLU(X W_g^T) ⊙ (X W_u^T).

    SambaY-MLP (Paper-Notes, 实验关键数据 > 消融实验, row "SambaY-MLP") lets the
    GMUs gate an MLP representation instead of the SSM readout; reading: the
    hidden activation of the self-decoder's last MLP, whose SwiGLU form is the
    Samba MLP.  X [T, Dm]; W_g, W_u [Dff, Dm].  Returns [T, Dff].
    """
    X = _f64(X)
    return silu(X @ _f64(W_g).T) * (X @ _f64(W_u).T)


def sambay_mlp_gmu_ref(X_cross, X_self, W_g, W_u, W1, W2, residual=False):
    """A SambaY-MLP GMU layer: the memory is the MLP representation of the
    self-decoder's input X_self, gated by the cross-decoder's X_cross.
    Returns (Y, M)."""
    M = mlp_representation_ref(X_self, W_g, W_u)
    Y, _, _ = gmu_ref(X_cross, M, W1, W2, residual=residual)
    return Y, M


def cross_attention_decode_ref(q, K, V, scale=None):
    """One decode query per sequence attending over the single KV cache.

    The cross-decoder layers that the GMU does not replace attend to the KV
    cache the self-decoder's full-attention layer wrote once (Paper-Notes,
    方法详解 > 整体框架; 研究背景与动机: the O(d_kv N) memory I/O per decoded
    token that the GMU avoids).  Standard softmax attention with grouped
    query heads:

        out[b, h] = sum_j softmax_j(scale q[b, h] . K[b, j, h // G]) V[b, j, h // G]

    q [B, Hq, dh]; K, V [B, N, Hkv, dh] with G = Hq / Hkv; scale defaults to
    1 / sqrt(dh).  Returns [B, Hq, dh].
    """
    q, K, V = map(_f64, (q, K, V))
    Bsz, Hq, dh = q.shape
    Hkv = K.shape[2]
    G = Hq // Hkv
    s = (1.0 / np.sqrt(dh)) if scale is None else float(scale)
    Kq = np.repeat(K, G, axis=2)                       # [B, N, Hq, dh]
    Vq = np.repeat(V, G, axis=2)
    logits = np.einsum("bhd,bnhd->bhn", q, Kq) * s      # [B, Hq, N]
    logits = logits - logits.max(axis=-1, keepdims=True)
    p = np.exp(logits)
    p = p / p.sum(axis=-1, keepdims=True)
    return np.einsum("bhn,bnhd->bhd", p, Vq)

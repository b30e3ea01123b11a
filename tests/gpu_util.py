"""Helpers shared by the GPU parity tests (not a test module)."""

import numpy as np

# Tolerances of the method's parity contract: max elementwise relative error
# |g - r| / (|r| + rms(r)) against the float64 oracle.
TOL_F32 = 1e-4     # float32 I/O, float32 arithmetic
TOL_BF16 = 2e-2    # bfloat16 I/O, float32 accumulation and state


def rel_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    rms = np.sqrt(np.mean(ref * ref)) + 1e-300
    return float(np.max(np.abs(got - ref) / (np.abs(ref) + rms)))


def norm_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(got - ref) / (np.linalg.norm(ref) + 1e-300))


def assert_close(got, ref, tol, what=""):
    e = rel_err(got, ref)
    n = norm_err(got, ref)
    assert np.all(np.isfinite(np.asarray(got, dtype=np.float64))), f"{what}: non-finite output"
    assert e <= tol, f"{what}: max rel err {e:.3g} > {tol} (normwise {n:.3g})"
    return e


def host(t):
    return t.float().cpu().numpy()


# A chain of L layers that pass their output to the next one as a bf16 tensor
# (the cross-decoder's X <- X + GMU_l(X, M)) rounds the residual stream L
# times: each layer's output may land on the other bf16 neighbour of the
# exact value (one bf16 step, 2^-8 relative), and that difference travels on.
# End-to-end the chain is held to the normwise limit and, elementwise, to the
# single-output limit plus one bf16 step per layer; every layer on its own is
# held to the single-output limit (assert_layers_per_layer).
def chain_tol(layers):
    return TOL_BF16 + layers * 2.0 ** -8


def assert_close_chain(got, ref, layers, what=""):
    e = rel_err(got, ref)
    n = norm_err(got, ref)
    assert np.all(np.isfinite(np.asarray(got, dtype=np.float64))), f"{what}: non-finite output"
    assert n <= TOL_BF16, f"{what}: normwise err {n:.3g} > {TOL_BF16}"
    assert e <= chain_tol(layers), f"{what}: max rel err {e:.3g} > {chain_tol(layers):.3g} (normwise {n:.3g})"
    return e


def assert_layers_per_layer(run_layer, X_full, M_full, rows, X_rows, M_rows, W1s, W2s, what=""):
    """Check each layer of a GMU chain on its own, at the single-output limit.

    The checked rows of the GPU's inputs are overwritten with the oracle's own
    chain state (bf16-rounded, as the layers exchange it), so each GPU layer
    sees exactly the input the oracle's layer sees; the other rows are filler.
    run_layer(l, X, M) runs GPU layer l on device tensors with the residual
    and returns its output."""
    import torch
    from oracle import sambay_ref as ref
    idx = torch.as_tensor(np.asarray(rows), device=X_full.device)
    x = ref.round_bf16(X_rows)
    m = ref.round_bf16(M_rows)
    Xb, Mb = X_full.clone(), M_full.clone()
    Mb[idx] = torch.from_numpy(m).to(Mb.device, Mb.dtype)
    worst = 0.0
    for l in range(len(W1s)):
        Xb[idx] = torch.from_numpy(x).to(Xb.device, Xb.dtype)
        Y = run_layer(l, Xb, Mb)
        want, _, _ = ref.gmu_ref(x, m, W1s[l], W2s[l], residual=True)
        worst = max(worst, assert_close(host(Y)[np.asarray(rows)], want, TOL_BF16, f"{what} layer {l}"))
        x = ref.round_bf16(want)
    return worst

"""Device-resident layers over the C ABI: a Mamba scan layer that produces the
memory readout M, and Gated Memory Units that reuse it.

These hold the weights and workspaces in torch-allocated device memory and
call the ABI entry points; they do no arithmetic of their own.
"""

from __future__ import annotations

import torch

from . import abi


def io_dtype(io: int) -> torch.dtype:
    return torch.bfloat16 if io == abi.BF16 else torch.float32


def to_device(a, io: int, device="cuda") -> torch.Tensor:
    """float32 numpy array (already rounded to the I/O type) -> device tensor."""
    return torch.from_numpy(a).to(device=device).to(io_dtype(io)).contiguous()


def to_device_f32(a, device="cuda") -> torch.Tensor:
    return torch.from_numpy(a).to(device=device, dtype=torch.float32).contiguous()


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


class ScanLayer:
    """The Mamba layer whose readout is the shared memory M."""

    def __init__(self, w: dict, d_model: int, io: int, device="cuda"):
        self.io = io
        self.dtype = io_dtype(io)
        self.d_inner, self.d_state = w["A"].shape
        self.d_conv = w["conv_w"].shape[1]
        self.dt_rank = w["dt_rank"]
        self.d_model = d_model
        self.conv_w = to_device(w["conv_w"], io, device)
        self.conv_b = to_device(w["conv_b"], io, device)
        self.x_proj_w = to_device(w["x_proj_w"], io, device)
        self.dt_proj_w = to_device(w["dt_proj_w"], io, device)
        self.dt_bias = to_device_f32(w["dt_bias"], device)
        self.A = to_device_f32(w["A"], device)
        self.D = to_device_f32(w["D"], device)
        self.abi_w = abi.make_weights(self.conv_w, self.conv_b, self.x_proj_w, self.dt_proj_w,
                                      self.dt_bias, self.A, self.D)
        self.device = device
        self._ws = {}

    def dims(self, batch: int, seqlen: int) -> abi.Dims:
        return abi.make_dims(batch, seqlen, self.d_model, self.d_inner, self.d_state, self.d_conv,
                             self.dt_rank, self.io)

    def _workspace(self, key, nbytes):
        ws = self._ws.get(key)
        if ws is None or ws.numel() < nbytes:
            ws = workspace(nbytes, self.device)
            self._ws[key] = ws
        return ws

    def new_state(self, batch: int):
        h = torch.zeros(batch, self.d_inner, self.d_state, dtype=torch.float32, device=self.device)
        cs = torch.zeros(batch, self.d_inner, self.d_conv, dtype=self.dtype, device=self.device)
        return h, cs

    def prefill(self, u, ssm_state=None, conv_state=None, M=None, fresh=None, stream=None):
        """u [B, L, Di] -> M [B, L, Di].  Without states (or with fresh=True)
        the prompt starts from zero state; otherwise it continues the given
        states.  States are returned and updated in place."""
        B, L, _ = u.shape
        if fresh is None:
            fresh = ssm_state is None
        if ssm_state is None:
            ssm_state, conv_state = self.new_state(B)
        if M is None:
            M = torch.empty_like(u)
        d = self.dims(B, L)
        ws = self._workspace(("prefill", B, L), abi.sambay_scan_prefill_workspace(d))
        abi.sambay_scan_prefill(self.abi_w, d, u, M, ssm_state, conv_state, fresh, ws, stream)
        return M, ssm_state, conv_state

    def step(self, u_t, ssm_state, conv_state, m_t=None, stream=None):
        """u_t [B, Di] -> m_t [B, Di]; states updated in place."""
        B = u_t.shape[0]
        if m_t is None:
            m_t = torch.empty_like(u_t)
        d = self.dims(B, 1)
        ws = self._workspace(("step", B), abi.sambay_scan_step_workspace(d))
        abi.sambay_scan_step(self.abi_w, d, u_t, m_t, ssm_state, conv_state, ws, stream)
        return m_t


class GMULayer:
    """Y = (M ⊙ SiLU(X W1^T)) W2 (+ X)."""

    def __init__(self, W1, W2, io: int, device="cuda"):
        self.io = io
        self.W1 = to_device(W1, io, device)
        self.W2 = to_device(W2, io, device)
        self.d_inner, self.d_model = W1.shape
        self.device = device
        self._ws = {}

    def dims(self, rows: int) -> abi.Dims:
        return abi.make_dims(rows, 1, self.d_model, self.d_inner, 16, 4, 4, self.io)

    def _workspace(self, key, nbytes):
        ws = self._ws.get(key)
        if ws is None or ws.numel() < nbytes:
            ws = workspace(nbytes, self.device)
            self._ws[key] = ws
        return ws

    def forward(self, X, M, residual=False, Y=None, stream=None):
        rows = X.shape[0]
        if Y is None:
            Y = torch.empty_like(X)
        d = self.dims(rows)
        ws = self._workspace(("fwd", rows), abi.gmu_forward_workspace(d, rows))
        abi.gmu_forward(d, rows, X, M, self.W1, self.W2, X if residual else None, Y, ws, stream)
        return Y

    def step(self, X, M, residual=False, Y=None, stream=None):
        rows = X.shape[0]
        if Y is None:
            Y = torch.empty_like(X)
        d = self.dims(rows)
        ws = self._workspace(("step", rows), abi.gmu_step_workspace(d, rows))
        abi.gmu_step(d, rows, X, M, self.W1, self.W2, X if residual else None, Y, ws, stream)
        return Y


class DecodeChain:
    """One decode token through the scan and a stack of GMU layers that reuse
    its readout: m_t = scan step(u_t); X <- X + GMU_l(X, m_t) for each layer,
    as one sambay_decode_step call (states and X updated in place)."""

    def __init__(self, scan: ScanLayer, gmus):
        self.scan = scan
        self.gmus = list(gmus)
        self.layers = abi.make_gmu_layers([(g.W1, g.W2) for g in self.gmus])
        self._ws = {}

    def step(self, u_t, ssm_state, conv_state, X, m_t=None, stream=None):
        B = u_t.shape[0]
        if m_t is None:
            m_t = torch.empty_like(u_t)
        d = self.scan.dims(B, 1)
        n = len(self.gmus)
        ws = self._ws.get(B)
        need = abi.sambay_decode_step_workspace(d, n)
        if ws is None or ws.numel() < need:
            ws = workspace(need, self.scan.device)
            self._ws[B] = ws
        abi.sambay_decode_step(self.scan.abi_w, d, u_t, m_t, ssm_state, conv_state, self.layers, n,
                               X if n else None, ws, stream)
        return m_t


class MambaLayer:
    """The whole Mamba layer whose scan readout is the shared memory M:
    u = X W_in^T, y = scan(u) (= M), out = (y ⊙ SiLU(X W_z^T)) W_out + X.
    The gated output projection is the GMU's computation with W1 = W_z and
    W2 = W_out, so it runs through gmu_forward / gmu_step."""

    def __init__(self, w: dict, bw: dict, d_model: int, io: int, device="cuda"):
        self.scan = ScanLayer(w, d_model, io, device)
        self.W_in = to_device(bw["W_in"], io, device)
        self.gate = GMULayer(bw["W_z"], bw["W_out"], io, device)
        self.io, self.device = io, device
        self.d_model, self.d_inner = d_model, self.scan.d_inner
        self._ws = {}

    def _proj(self, X2, u2, stream):
        rows = X2.shape[0]
        d = self.gate.dims(rows)
        ws = self._ws.get(rows)
        need = abi.sambay_in_proj_workspace(d, rows)
        if ws is None or ws.numel() < need:
            ws = workspace(need, self.device)
            self._ws[rows] = ws
        abi.sambay_in_proj(d, rows, X2, self.W_in, u2, ws, stream)

    def prefill(self, X, ssm_state=None, conv_state=None, fresh=None, stream=None):
        """X [B, L, Dm] -> (out [B, L, Dm], M [B, L, Di], ssm_state, conv_state)."""
        B, L, Dm = X.shape
        X2 = X.reshape(B * L, Dm)
        u = torch.empty(B, L, self.d_inner, dtype=X.dtype, device=X.device)
        self._proj(X2, u.view(B * L, self.d_inner), stream)
        M, h, cs = self.scan.prefill(u, ssm_state, conv_state, fresh=fresh, stream=stream)
        out = self.gate.forward(X2, M.view(B * L, self.d_inner), residual=True, stream=stream)
        return out.view(B, L, Dm), M, h, cs

    def step(self, x_t, ssm_state, conv_state, stream=None):
        """x_t [B, Dm] -> (out_t [B, Dm], m_t [B, Di]); states updated in place."""
        u_t = torch.empty(x_t.shape[0], self.d_inner, dtype=x_t.dtype, device=x_t.device)
        self._proj(x_t, u_t, stream)
        m_t = self.scan.step(u_t, ssm_state, conv_state, stream=stream)
        out = self.gate.step(x_t, m_t, residual=True, stream=stream)
        return out, m_t


class MLPMemory:
    """SambaY-MLP's memory: the SwiGLU hidden activation SiLU(X W_g^T) ⊙ (X W_u^T)."""

    def __init__(self, W_g, W_u, io: int, device="cuda"):
        self.W_g = to_device(W_g, io, device)
        self.W_u = to_device(W_u, io, device)
        self.d_ff, self.d_model = W_g.shape
        self.io, self.device = io, device
        self._ws = {}

    def forward(self, X, M=None, stream=None):
        rows = X.shape[0]
        if M is None:
            M = torch.empty(rows, self.d_ff, dtype=X.dtype, device=X.device)
        d = abi.make_dims(rows, 1, self.d_model, self.d_ff, 16, 4, 4, self.io)
        ws = self._ws.get(rows)
        need = abi.sambay_mlp_memory_workspace(d, rows)
        if ws is None or ws.numel() < need:
            ws = workspace(need, self.device)
            self._ws[rows] = ws
        abi.sambay_mlp_memory(d, rows, X, self.W_g, self.W_u, M, ws, stream)
        return M


class Mamba2Scan:
    """The SambaY-2 memory: a Mamba-2 (SSD) layer's readout over a prompt."""

    def __init__(self, w: dict, io: int = abi.BF16, device="cuda"):
        self.io = io
        self.dtype = io_dtype(io)
        self.nheads = int(w["A"].shape[0])
        self.headdim = int(w["P"])
        self.d_state = int(w["N"])
        self.channels, self.d_conv = w["conv_w"].shape
        self.conv_w = to_device(w["conv_w"], io, device)
        self.conv_b = to_device(w["conv_b"], io, device)
        self.dt_bias = to_device_f32(w["dt_bias"], device)
        self.A = to_device_f32(w["A"], device)
        self.D = to_device_f32(w["D"], device)
        self.abi_w = abi.SsdWeights(self.conv_w.data_ptr(), self.conv_b.data_ptr(), self.dt_bias.data_ptr(),
                                    self.A.data_ptr(), self.D.data_ptr())
        self.device = device
        self._ws = {}

    def dims(self, batch: int, seqlen: int) -> abi.SsdDims:
        return abi.SsdDims(batch, seqlen, self.nheads, self.headdim, self.d_state, self.d_conv, self.io)

    def new_state(self, batch: int):
        h = torch.zeros(batch, self.nheads, self.headdim, self.d_state, dtype=torch.float32, device=self.device)
        cs = torch.zeros(batch, self.channels, self.d_conv, dtype=self.dtype, device=self.device)
        return h, cs

    def prefill(self, xbc, dt_raw, ssm_state=None, conv_state=None, M=None, fresh=None, stream=None):
        """xbc [B, L, C], dt_raw [B, L, H] -> M [B, L, H * P]; states as for
        ScanLayer.prefill (returned, updated in place)."""
        B, L, _ = xbc.shape
        if fresh is None:
            fresh = ssm_state is None
        if ssm_state is None:
            ssm_state, conv_state = self.new_state(B)
        if M is None:
            M = torch.empty(B, L, self.nheads * self.headdim, dtype=self.dtype, device=self.device)
        d = self.dims(B, L)
        n = abi.sambay_ssd_prefill_workspace(d)
        ws = self._ws.get((B, L))
        if ws is None:
            ws = workspace(n, self.device)
            self._ws[(B, L)] = ws
        abi.sambay_ssd_prefill(self.abi_w, d, xbc, dt_raw, M, ssm_state, conv_state, fresh, ws, stream)
        return M, ssm_state, conv_state

    def step(self, xbc_t, dt_raw_t, ssm_state, conv_state, m_t=None, stream=None):
        """xbc_t [B, C], dt_raw_t [B, H] -> m_t [B, H * P]; states updated in place."""
        B = xbc_t.shape[0]
        if m_t is None:
            m_t = torch.empty(B, self.nheads * self.headdim, dtype=self.dtype, device=self.device)
        d = self.dims(B, 1)
        n = abi.sambay_ssd_step_workspace(d)
        ws = self._ws.get(("step", B))
        if ws is None:
            ws = workspace(n, self.device)
            self._ws[("step", B)] = ws
        abi.sambay_ssd_step(self.abi_w, d, xbc_t, dt_raw_t, m_t, ssm_state, conv_state, ws, stream)
        return m_t

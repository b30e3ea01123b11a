"""Thin ctypes binding of libsambay (the C ABI in ``include/sambay.h``).

Argument marshalling only: every function takes torch tensors that already
live on the current CUDA device, passes their ``data_ptr()`` and the current
CUDA stream to the C entry point of the same name, and raises
:class:`SambayError` on a non-OK status.  There is no fallback: if the
library has not been built, importing the symbols raises.
"""

from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "lib", "libsambay.so")

F32 = 0
BF16 = 1

STATUS = {
    0: "SAMBAY_OK",
    1: "SAMBAY_ERR_INVALID_ARG",
    2: "SAMBAY_ERR_UNSUPPORTED",
    3: "SAMBAY_ERR_WORKSPACE",
    4: "SAMBAY_ERR_CUDA",
    5: "SAMBAY_ERR_TIMEOUT",
    6: "SAMBAY_ERR_DEVICE",
}

EXPORTS = (
    "sambay_scan_prefill_workspace",
    "sambay_scan_step_workspace",
    "gmu_forward_workspace",
    "gmu_step_workspace",
    "sambay_scan_prefill",
    "sambay_scan_prefill_xproj",
    "sambay_scan_prefill_finish",
    "sambay_scan_step",
    "sambay_scan_step_noalloc",
    "gmu_forward",
    "gmu_forward_partial",
    "gmu_finish",
    "gmu_step",
    "sambay_in_proj_workspace",
    "sambay_in_proj",
    "sambay_mlp_memory_workspace",
    "sambay_mlp_memory",
    "sambay_decode_step_workspace",
    "sambay_decode_step",
    "sambay_cross_attn_decode_workspace",
    "sambay_cross_attn_decode",
    "sambay_ssd_prefill_workspace",
    "sambay_ssd_prefill",
    "sambay_ssd_step_workspace",
    "sambay_ssd_step",
    "sambay_gmu_step_stall_test",
    "sambay_profile_begin",
    "sambay_profile_end",
    "sambay_device_status",
    "sambay_status_string",
    "sambay_version",
)


class SambayError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} returned {STATUS.get(code, code)}")


class Dims(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("seqlen", ctypes.c_int32),
        ("d_model", ctypes.c_int32),
        ("d_inner", ctypes.c_int32),
        ("d_state", ctypes.c_int32),
        ("d_conv", ctypes.c_int32),
        ("dt_rank", ctypes.c_int32),
        ("io", ctypes.c_int32),
    ]


class ScanWeights(ctypes.Structure):
    _fields_ = [
        ("conv_w", ctypes.c_void_p),
        ("conv_b", ctypes.c_void_p),
        ("x_proj_w", ctypes.c_void_p),
        ("dt_proj_w", ctypes.c_void_p),
        ("dt_bias", ctypes.c_void_p),
        ("A", ctypes.c_void_p),
        ("D", ctypes.c_void_p),
    ]


class AttnDims(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("kv_len", ctypes.c_int32),
        ("q_heads", ctypes.c_int32),
        ("kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
    ]


class SsdDims(ctypes.Structure):
    """sambay_ssd_dims: the SambaY-2 (Mamba-2) layer's sizes."""
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("seqlen", ctypes.c_int32),
        ("nheads", ctypes.c_int32),
        ("headdim", ctypes.c_int32),
        ("d_state", ctypes.c_int32),
        ("d_conv", ctypes.c_int32),
        ("io", ctypes.c_int32),
    ]


class SsdWeights(ctypes.Structure):
    _fields_ = [
        ("conv_w", ctypes.c_void_p),
        ("conv_b", ctypes.c_void_p),
        ("dt_bias", ctypes.c_void_p),
        ("A", ctypes.c_void_p),
        ("D", ctypes.c_void_p),
    ]


class GmuWeights(ctypes.Structure):
    _fields_ = [
        ("W1", ctypes.c_void_p),
        ("W2", ctypes.c_void_p),
    ]


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libsambay once; raise if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"libsambay is not built ({path} missing): run "
            "`python -m gated_memory_sharing_b200.build` or __graft_entry__.build()")
    lib = ctypes.CDLL(path)
    vp, sz, i32, i64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_int64
    pd, pw = ctypes.POINTER(Dims), ctypes.POINTER(ScanWeights)
    pg = ctypes.POINTER(GmuWeights)
    pa = ctypes.POINTER(AttnDims)
    psd, psw = ctypes.POINTER(SsdDims), ctypes.POINTER(SsdWeights)
    sig = {
        "sambay_scan_prefill_workspace": (sz, [pd]),
        "sambay_scan_step_workspace": (sz, [pd]),
        "gmu_forward_workspace": (sz, [pd, i64]),
        "gmu_step_workspace": (sz, [pd, i64]),
        "sambay_scan_prefill": (ctypes.c_int, [pw, pd, vp, vp, vp, vp, ctypes.c_int, vp, sz, vp]),
        "sambay_scan_prefill_xproj": (ctypes.c_int, [pw, pd, vp, vp, ctypes.c_int, vp, vp, sz, vp]),
        "sambay_scan_prefill_finish": (ctypes.c_int, [pw, pd, vp, vp, vp, vp, vp, ctypes.c_int, vp, sz, vp]),
        "sambay_scan_step": (ctypes.c_int, [pw, pd, vp, vp, vp, vp, vp, sz, vp]),
        "sambay_scan_step_noalloc": (ctypes.c_int, [pw, pd, vp, vp, vp, vp, vp]),
        "gmu_forward": (ctypes.c_int, [pd, i64, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "gmu_forward_partial": (ctypes.c_int, [pd, i64, vp, vp, vp, vp, vp, vp, sz, vp]),
        "gmu_finish": (ctypes.c_int, [pd, i64, vp, vp, vp, vp]),
        "gmu_step": (ctypes.c_int, [pd, i64, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "sambay_in_proj_workspace": (sz, [pd, i64]),
        "sambay_in_proj": (ctypes.c_int, [pd, i64, vp, vp, vp, vp, sz, vp]),
        "sambay_mlp_memory_workspace": (sz, [pd, i64]),
        "sambay_mlp_memory": (ctypes.c_int, [pd, i64, vp, vp, vp, vp, vp, sz, vp]),
        "sambay_decode_step_workspace": (sz, [pd, i32]),
        "sambay_cross_attn_decode_workspace": (sz, [pa]),
        "sambay_cross_attn_decode": (ctypes.c_int, [pa, vp, vp, vp, vp, ctypes.c_float, vp, sz, vp]),
        "sambay_ssd_prefill_workspace": (sz, [psd]),
        "sambay_ssd_prefill": (ctypes.c_int, [psw, psd, vp, vp, vp, vp, vp, i32, vp, sz, vp]),
        "sambay_ssd_step_workspace": (sz, [psd]),
        "sambay_ssd_step": (ctypes.c_int, [psw, psd, vp, vp, vp, vp, vp, vp, sz, vp]),
        "sambay_decode_step": (ctypes.c_int, [pw, pd, vp, vp, vp, vp, i32, pg, vp, vp, sz, vp]),
        "sambay_gmu_step_stall_test": (ctypes.c_int, [pd, i64, vp, vp, vp, vp, vp, vp, vp, sz,
                                                      ctypes.c_uint64, vp]),
        "sambay_profile_begin": (ctypes.c_int, [ctypes.POINTER(vp), i32]),
        "sambay_profile_end": (i32, [ctypes.POINTER(ctypes.c_char_p), i32]),
        "sambay_device_status": (ctypes.c_int, [vp, ctypes.POINTER(i32)]),
        "sambay_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "sambay_version": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


# ----------------------------------------------------------------- marshalling

def _p(t):
    """Device pointer of a tensor (None -> NULL)."""
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn: str, code: int):
    if code != 0:
        raise SambayError(fn, code)


def make_dims(batch, seqlen, d_model, d_inner, d_state=16, d_conv=4, dt_rank=160, io=BF16) -> Dims:
    return Dims(batch, seqlen, d_model, d_inner, d_state, d_conv, dt_rank, io)


def make_weights(conv_w, conv_b, x_proj_w, dt_proj_w, dt_bias, A, D) -> ScanWeights:
    return ScanWeights(*(t.data_ptr() for t in (conv_w, conv_b, x_proj_w, dt_proj_w, dt_bias, A, D)))


def sambay_scan_prefill_workspace(dims: Dims) -> int:
    return load().sambay_scan_prefill_workspace(ctypes.byref(dims))


def sambay_scan_step_workspace(dims: Dims) -> int:
    return load().sambay_scan_step_workspace(ctypes.byref(dims))


def gmu_forward_workspace(dims: Dims, rows: int) -> int:
    return load().gmu_forward_workspace(ctypes.byref(dims), rows)


def gmu_step_workspace(dims: Dims, rows: int) -> int:
    return load().gmu_step_workspace(ctypes.byref(dims), rows)


def sambay_scan_prefill(weights: ScanWeights, dims: Dims, u, M, ssm_state, conv_state,
                        zero_init_state: bool, ws, stream=None):
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("sambay_scan_prefill", load().sambay_scan_prefill(
        ctypes.byref(weights), ctypes.byref(dims), _p(u), _p(M), _p(ssm_state), _p(conv_state),
        1 if zero_init_state else 0, _p(ws), ws_bytes, _stream(stream)))


def sambay_scan_prefill_xproj(weights: ScanWeights, dims: Dims, u, conv_state, zero_init_state: bool,
                              xdbl, ws, stream=None):
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("sambay_scan_prefill_xproj", load().sambay_scan_prefill_xproj(
        ctypes.byref(weights), ctypes.byref(dims), _p(u), _p(conv_state), 1 if zero_init_state else 0,
        _p(xdbl), _p(ws), ws_bytes, _stream(stream)))


def sambay_scan_prefill_finish(weights: ScanWeights, dims: Dims, u, xdbl, M, ssm_state, conv_state,
                               zero_init_state: bool, ws, stream=None):
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("sambay_scan_prefill_finish", load().sambay_scan_prefill_finish(
        ctypes.byref(weights), ctypes.byref(dims), _p(u), _p(xdbl), _p(M), _p(ssm_state), _p(conv_state),
        1 if zero_init_state else 0, _p(ws), ws_bytes, _stream(stream)))


def sambay_scan_step(weights: ScanWeights, dims: Dims, u_t, m_t, ssm_state, conv_state, ws,
                     stream=None):
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("sambay_scan_step", load().sambay_scan_step(
        ctypes.byref(weights), ctypes.byref(dims), _p(u_t), _p(m_t), _p(ssm_state),
        _p(conv_state), _p(ws), ws_bytes, _stream(stream)))


def sambay_in_proj_workspace(dims: Dims, rows: int) -> int:
    return load().sambay_in_proj_workspace(ctypes.byref(dims), rows)


def sambay_in_proj(dims: Dims, rows: int, X, W_in, u, ws, stream=None):
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("sambay_in_proj", load().sambay_in_proj(
        ctypes.byref(dims), rows, _p(X), _p(W_in), _p(u), _p(ws), ws_bytes, _stream(stream)))


def sambay_mlp_memory_workspace(dims: Dims, rows: int) -> int:
    return load().sambay_mlp_memory_workspace(ctypes.byref(dims), rows)


def sambay_mlp_memory(dims: Dims, rows: int, X, W_g, W_u, M, ws, stream=None):
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("sambay_mlp_memory", load().sambay_mlp_memory(
        ctypes.byref(dims), rows, _p(X), _p(W_g), _p(W_u), _p(M), _p(ws), ws_bytes, _stream(stream)))


def sambay_cross_attn_decode_workspace(dims: AttnDims) -> int:
    return load().sambay_cross_attn_decode_workspace(ctypes.byref(dims))


def sambay_cross_attn_decode(dims: AttnDims, q, K, V, out, scale: float, ws, stream=None):
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("sambay_cross_attn_decode", load().sambay_cross_attn_decode(
        ctypes.byref(dims), _p(q), _p(K), _p(V), _p(out), scale, _p(ws), ws_bytes, _stream(stream)))


def sambay_ssd_prefill_workspace(dims: SsdDims) -> int:
    return load().sambay_ssd_prefill_workspace(ctypes.byref(dims))


def sambay_ssd_prefill(w: SsdWeights, dims: SsdDims, xbc, dt_raw, M, ssm_state, conv_state, zero_init: bool, ws,
                       stream=None):
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("sambay_ssd_prefill", load().sambay_ssd_prefill(
        ctypes.byref(w), ctypes.byref(dims), _p(xbc), _p(dt_raw), _p(M), _p(ssm_state), _p(conv_state),
        1 if zero_init else 0, _p(ws), ws_bytes, _stream(stream)))


def sambay_ssd_step_workspace(dims: SsdDims) -> int:
    return load().sambay_ssd_step_workspace(ctypes.byref(dims))


def sambay_ssd_step(w: SsdWeights, dims: SsdDims, xbc_t, dt_raw_t, m_t, ssm_state, conv_state, ws, stream=None):
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("sambay_ssd_step", load().sambay_ssd_step(
        ctypes.byref(w), ctypes.byref(dims), _p(xbc_t), _p(dt_raw_t), _p(m_t), _p(ssm_state), _p(conv_state),
        _p(ws), ws_bytes, _stream(stream)))


def sambay_decode_step_workspace(dims: Dims, n_layers: int) -> int:
    return load().sambay_decode_step_workspace(ctypes.byref(dims), n_layers)


def make_gmu_layers(pairs):
    """Host array of GmuWeights from (W1, W2) tensor pairs."""
    arr = (GmuWeights * max(1, len(pairs)))()
    for i, (w1, w2) in enumerate(pairs):
        arr[i] = GmuWeights(w1.data_ptr(), w2.data_ptr())
    return arr


def sambay_decode_step(weights: ScanWeights, dims: Dims, u_t, m_t, ssm_state, conv_state, layers,
                       n_layers: int, X, ws, stream=None):
    """One decode token: scan step, then X <- X + GMU_l(X, m_t) for each layer
    (``layers``: the array make_gmu_layers returns)."""
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("sambay_decode_step", load().sambay_decode_step(
        ctypes.byref(weights), ctypes.byref(dims), _p(u_t), _p(m_t), _p(ssm_state), _p(conv_state),
        n_layers, layers, _p(X), _p(ws), ws_bytes, _stream(stream)))


def sambay_gmu_step_stall_test(dims: Dims, rows: int, X, M, W1, W2, residual, Y, ws,
                               wait_limit_cycles: int, stream=None):
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("sambay_gmu_step_stall_test", load().sambay_gmu_step_stall_test(
        ctypes.byref(dims), rows, _p(X), _p(M), _p(W1), _p(W2), _p(residual), _p(Y), _p(ws),
        ws_bytes, wait_limit_cycles, _stream(stream)))


# Library-owned scratch size of sambay_scan_step_noalloc (bytes, per GPU).
NOALLOC_SCRATCH_BYTES = 8 << 20


def sambay_scan_step_noalloc(weights: ScanWeights, dims: Dims, u_t, m_t, ssm_state, conv_state,
                             stream=None):
    """sambay_scan_step without a workspace argument, for callers that cannot
    allocate device memory: the library uses a fixed scratch array of its own
    (shared by all calls on a device, so calls must not overlap on the GPU)."""
    _check("sambay_scan_step_noalloc", load().sambay_scan_step_noalloc(
        ctypes.byref(weights), ctypes.byref(dims), _p(u_t), _p(m_t), _p(ssm_state),
        _p(conv_state), _stream(stream)))


def gmu_forward(dims: Dims, rows: int, X, M, W1, W2, residual, Y, ws, stream=None):
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("gmu_forward", load().gmu_forward(
        ctypes.byref(dims), rows, _p(X), _p(M), _p(W1), _p(W2), _p(residual), _p(Y), _p(ws),
        ws_bytes, _stream(stream)))


def gmu_forward_partial(dims: Dims, rows: int, X, M, W1, W2, Y_part, ws, stream=None):
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("gmu_forward_partial", load().gmu_forward_partial(
        ctypes.byref(dims), rows, _p(X), _p(M), _p(W1), _p(W2), _p(Y_part), _p(ws), ws_bytes,
        _stream(stream)))


def gmu_finish(dims: Dims, rows: int, Y_sum, residual, Y, stream=None):
    _check("gmu_finish", load().gmu_finish(
        ctypes.byref(dims), rows, _p(Y_sum), _p(residual), _p(Y), _stream(stream)))


def gmu_step(dims: Dims, rows: int, X, M, W1, W2, residual, Y, ws, stream=None):
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("gmu_step", load().gmu_step(
        ctypes.byref(dims), rows, _p(X), _p(M), _p(W1), _p(W2), _p(residual), _p(Y), _p(ws),
        ws_bytes, _stream(stream)))


class KernelTimer:
    """Times each kernel the library launches, with caller-owned CUDA events.

        with KernelTimer(max_launches=64) as kt:
            ...library calls...
        kt.durations_ms()   # [(kernel name, ms), ...] in launch order
    """

    def __init__(self, max_launches: int = 256):
        import torch
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(2 * max_launches)]
        for e in self.events:          # torch creates the CUDA event on first record
            e.record()
        torch.cuda.synchronize()
        self._handles = (ctypes.c_void_p * len(self.events))(*[e.cuda_event for e in self.events])
        self.names = []

    def __enter__(self):
        _check("sambay_profile_begin", load().sambay_profile_begin(self._handles, len(self.events)))
        return self

    def __exit__(self, *exc):
        buf = (ctypes.c_char_p * (len(self.events) // 2))()
        n = load().sambay_profile_end(buf, len(buf))
        self.names = [buf[i].decode() for i in range(n)]
        return False

    def durations_ms(self):
        return [(name, self.events[2 * i].elapsed_time(self.events[2 * i + 1]))
                for i, name in enumerate(self.names)]


def sambay_device_status(stream=None) -> int:
    code = ctypes.c_int32(0)
    _check("sambay_device_status", load().sambay_device_status(_stream(stream), ctypes.byref(code)))
    return code.value


def sambay_status_string(code: int) -> str:
    return load().sambay_status_string(code).decode()


def sambay_version() -> str:
    return load().sambay_version().decode()

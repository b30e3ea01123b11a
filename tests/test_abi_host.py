"""Host-side checks of the C ABI that need no GPU.

The library must load and export every symbol include/sambay.h declares; the
workspace queries and status strings are pure host functions; and every
argument error is reported before the library touches a device.  The error
cases below are all built so that validation fails, so no call here can reach
a kernel launch even on a GPU machine.
"""

import ctypes
import os
import re

import pytest

from gated_memory_sharing_b200 import abi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return abi.load()


def _declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names.update(re.findall(r"^SAMBAY_API\s+[^;(]*?\b(\w+)\s*\(", src, re.M))
    return names


def test_exports_every_declared_symbol(lib):
    declared = _declared_symbols()
    assert declared == set(abi.EXPORTS)
    for name in declared:
        assert hasattr(lib, name), f"libsambay does not export {name}"


def test_noalloc_limit_matches_the_header():
    src = open(os.path.join(ROOT, "include", "sambay.h")).read()
    m = re.search(r"#define\s+SAMBAY_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", src)
    assert m, "SAMBAY_NOALLOC_SCRATCH_BYTES not found in include/sambay.h"
    assert abi.NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))


def test_decode_step_argument_errors(lib):
    d = abi.make_dims(4, 1, 128, 256, 16, 4, 16, abi.BF16)
    p = _FakePtr(0x10000)
    layers = abi.make_gmu_layers([(p, p)])
    # m_t aliases u_t
    with pytest.raises(abi.SambayError) as e:
        abi.sambay_decode_step(_weights(), d, p, p, _FakePtr(0x20000), _FakePtr(0x30000), layers, 1,
                               _FakePtr(0x40000), p, 0)
    assert e.value.code == 1
    # X aliases m_t
    with pytest.raises(abi.SambayError) as e:
        abi.sambay_decode_step(_weights(), d, p, _FakePtr(0x20000), _FakePtr(0x30000), _FakePtr(0x40000),
                               layers, 1, _FakePtr(0x20000), p, 0)
    assert e.value.code == 1
    # a NULL layer weight
    bad = abi.make_gmu_layers([(p, p)])
    bad[0].W2 = None
    with pytest.raises(abi.SambayError) as e:
        abi.sambay_decode_step(_weights(), d, p, _FakePtr(0x20000), _FakePtr(0x30000), _FakePtr(0x40000),
                               bad, 1, _FakePtr(0x50000), p, 0)
    assert e.value.code == 1
    # more than 256 sequences
    with pytest.raises(abi.SambayError) as e:
        abi.sambay_decode_step(_weights(), abi.make_dims(300, 1, 128, 256, 16, 4, 16, abi.BF16), p,
                               _FakePtr(0x20000), _FakePtr(0x30000), _FakePtr(0x40000), layers, 1,
                               _FakePtr(0x50000), p, 0)
    assert e.value.code == 2
    # workspace too small for the layers' H (1 byte)
    with pytest.raises(abi.SambayError) as e:
        abi.sambay_decode_step(_weights(), d, p, _FakePtr(0x20000), _FakePtr(0x30000), _FakePtr(0x40000),
                               layers, 1, _FakePtr(0x50000), p, 0)
    assert e.value.code == 3
    # the fault-detector test entry point validates like gmu_step
    with pytest.raises(abi.SambayError) as e:
        abi.sambay_gmu_step_stall_test(d, 4, p, p, p, p, None, p, p, 0, 0)
    assert e.value.code == 1


def test_cross_attn_argument_errors(lib):
    p = _FakePtr(0x10000)
    ok = abi.AttnDims(2, 1000, 4, 2, 64)
    # 4 (sequence, KV head) pairs: the KV range splits over CTAs, whose partials need scratch
    assert abi.sambay_cross_attn_decode_workspace(ok) > 0
    assert abi.sambay_cross_attn_decode_workspace(abi.AttnDims(64, 2048, 40, 20, 64)) == 0
    for bad, code in ((abi.AttnDims(2, 100, 4, 2, 96), 2),     # head size
                      (abi.AttnDims(2, 100, 6, 4, 64), 2),     # heads not grouped evenly
                      (abi.AttnDims(2, 100, 34, 2, 64), 2),    # more than 16 query heads per KV head
                      (abi.AttnDims(0, 100, 4, 2, 64), 1)):
        assert abi.sambay_cross_attn_decode_workspace(bad) == 0
        with pytest.raises(abi.SambayError) as e:
            abi.sambay_cross_attn_decode(bad, p, _FakePtr(0x20000), _FakePtr(0x30000), _FakePtr(0x40000), 0.0, p, 0)
        assert e.value.code == code
    with pytest.raises(abi.SambayError) as e:     # NULL input
        abi.sambay_cross_attn_decode(ok, None, _FakePtr(0x20000), _FakePtr(0x30000), _FakePtr(0x40000), 0.0, p, 0)
    assert e.value.code == 1
    with pytest.raises(abi.SambayError) as e:     # NaN scale
        abi.sambay_cross_attn_decode(ok, p, _FakePtr(0x20000), _FakePtr(0x30000), _FakePtr(0x40000),
                                     float("nan"), p, 0)
    assert e.value.code == 1
    with pytest.raises(abi.SambayError) as e:     # workspace too small
        abi.sambay_cross_attn_decode(ok, p, _FakePtr(0x20000), _FakePtr(0x30000), _FakePtr(0x40000), 0.0, p, 0)
    assert e.value.code == 3


def test_status_strings_and_version(lib):
    assert abi.sambay_version() == "0.1.0"
    assert abi.sambay_status_string(0) == "ok"
    for code in range(1, 7):
        s = abi.sambay_status_string(code)
        assert s and s != "unknown status"
    assert abi.sambay_status_string(99) == "unknown status"


def test_workspace_queries(lib):
    d = abi.make_dims(1, 2048, 2560, 5120, 16, 4, 160, abi.BF16)
    T, Di, ldx, R = 2048, 5120, 192, 160
    def r256(x):
        return (x + 255) // 256 * 256
    # uc as the bf16 split pair (4 bytes per element) + x_proj split-K partials
    # (9 splits for 16 row tiles over 160 k-blocks; 54 splits of 3 k-blocks for
    # one row tile)
    # + xdbl + split delta (bf16, 2 x dt_rank padded to 192) + dt (f32)
    # + B | C regrouped into token pairs (64 floats per pair)
    Rp = 192
    want = (r256(T * Di * 4) + r256(9 * T * ldx * 4) + r256(T * ldx * 4) + r256(T * 2 * Rp * 2)
            + r256(T * Di * 4) + r256(T // 2 * 64 * 4))
    assert abi.sambay_scan_prefill_workspace(d) == want
    # bf16 decode step: conv output, x_proj partials of 128 slices of 40
    # channels, the split delta, B | C, and the single-kernel step's
    # generation word + two meeting flags per slice (a 128-byte line each)
    step64 = (r256(64 * Di * 4) + r256(128 * ldx * 64 * 4) + r256(2 * 64 * 160 * 2) + r256(64 * 32 * 4)
              + r256(16 * (1 + 2 * 128) * 8))
    assert abi.sambay_scan_step_workspace(abi.make_dims(64, 999, 2560, 5120)) == step64
    assert step64 <= abi.NOALLOC_SCRATCH_BYTES
    # float32 decode step: conv output, x_proj output and dt (the step reads B | C
    # from the x_proj output)
    f64 = abi.make_dims(64, 999, 64, 128, 16, 4, 8, abi.F32)
    assert abi.sambay_scan_step_workspace(f64) == r256(64 * 128 * 4) + r256(64 * 40 * 4) \
        + r256(64 * 128 * 4)
    # decode step with GMU layers: the scan step's scratch, then H [B, Di]
    assert abi.sambay_decode_step_workspace(abi.make_dims(64, 1, 2560, 5120), 8) == step64 + r256(64 * 5120 * 2)
    assert abi.sambay_decode_step_workspace(abi.make_dims(64, 1, 2560, 5120), 0) == step64
    assert abi.sambay_decode_step_workspace(abi.make_dims(257, 1, 2560, 5120), 1) == 0
    # float32 mode: no partials, no split delta
    f = abi.make_dims(1, 64, 64, 128, 16, 4, 4, abi.F32)
    assert abi.sambay_scan_prefill_workspace(f) == r256(64 * 128 * 4) + r256(64 * 36 * 4) + r256(64 * 128 * 4) \
        + r256(32 * 64 * 4)
    # H, then (more than one 256-row tile) one fp32 256 x 256 partial tile per
    # CTA pair of 148 SMs for a GEMM's K-split tail, and their arrival flags
    assert abi.gmu_forward_workspace(d, 2048) == r256(2048 * 5120 * 2) + r256(74 * 256 * 256 * 4 + 4096)
    assert abi.gmu_forward_workspace(d, 256) == r256(256 * 5120 * 2)
    # H only: the decode GEMMs reduce their K splits in shared memory
    assert abi.gmu_step_workspace(d, 64) == r256(64 * 5120 * 2)
    # invalid or unsupported dims -> 0
    assert abi.sambay_scan_prefill_workspace(abi.make_dims(1, 16, 64, 128, 8, 4, 8, abi.BF16)) == 0
    assert abi.sambay_scan_prefill_workspace(abi.make_dims(0, 16, 64, 128)) == 0
    assert abi.gmu_step_workspace(d, 257) == 0
    assert abi.gmu_forward_workspace(abi.make_dims(1, 1, 100, 128), 4) == 0


class _FakePtr:
    """Stands in for a tensor in calls that must fail validation."""

    def __init__(self, addr):
        self.addr = addr

    def data_ptr(self):
        return self.addr

    def numel(self):
        return 1

    def element_size(self):
        return 1


def _weights(addr=0x10000):
    return abi.ScanWeights(*([addr] * 7))


def test_scan_argument_errors(lib):
    d = abi.make_dims(1, 16, 64, 128, 16, 4, 8, abi.BF16)
    p = _FakePtr(0x10000)
    st = 0
    # NULL input
    with pytest.raises(abi.SambayError) as e:
        abi.sambay_scan_prefill(_weights(), d, None, p, p, p, True, p, st)
    assert e.value.code == 1
    # NULL weight pointer
    w = _weights(); w.A = None
    with pytest.raises(abi.SambayError) as e:
        abi.sambay_scan_prefill(w, d, p, _FakePtr(0x20000), p, p, True, p, st)
    assert e.value.code == 1
    # misaligned pointer
    with pytest.raises(abi.SambayError) as e:
        abi.sambay_scan_prefill(_weights(), d, _FakePtr(0x10008), _FakePtr(0x20000), p, p, True, p, st)
    assert e.value.code == 2
    # M aliasing u
    with pytest.raises(abi.SambayError) as e:
        abi.sambay_scan_prefill(_weights(), d, p, p, p, p, True, p, st)
    assert e.value.code == 1
    # unsupported d_state / d_conv / dt_rank
    for bad in (abi.make_dims(1, 16, 64, 128, 8, 4, 8, abi.BF16),
                abi.make_dims(1, 16, 64, 128, 16, 3, 8, abi.BF16),
                abi.make_dims(1, 16, 64, 128, 16, 4, 12, abi.BF16),
                abi.make_dims(1, 16, 64, 96, 16, 4, 8, abi.BF16)):
        with pytest.raises(abi.SambayError) as e:
            abi.sambay_scan_prefill(_weights(), bad, p, _FakePtr(0x20000), p, p, True, p, st)
        assert e.value.code == 2
    # bad enum / sizes
    with pytest.raises(abi.SambayError) as e:
        abi.sambay_scan_prefill(_weights(), abi.make_dims(1, 0, 64, 128), p, _FakePtr(0x20000), p, p, True, p, st)
    assert e.value.code == 1
    with pytest.raises(abi.SambayError) as e:
        abi.sambay_scan_prefill(_weights(), abi.make_dims(1, 16, 64, 128, io=7), p, _FakePtr(0x20000), p, p, True, p, st)
    assert e.value.code == 1
    # workspace too small (1 byte)
    with pytest.raises(abi.SambayError) as e:
        abi.sambay_scan_prefill(_weights(), d, p, _FakePtr(0x20000), p, p, True, p, st)
    assert e.value.code == 3
    d32 = abi.make_dims(1, 16, 64, 128, 16, 4, 8, abi.F32)
    with pytest.raises(abi.SambayError) as e:
        abi.sambay_scan_step(_weights(), d32, p, _FakePtr(0x20000), p, p, p, st)
    assert e.value.code == 3
    with pytest.raises(abi.SambayError) as e:
        abi.sambay_scan_step(_weights(), d, p, p, p, p, p, st)
    assert e.value.code == 1


def test_gmu_argument_errors(lib):
    d = abi.make_dims(1, 1, 64, 128, io=abi.BF16)
    X, M, W1, W2, Y = (_FakePtr(a) for a in (0x10000, 0x20000, 0x30000, 0x40000, 0x50000))
    tiny_ws = _FakePtr(0x60000)
    st = 0
    for fn in (abi.gmu_forward, abi.gmu_step):
        with pytest.raises(abi.SambayError) as e:
            fn(d, 4, X, M, W1, W2, None, Y, tiny_ws, st)
        assert e.value.code == 3
        with pytest.raises(abi.SambayError) as e:
            fn(d, 4, None, M, W1, W2, None, Y, tiny_ws, st)
        assert e.value.code == 1
        with pytest.raises(abi.SambayError) as e:
            fn(d, 0, X, M, W1, W2, None, Y, tiny_ws, st)
        assert e.value.code == 1
        with pytest.raises(abi.SambayError) as e:   # Y aliases M
            fn(d, 4, X, M, W1, W2, None, M, tiny_ws, st)
        assert e.value.code == 1
        with pytest.raises(abi.SambayError) as e:   # d_model not a multiple of 64 in bf16
            fn(abi.make_dims(1, 1, 96, 128, io=abi.BF16), 4, X, M, W1, W2, None, Y, tiny_ws, st)
        assert e.value.code == 2
    with pytest.raises(abi.SambayError) as e:
        abi.gmu_step(d, 300, X, M, W1, W2, None, Y, tiny_ws, st)
    assert e.value.code in (2, 3)


def test_device_status_null_out(lib):
    assert lib.sambay_device_status(None, None) == 1


def test_product_path_has_no_oracle_or_fallback():
    """The package never imports the oracle, and fails loudly without the library."""
    pkg = os.path.join(ROOT, "gated_memory_sharing_b200")
    for fn in os.listdir(pkg):
        if fn.endswith(".py"):
            src = open(os.path.join(pkg, fn)).read()
            assert not re.search(r"^\s*(import|from)\s+oracle", src, re.M), fn
    with pytest.raises(RuntimeError):
        abi._lib_backup = abi._lib
        try:
            abi._lib = None
            abi.load("/nonexistent/libsambay.so")
        finally:
            abi._lib = abi._lib_backup


def test_ssd_argument_errors(lib):
    ok = abi.SsdDims(1, 2048, 80, 64, 128, 4, abi.BF16)
    # the conv output as a bf16 split pair: L x (H P + 2 N) x 4 bytes
    assert abi.sambay_ssd_prefill_workspace(ok) == 2048 * (80 * 64 + 256) * 4
    p = _FakePtr(0x10000)
    w = abi.SsdWeights(0x10000, 0x10000, 0x10000, 0x10000, 0x10000)
    for bad, code in ((abi.SsdDims(1, 64, 2, 64, 128, 4, abi.F32), 2),      # float32 I/O
                      (abi.SsdDims(1, 64, 2, 128, 128, 4, abi.BF16), 2),    # head dim
                      (abi.SsdDims(1, 64, 2, 64, 96, 4, abi.BF16), 2),      # d_state
                      (abi.SsdDims(1, 64, 2, 64, 64, 3, abi.BF16), 2),      # conv width
                      (abi.SsdDims(0, 64, 2, 64, 64, 4, abi.BF16), 1)):
        assert abi.sambay_ssd_prefill_workspace(bad) == 0
        with pytest.raises(abi.SambayError) as e:
            abi.sambay_ssd_prefill(w, bad, p, _FakePtr(0x20000), _FakePtr(0x30000), _FakePtr(0x40000),
                                   _FakePtr(0x50000), True, p, 0)
        assert e.value.code == code
    with pytest.raises(abi.SambayError) as e:     # M aliases xbc
        abi.sambay_ssd_prefill(w, ok, p, _FakePtr(0x20000), p, _FakePtr(0x40000), _FakePtr(0x50000), True, p, 0)
    assert e.value.code == 1
    with pytest.raises(abi.SambayError) as e:     # workspace too small
        abi.sambay_ssd_prefill(w, ok, p, _FakePtr(0x20000), _FakePtr(0x30000), _FakePtr(0x40000),
                               _FakePtr(0x50000), True, p, 0)
    assert e.value.code == 3


def test_sharded_prefill_argument_errors(lib):
    """The channel-sharded prefill's calls reject bad arguments on the host,
    before any launch (status codes 1 invalid, 2 unsupported, 3 workspace)."""
    ok = abi.make_dims(1, 64, 128, 256, 16, 4, 16, abi.BF16)
    w = abi.ScanWeights(*([0x10000] * 7))
    u, cs, M, h = _FakePtr(0x20000), _FakePtr(0x30000), _FakePtr(0x40000), _FakePtr(0x50000)
    big_ws = _FakePtr(0x60000)
    big_ws.numel = lambda: abi.sambay_scan_prefill_workspace(ok)
    cases = [
        (lambda: abi.sambay_scan_prefill_xproj(w, ok, u, cs, True, None, big_ws, 0), 1),              # no xdbl
        (lambda: abi.sambay_scan_prefill_xproj(w, ok, u, cs, True, _FakePtr(0x70004), big_ws, 0), 2),  # misaligned
        (lambda: abi.sambay_scan_prefill_xproj(w, ok, u, cs, True, _FakePtr(0x70000), _FakePtr(0x60000), 0), 3),
        (lambda: abi.sambay_scan_prefill_xproj(w, abi.make_dims(1, 64, 128, 256, 32, 4, 16, abi.BF16), u, cs,
                                               True, _FakePtr(0x70000), big_ws, 0), 2),                # d_state
        (lambda: abi.sambay_scan_prefill_finish(w, ok, u, _FakePtr(0x70000), u, h, cs, True, big_ws, 0), 1),  # M is u
        (lambda: abi.sambay_scan_prefill_finish(w, ok, u, None, M, h, cs, True, big_ws, 0), 1),        # no xdbl
    ]
    g = abi.make_dims(64, 1, 128, 256, 16, 4, 4, abi.BF16)
    X, Mg, W1, W2, Yp = (_FakePtr(a) for a in (0x20000, 0x30000, 0x40000, 0x50000, 0x60000))
    cases += [
        (lambda: abi.gmu_forward_partial(g, 0, X, Mg, W1, W2, Yp, big_ws, 0), 1),                      # no rows
        (lambda: abi.gmu_forward_partial(g, 64, X, Mg, W1, W2, X, big_ws, 0), 1),                      # Y_part is X
        (lambda: abi.gmu_finish(g, 0, Yp, None, X, 0), 1),                                             # no rows
        (lambda: abi.gmu_finish(g, 64, Yp, None, Yp, 0), 1),                                           # Y is Y_sum
        (lambda: abi.gmu_finish(g, 64, Yp, _FakePtr(0x70002), X, 0), 2),                               # residual
    ]
    for call, code in cases:
        with pytest.raises(abi.SambayError) as e:
            call()
        assert e.value.code == code

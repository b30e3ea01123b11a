"""The decode step for callers that cannot allocate device memory.

Some callers of this library cannot hand it a workspace: a serving engine's
per-token decode loop whose device memory is planned once up front and may
not allocate afterwards, or a plugin host that passes only input and output
pointers.  For them sambay_scan_step_noalloc runs the decode step with a
scratch array that lives inside the library.  It must produce what the
workspace entry point sambay_scan_step produces, call after call, since
every call reuses (and leaves behind) the same scratch contents.

This file is collected last on purpose, and it builds and loads the library
itself, so it passes both on its own in a fresh process and after the rest
of the suite.
"""

import numpy as np
import pytest
import torch

from gated_memory_sharing_b200 import abi, synth
from gated_memory_sharing_b200.layers import ScanLayer, to_device
from tests.gpu_util import host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from gated_memory_sharing_b200 import build
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    abi.load()
    torch.cuda.set_device(0)
    yield
    assert abi.sambay_device_status() == 0


CASES = {
    # the decode workload's width: 64 sequences, d_inner 5120, dt_rank 160
    # (7.7 MB of the 8 MiB array: conv output, x_proj partials, delta, B | C)
    "bf16": synth.Dims(64, 8, 2560, 5120, 16, 4, 160, synth.BF16),
    # float32 I/O: the step's kernels exchange the conv output, x_proj output,
    # dt and B | C through the scratch array
    "f32": synth.Dims(3, 8, 64, 128, 16, 4, 8, synth.F32),
    "f32_wide": synth.Dims(16, 8, 512, 1024, 16, 4, 32, synth.F32),
}


@pytest.mark.parametrize("name", ["bf16", "f32", "f32_wide"])
def test_noalloc_step_matches_workspace_step_twice(name):
    d = CASES[name]
    io = abi.BF16 if d.io == synth.BF16 else abi.F32
    seed = 4242
    w = synth.scan_weights(d, seed)
    u = synth.scan_inputs(d, seed, seqlen=d.seqlen + 2)
    layer = ScanLayer(w, d.d_model, io)
    _, h, cs = layer.prefill(to_device(u[:, :d.seqlen], io))
    h_ws, cs_ws = h.clone(), cs.clone()      # state advanced by sambay_scan_step
    h_na, cs_na = h.clone(), cs.clone()      # state advanced by the no-alloc variant
    dims = layer.dims(d.batch, 1)
    assert abi.sambay_scan_step_workspace(dims) <= abi.NOALLOC_SCRATCH_BYTES
    free_before = None
    for call in range(2):
        u_t = to_device(np.ascontiguousarray(u[:, d.seqlen + call]), io)
        m_ws = layer.step(u_t, h_ws, cs_ws)
        m_na = torch.empty_like(u_t)
        torch.cuda.synchronize()
        if call == 1:
            free_before = torch.cuda.mem_get_info()[0]
        abi.sambay_scan_step_noalloc(layer.abi_w, dims, u_t, m_na, h_na, cs_na)
        torch.cuda.synchronize()
        if call == 1:
            # the entry point itself takes no device memory (the first call
            # has looked up the scratch array's address already)
            assert torch.cuda.mem_get_info()[0] == free_before
        # the same kernels on the same inputs: the same bits, call after call,
        # whatever the previous call left in the scratch array
        np.testing.assert_array_equal(host(m_na), host(m_ws), err_msg=f"{name} call {call}: m_t")
        np.testing.assert_array_equal(host(h_na), host(h_ws), err_msg=f"{name} call {call}: ssm_state")
        np.testing.assert_array_equal(host(cs_na), host(cs_ws))


def test_noalloc_step_rejects_sizes_beyond_its_scratch():
    # float32 I/O, 256 sequences at d_inner 5120: 21 MB of step scratch
    d = synth.Dims(256, 1, 2560, 5120, 16, 4, 160, synth.F32)
    dims = abi.make_dims(d.batch, 1, d.d_model, d.d_inner, 16, 4, 160, abi.F32)
    assert abi.sambay_scan_step_workspace(dims) > abi.NOALLOC_SCRATCH_BYTES
    layer = ScanLayer(synth.scan_weights(d, 1), d.d_model, abi.F32)
    h, cs = layer.new_state(d.batch)
    u_t = torch.zeros(d.batch, d.d_inner, dtype=torch.float32, device="cuda")
    m_t = torch.empty_like(u_t)
    with pytest.raises(abi.SambayError) as e:
        abi.sambay_scan_step_noalloc(layer.abi_w, dims, u_t, m_t, h, cs)
    assert e.value.code == 2      # SAMBAY_ERR_UNSUPPORTED, before any launch

"""The multi-rank path of bench.py on the host: world size 2 over gloo.

`bench.py --gpus N` runs one process per GPU under torchrun; sequences are
independent, so each rank benchmarks its own sequence with no collective on
the data path, and the only cross-rank operations are the barriers around the
timed regions and the maximum of the ranks' times.  These tests run that
plumbing as two CPU processes (gloo, 127.0.0.1), with no GPU.
"""

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch
    import bench
    from gated_memory_sharing_b200 import synth
    w, r, loc = bench.dist_env()
    dist = bench.init_dist(w, "gloo")
    try:
        # the job's time is the slowest rank's
        t = bench.max_over_ranks(10.0 + rank, w, torch.device("cpu"))
        bench.barrier(w)
        # each rank draws its own sequence from the rank-shifted seed, the same weights
        d, seed = synth.workload("tiny_f32")
        u = synth.scan_inputs(d, seed + 7919 * r)
        wts = synth.scan_weights(d, seed)
        out[rank] = (w, r, loc, t, float(u.sum()), float(wts["A"].sum()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_barrier_and_sharding():
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(2, _free_port(), out), nprocs=2, start_method="spawn", join=True)
    r0, r1 = out[0], out[1]
    assert (r0[0], r0[1], r0[2]) == (2, 0, 0) and (r1[0], r1[1], r1[2]) == (2, 1, 1)
    assert r0[3] == r1[3] == 11.0                 # max over ranks, seen by both
    assert r0[4] != r1[4]                         # distinct sequences per rank
    assert r0[5] == r1[5]                         # identical weights


def _ref_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import contextlib
    import io
    import bench

    class A:
        steps, warmup, gpus, workload = 1, 0, world, bench.HEADLINE
    buf = io.StringIO()
    orig = bench.synth.workload
    bench.synth.workload = lambda name: orig("tiny_f32")      # a small stand-in
    try:
        with contextlib.redirect_stdout(buf):
            bench.run_reference(A, world, rank)
    finally:
        bench.synth.workload = orig
    out[rank] = buf.getvalue()


def test_reference_arm_prints_on_rank_zero_only():
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_ref_worker, args=(2, _free_port(), out), nprocs=2, start_method="spawn", join=True)
    import json
    line = json.loads(out[0].strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["e2e"]["value"] == line["value"]
    assert out[1] == ""

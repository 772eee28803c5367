"""Blocks that run at the same time: two plans on two streams, and one plan
driven from two host threads on two streams.

Each call enqueues its chunk-overlap events and launches under its plan's
lock, so concurrent calls never wait on each other's events; their results
must equal those of the same calls run one after another (bit for bit: the
kernels are deterministic) and the float64 oracle (within the bf16
tolerances)."""

import threading

import numpy as np
import pytest
import torch

from oracle import attention as oa
from oracle import layout as ol
from tests.gpu_util import assert_close, device_bits, to_device
from ulysses_sequence_attention_sp_b200.synth import make_qkv, storage_to_f64
from ulysses_sequence_attention_sp_b200.workloads import Workload

pytestmark = pytest.mark.gpu

A = Workload("conc-a-bf16-T2000-H6-D128-P3", 1, 2000, 0, 6, 128, 3, "bf16", 1.0, 9301, (3,))
B = Workload("conc-b-bf16-B2-T900-cls-H8-D64-P4", 2, 900, 1, 8, 64, 4, "bf16", 1.0, 9302, (2,))


@pytest.fixture(scope="module")
def usp():
    from ulysses_sequence_attention_sp_b200 import usp as mod
    assert torch.cuda.is_available()
    mod.device_status(reset=True)
    return mod


def _plan(usp, w):
    return usp.Plan(w.batch, w.seq_len, w.heads, w.head_dim, w.world, w.dtype, w.prefix)


def _inputs(usp, plan, w, seed):
    storage = make_qkv(w, seed)
    return storage, [usp.scatter_sequence(plan, to_device(x, w.dtype)) for x in storage]


def _oracle(plan, w, storage):
    f64 = [storage_to_f64(x, w.dtype) for x in storage]
    shards = [ol.scatter_sequence(x, plan.token_ranges, prefix=w.prefix) for x in f64]
    return oa.ulysses_attention(*shards, plan.token_ranges, plan.head_ranges, prefix=w.prefix)


def _bits(shards):
    return [device_bits(t) for t in shards]


def test_two_plans_on_two_streams(usp):
    plans = [_plan(usp, A), _plan(usp, B)]
    ins = [_inputs(usp, p, w, w.seed) for p, w in zip(plans, (A, B))]
    # serial results first
    serial = []
    for p, w, (_, sh) in zip(plans, (A, B), ins):
        serial.append(_bits(usp.ulysses_attention(p, *sh, num_chunks=w.num_chunks[0])))
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = [p.empty_seq_shards(fill=float("nan")) for p in plans]
    wss = [torch.empty(p.workspace_bytes(w.num_chunks[0]), dtype=torch.uint8, device="cuda")
           for p, w in zip(plans, (A, B))]
    for s in streams:
        s.wait_stream(torch.cuda.current_stream())
    for _ in range(3):  # several rounds, so the two blocks overlap on the GPU
        for p, w, (_, sh), o, ws, s in zip(plans, (A, B), ins, outs, wss, streams):
            with torch.cuda.stream(s):
                usp.ulysses_attention(p, *sh, out=o, num_chunks=w.num_chunks[0], workspace=ws)
    torch.cuda.synchronize()
    assert usp.device_status() == 0
    for p, w, (storage, _), o, ser in zip(plans, (A, B), ins, outs, serial):
        got = _bits(o)
        for r in range(p.world):
            np.testing.assert_array_equal(got[r], ser[r], err_msg=f"{w.name} rank {r}")
        ref = _oracle(p, w, storage)
        for r in range(p.world):
            assert_close(storage_to_f64(got[r], w.dtype), ref[r], w.dtype, f"{w.name} rank {r}")
    for p in plans:
        p.close()


def test_one_plan_from_two_threads(usp):
    plan = _plan(usp, A)
    n_chunks = A.num_chunks[0]
    jobs = [_inputs(usp, plan, A, A.seed + i) for i in range(2)]
    serial = [_bits(usp.ulysses_attention(plan, *sh, num_chunks=n_chunks)) for _, sh in jobs]
    torch.cuda.synchronize()
    outs = [plan.empty_seq_shards(fill=float("nan")) for _ in jobs]
    wss = [torch.empty(plan.workspace_bytes(n_chunks), dtype=torch.uint8, device="cuda") for _ in jobs]
    streams = [torch.cuda.Stream() for _ in jobs]
    for s in streams:
        s.wait_stream(torch.cuda.current_stream())
    errors = []
    start = threading.Barrier(len(jobs))

    def worker(i):
        try:
            torch.cuda.set_device(0)
            start.wait()
            with torch.cuda.stream(streams[i]):
                for _ in range(8):
                    usp.ulysses_attention(plan, *jobs[i][1], out=outs[i], num_chunks=n_chunks, workspace=wss[i])
        except Exception as e:  # reported below, in the main thread
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(len(jobs))]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not errors, errors
    torch.cuda.synchronize()
    assert usp.device_status() == 0
    for i, ((storage, _), o) in enumerate(zip(jobs, outs)):
        got = _bits(o)
        for r in range(plan.world):
            np.testing.assert_array_equal(got[r], serial[i][r], err_msg=f"thread {i} rank {r}")
        ref = _oracle(plan, A, storage)
        for r in range(plan.world):
            assert_close(storage_to_f64(got[r], "bf16"), ref[r], "bf16", f"thread {i} rank {r}")
    plan.close()

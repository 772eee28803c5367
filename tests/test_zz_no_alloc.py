"""The allocation-free entry point, usp_ulysses_attention_noalloc.

It exists for callers that cannot allocate device memory when they call the
block (a plugin whose host framework owns all device memory, or a path that
must not synchronise the device the way cudaFree does): its scratch is a fixed
array inside the library. This test calls it through the C ABI twice in a row,
on different inputs, and checks each result against the regular entry point
(caller-owned workspace) within the tolerance the other attention tests use.
It also checks that a plan needing more scratch than the array is refused.

The file is named so that pytest collects it last; it also passes on its own
in a fresh process (it builds every input itself).
"""

import ctypes

import numpy as np
import pytest
import torch

from tests.gpu_util import assert_close, to_device, to_f64
from ulysses_sequence_attention_sp_b200.synth import make_qkv
from ulysses_sequence_attention_sp_b200.workloads import Workload

pytestmark = pytest.mark.gpu

CASES = [
    Workload("noalloc-bf16-T1000-cls-H6-D128-P4", 1, 1000, 1, 6, 128, 4, "bf16", 1.0, 9101, (1, 2)),
    Workload("noalloc-bf16-B3-T300-H5-D80-P3", 3, 300, 0, 5, 80, 3, "bf16", 0.5, 9102, (1, 3)),
    # grouped-query attention: 8 query heads over 4 kv heads (separate kv head ranges in the scratch)
    Workload("noalloc-gqa-bf16-T700-H8-KV4-D64-P4", 1, 700, 0, 8, 64, 4, "bf16", 1.0, 9103, (1, 2), kv_heads=4),
    # Ulysses 2 x Ring 2 hybrid with a cls row (ring key blocks in the scratch)
    Workload("noalloc-hybrid-bf16-T900-cls-H4-D128-U2xR2", 1, 900, 1, 4, 128, 4, "bf16", 1.0, 9104, (1, 2),
             ring=2),
]


@pytest.fixture(scope="module")
def usp():
    from ulysses_sequence_attention_sp_b200 import usp as mod
    assert torch.cuda.is_available()
    return mod


def _noalloc_call(usp, plan, q, k, v, out, num_chunks):
    """Calls the C entry point directly with ctypes (plain pointers, current stream)."""
    lib = ctypes.CDLL(usp.library_path())
    fn = lib.usp_ulysses_attention_noalloc
    fn.restype = ctypes.c_int
    ptrs = lambda ts: (ctypes.c_void_p * len(ts))(*[t.data_ptr() for t in ts])
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = fn(plan.handle, ptrs(q), ptrs(k), ptrs(v), ptrs(out), ctypes.c_float(0.0), ctypes.c_int32(num_chunks), stream)
    return rc


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_noalloc_matches_regular_entry_point_twice(usp, w):
    plan = usp.Plan(w.batch, w.seq_len, w.heads, w.head_dim, w.world, w.dtype, w.prefix, kv_heads=w.heads_kv,
                    ring_size=w.ring)
    for call, seed in enumerate((w.seed, w.seed + 1)):
        num_chunks = w.num_chunks[call % len(w.num_chunks)]
        shards = [usp.scatter_sequence(plan, to_device(x, w.dtype)) for x in make_qkv(w, seed)]
        ref = usp.ulysses_attention(plan, *shards, num_chunks=num_chunks)
        got = plan.empty_seq_shards(fill=float("nan"))
        torch.cuda.synchronize()
        # the call itself reserves no device memory: neither torch's allocator
        # nor the device's free memory moves across it
        allocated, free = torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0]
        assert _noalloc_call(usp, plan, *shards, got, num_chunks) == usp.USP_OK, usp._lib.usp_last_error_message()
        torch.cuda.synchronize()
        if call == 1:  # the first call may still load kernels' code on first use
            assert torch.cuda.memory_allocated() == allocated
            assert torch.cuda.mem_get_info()[0] == free
        assert usp.device_status() == 0
        for r in range(plan.world):
            assert_close(to_f64(got[r], w.dtype), to_f64(ref[r], w.dtype), w.dtype, f"call {call} rank {r}")
    plan.close()


def test_noalloc_rejects_plans_above_its_scratch(usp):
    # 3 x B*T'*H*D*2 bytes of head shards: 3 x 2 x 16384 x 8 x 128 x 2 = 192 MiB > 64 MiB
    plan = usp.Plan(2, 16384, 8, 128, 4, "bf16", 0)
    assert plan.workspace_bytes(1) > usp.NOALLOC_SCRATCH_BYTES
    shards = plan.empty_seq_shards(fill=0.0)
    out = plan.empty_seq_shards(fill=0.0)
    launches = usp.kernel_launches()
    assert _noalloc_call(usp, plan, shards, shards, shards, out, 1) == usp.USP_ERR_SHAPE
    assert b"scratch" in usp._lib.usp_last_error_message()
    assert usp.kernel_launches() == launches
    plan.close()

"""The library-owned CUDA graph of the block (usp_ulysses_attention_graph_create
/ usp_graph_launch): a replay gives the same bits as a direct call, also after
new inputs are written into the captured buffers, for the plain block with
chunk overlap and for the Ulysses + Ring hybrid with the TMA pack."""

import pytest
import torch

from tests.gpu_util import to_device
from ulysses_sequence_attention_sp_b200.synth import make_qkv
from ulysses_sequence_attention_sp_b200.workloads import Workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def usp():
    from ulysses_sequence_attention_sp_b200 import usp as mod
    assert torch.cuda.is_available()
    mod.device_status(reset=True)
    return mod


CASES = [  # workload, num_chunks, ring size, pack mode
    (Workload("g-plain", 2, 300, 1, 6, 128, 4, "bf16", 1.0, 91, (1,)), 1, 1, "vector"),
    (Workload("g-chunks", 1, 517, 0, 9, 64, 3, "bf16", 1.0, 92, (1,)), 3, 1, "vector"),
    (Workload("g-hybrid", 1, 600, 0, 8, 128, 8, "bf16", 1.0, 93, (1,), 4), 2, 2, "tma"),
    (Workload("g-fp32", 1, 37, 0, 6, 16, 4, "fp32", 1.0, 94, (1,)), 2, 1, "vector"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0].name)
def test_graph_replay_matches_direct_call(usp, case):
    w, n, ring, mode = case
    plan = usp.Plan(w.batch, w.seq_len, w.heads, w.head_dim, w.world, w.dtype, w.prefix, kv_heads=w.heads_kv,
                    ring_size=ring)
    plan.set_pack_mode(mode)
    shapes = [plan.seq_shard_shape(r) for r in range(plan.world)]
    kv_shapes = [plan.kv_seq_shard_shape(r) for r in range(plan.world)]
    ins = [[torch.empty(s, dtype=plan.torch_dtype, device="cuda") for s in sh] for sh in (shapes, kv_shapes, kv_shapes)]

    def load(seed):
        for x, dst in zip(make_qkv(w, seed), ins):
            usp.scatter_sequence(plan, to_device(x, w.dtype), out=dst)

    load(1)
    g = usp.AttentionGraph(plan, *ins, num_chunks=n)
    bits = torch.int16 if w.dtype == "bf16" else torch.int32
    for seed in (1, 2, 3):
        load(seed)
        for o in g.out:
            o.fill_(float("nan"))
        g.launch()
        ref = usp.ulysses_attention(plan, *ins, num_chunks=n)
        torch.cuda.synchronize()
        for a, b in zip(g.out, ref):
            assert torch.equal(a.view(bits), b.view(bits)), f"seed {seed}"
    assert usp.device_status() == 0
    g.close()
    plan.close()


def test_graph_create_rejects_bad_arguments_and_leaves_no_capture(usp):
    plan = usp.Plan(1, 64, 4, 32, 2, "bf16")
    q = plan.empty_seq_shards(fill=0.0)
    with pytest.raises(usp.UspError):
        usp.AttentionGraph(plan, q, q, q, num_chunks=0)
    out = usp.ulysses_attention(plan, q, q, q)  # the stream is not left capturing
    torch.cuda.synchronize()
    assert all(not torch.isnan(o).any() for o in out)
    plan.close()

"""The TMA-staged sequence -> head pack against the 16-byte vector pack.

Both move the same bytes, so the Ulysses block (whose q/k/v pack into the
head-major workspace is the hot use of the TMA pack) must give bit-identical
outputs with either; the public exchange is compared with the oracle bit for
bit in test_gpu_layout.py under both modes."""

import pytest
import torch

from tests.gpu_util import to_device
from ulysses_sequence_attention_sp_b200.synth import make_qkv
from ulysses_sequence_attention_sp_b200.workloads import CHUNKED, VIDEO, VIT, Workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def usp():
    from ulysses_sequence_attention_sp_b200 import usp as mod
    assert torch.cuda.is_available()
    mod.device_status(reset=True)
    return mod


CASES = [  # workload, num_chunks, ring size
    (Workload("t1", 1, 300, 0, 6, 128, 4, "bf16", 1.0, 61, (1,)), 1, 1),
    (Workload("t2", 2, 200, 1, 5, 80, 3, "bf16", 1.0, 62, (1,)), 2, 1),
    (Workload("t3", 1, 517, 0, 8, 64, 2, "bf16", 1.0, 63, (1,), 2), 3, 1),    # GQA: q and k/v packs
    (Workload("t4", 1, 37, 0, 6, 16, 4, "fp32", 1.0, 64, (1,)), 2, 1),        # 64-byte fp32 units
    (Workload("t5", 3, 9, 1, 4, 48, 4, "bf16", 1.0, 65, (1,)), 1, 1),         # ranks of 2 and 3 rows
    (Workload("t6", 1, 600, 0, 4, 128, 4, "bf16", 1.0, 66, (1,)), 2, 2),      # Ulysses 2 x Ring 2
    (VIT, 1, 1),
    (CHUNKED, 3, 1),
    (VIDEO, 1, 1),
]


def _run(usp, w, ring, num_chunks, mode, storage):
    plan = usp.Plan(w.batch, w.seq_len, w.heads, w.head_dim, w.world, w.dtype, w.prefix, kv_heads=w.heads_kv,
                    ring_size=ring)
    plan.set_pack_mode(mode)
    shards = [usp.scatter_sequence(plan, to_device(x, w.dtype)) for x in storage]
    out = plan.empty_seq_shards(fill=float("nan"))
    usp.ulysses_attention(plan, *shards, out=out, num_chunks=num_chunks)
    torch.cuda.synchronize()
    assert usp.device_status() == 0
    assert not any(torch.isnan(o).any().item() for o in out)  # every row was written
    bits = [o.view(torch.int16 if o.element_size() == 2 else torch.int32).cpu() for o in out]
    plan.close()
    return bits


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0].name}-chunks{c[1]}-ring{c[2]}")
def test_block_identical_with_either_pack(usp, case):
    w, num_chunks, ring = case
    storage = make_qkv(w)
    vec = _run(usp, w, ring, num_chunks, "vector", storage)
    tma = _run(usp, w, ring, num_chunks, "tma", storage)
    for r, (a, b) in enumerate(zip(vec, tma)):
        assert torch.equal(a, b), f"rank {r}"


def test_pack_mode_argument(usp):
    plan = usp.Plan(1, 16, 4, 16, 2, "bf16")
    with pytest.raises(usp.UspError):
        plan.set_pack_mode("bulk")
    plan.set_pack_mode("tma")
    plan.set_pack_mode("vector")
    plan.close()

"""GPU parity of the rank-local (multi-process) entry points on one device.

Each of the P ranks' calls runs on this one GPU against its own buffers; the
collective between them is emulated by copying the blocks the split lists
name (rank r's send block for peer j lands at peer j's receive offset for
source r). So the pack and unpack kernels, the attention writing its output
into the send blocks of the way back, and the split lists are checked exactly
as a multi-process run would use them:
- layouts bit for bit against the oracle's seq_to_head / head_to_seq;
- the attention bit for bit against the one-device block (the same kernel on
  the same head-major workspace layout), and within the bf16 tolerances
  against the float64 oracle;
- the all-gather form equal to the all-to-all form.
No kernel waits on another rank's kernel (the ranks' calls run one after
another on one stream)."""

import numpy as np
import pytest
import torch
import torch.distributed as dist

from oracle import attention as oa
from oracle import layout as ol
from tests.gpu_util import assert_close, bits_to_device, device_bits, to_device
from ulysses_sequence_attention_sp_b200.synth import make_bits, make_qkv, storage_to_f64
from ulysses_sequence_attention_sp_b200.workloads import Workload

pytestmark = pytest.mark.gpu

CASES = [
    Workload("dist-bf16-T1000-H6-D128-P3", 1, 1000, 0, 6, 128, 3, "bf16", 1.0, 9401, (1, 2, 3)),
    Workload("dist-bf16-B2-T600-cls-H8-KV4-D64-P4", 2, 600, 1, 8, 64, 4, "bf16", 1.0, 9402, (1, 2), kv_heads=4),
    Workload("dist-bf16-T777-cls-H7-D80-P3", 1, 777, 1, 7, 80, 3, "bf16", 0.5, 9403, (1, 2)),
    Workload("dist-fp32-T37-H6-D16-P4", 1, 37, 0, 6, 16, 4, "fp32", 1.0, 9404, (1, 2)),
]


@pytest.fixture(scope="module")
def usp():
    from ulysses_sequence_attention_sp_b200 import usp as mod
    assert torch.cuda.is_available()
    mod.device_status(reset=True)
    return mod


def _plan(usp, w):
    return usp.Plan(w.batch, w.seq_len, w.heads, w.head_dim, w.world, w.dtype, w.prefix, kv_heads=w.heads_kv)


def _exchange(usp, plan, kind, nt, n, c, sends):
    """Emulated collective: per rank (send counts, displs, recv counts, displs)
    from the library, and every block copied to its receiver."""
    cnts = [usp.dist_counts(plan, r, kind, nt, n, c) for r in range(plan.world)]
    gather = kind in (usp.DIST_GATHER_SEQ, usp.DIST_GATHER_HEADS)
    recvs = [torch.full((max(sum(cnt[2]), 1),), float("nan"), dtype=plan.torch_dtype, device="cuda") for cnt in cnts]
    for src in range(plan.world):
        sc, sd = cnts[src][0], cnts[src][1]
        for dst in range(plan.world):
            rc, rd = cnts[dst][2], cnts[dst][3]
            assert sc[dst] == rc[src], (src, dst, sc[dst], rc[src])
            if sc[dst]:
                recvs[dst][rd[src]:rd[src] + rc[src]].copy_(sends[src][sd[dst]:sd[dst] + sc[dst]])
    return recvs, cnts


def _send(plan, cnt, gather):
    n = cnt[0][0] if gather else sum(cnt[0])
    return torch.full((max(n, 1),), float("nan"), dtype=plan.torch_dtype, device="cuda")


def _bits(t):
    return device_bits(t)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
@pytest.mark.parametrize("gather", [False, True], ids=["all_to_all", "all_gather"])
def test_layout_exchanges_bit_exact(usp, w, gather):
    """seq->head of q, k, v and head->seq, every chunk count, against the oracle."""
    plan = _plan(usp, w)
    elem = 2 if w.dtype == "bf16" else 4
    full = [make_bits((w.batch, w.tokens, h, w.head_dim), elem, 700 + i) for i, h in
            enumerate((w.heads, w.heads_kv, w.heads_kv))]
    tr, hr, kr = plan.token_ranges, plan.head_ranges, plan.kv_head_ranges
    seq = [ol.scatter_sequence(x, tr, prefix=w.prefix) for x in full]
    ref = [ol.seq_to_head(seq[0], tr, hr, prefix=w.prefix), ol.seq_to_head(seq[1], tr, kr, prefix=w.prefix),
           ol.seq_to_head(seq[2], tr, kr, prefix=w.prefix)]
    dev_seq = [[bits_to_device(s).view(plan.torch_dtype) for s in seq[t]] for t in range(3)]
    kind_in = usp.DIST_GATHER_SEQ if gather else usp.DIST_SEQ_TO_HEAD
    kind_out = usp.DIST_GATHER_HEADS if gather else usp.DIST_HEAD_TO_SEQ
    for n in w.num_chunks:
        nchunks = len(usp.head_chunk_ranges(hr[0][1] - hr[0][0], n))
        heads = [[torch.full(sh, float("nan"), dtype=plan.torch_dtype, device="cuda")
                  for sh in (plan.head_shard_shape(r), plan.kv_head_shard_shape(r), plan.kv_head_shard_shape(r))]
                 for r in range(plan.world)]
        for c in range(nchunks):
            cnt0 = usp.dist_counts(plan, 0, kind_in, 3, n, c)
            sends = []
            for r in range(plan.world):
                s = _send(plan, usp.dist_counts(plan, r, kind_in, 3, n, c), gather)
                usp.dist_pack(plan, r, kind_in, [dev_seq[t][r] for t in range(3)], s, n, c)
                sends.append(s)
            recvs, _ = _exchange(usp, plan, kind_in, 3, n, c, sends)
            for r in range(plan.world):
                usp.dist_unpack(plan, r, kind_in, recvs[r], heads[r], n, c)
            del cnt0
        torch.cuda.synchronize()
        for r in range(plan.world):
            for t in range(3):
                np.testing.assert_array_equal(_bits(heads[r][t]), ref[t][r], err_msg=f"n={n} rank {r} tensor {t}")
        # the q head shards back to q sequence shards
        back = [torch.full(plan.seq_shard_shape(r), float("nan"), dtype=plan.torch_dtype, device="cuda")
                for r in range(plan.world)]
        for c in range(nchunks):
            sends = []
            for r in range(plan.world):
                s = _send(plan, usp.dist_counts(plan, r, kind_out, 1, n, c), gather)
                usp.dist_pack(plan, r, kind_out, [heads[r][0]], s, n, c)
                sends.append(s)
            recvs, _ = _exchange(usp, plan, kind_out, 1, n, c, sends)
            for r in range(plan.world):
                usp.dist_unpack(plan, r, kind_out, recvs[r], [back[r]], n, c)
        torch.cuda.synchronize()
        for r in range(plan.world):
            np.testing.assert_array_equal(_bits(back[r]), seq[0][r], err_msg=f"n={n} head_to_seq rank {r}")
    assert usp.device_status() == 0
    plan.close()


def _dist_block(usp, plan, shards, n, gather):
    """The whole block the way a multi-process run does it, rank by rank."""
    kind_in = usp.DIST_GATHER_SEQ if gather else usp.DIST_SEQ_TO_HEAD
    kind_out = usp.DIST_GATHER_HEADS if gather else usp.DIST_HEAD_TO_SEQ
    P = plan.world
    hr = plan.head_ranges
    nchunks = len(usp.head_chunk_ranges(hr[0][1] - hr[0][0], n))
    out = [torch.full(plan.seq_shard_shape(r), float("nan"), dtype=plan.torch_dtype, device="cuda") for r in range(P)]
    wss = [torch.empty(usp.dist_workspace_bytes(plan, r), dtype=torch.uint8, device="cuda") for r in range(P)]
    recv_in = None
    for c in range(nchunks):
        if not gather or c == 0:
            sends = []
            for r in range(P):
                s = _send(plan, usp.dist_counts(plan, r, kind_in, 3, n, c), gather)
                usp.dist_pack(plan, r, kind_in, [shards[t][r] for t in range(3)], s, n, c)
                sends.append(s)
            recv_in, _ = _exchange(usp, plan, kind_in, 3, n, c, sends)
        send_o = []
        for r in range(P):
            s = _send(plan, usp.dist_counts(plan, r, kind_out, 1, n, c), gather)
            usp.dist_attention(plan, r, kind_in, recv_in[r], s, wss[r], n, c)
            send_o.append(s)
        recv_o, _ = _exchange(usp, plan, kind_out, 1, n, c, send_o)
        for r in range(P):
            usp.dist_unpack(plan, r, kind_out, recv_o[r], [out[r]], n, c)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_attention_equals_one_device_block_and_oracle(usp, w):
    plan = _plan(usp, w)
    storage = make_qkv(w)
    shards = [usp.scatter_sequence(plan, to_device(x, w.dtype)) for x in storage]
    ref_dev = [_bits(o) for o in usp.ulysses_attention(plan, *shards)]
    f64 = [storage_to_f64(x, w.dtype) for x in storage]
    sh64 = [ol.scatter_sequence(x, plan.token_ranges, prefix=w.prefix) for x in f64]
    ref = oa.ulysses_attention(*sh64, plan.token_ranges, plan.head_ranges, kv_head_ranges=plan.kv_head_ranges,
                               prefix=w.prefix)
    for gather in (False, True):
        for n in w.num_chunks:
            out = _dist_block(usp, plan, shards, n, gather)
            assert usp.device_status() == 0
            for r in range(plan.world):
                got = _bits(out[r])
                np.testing.assert_array_equal(got, ref_dev[r], err_msg=f"gather={gather} n={n} rank {r}")
                val = got.view(np.float32) if w.dtype == "fp32" else got
                assert_close(storage_to_f64(val, w.dtype), ref[r], w.dtype, f"gather={gather} n={n} rank {r}")
    plan.close()


def test_rank_local_calls_reject_bad_arguments(usp):
    w = CASES[0]
    plan = _plan(usp, w)
    buf = torch.empty(1 << 20, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(usp.dist_workspace_bytes(plan, 0), dtype=torch.uint8, device="cuda")
    launches = usp.kernel_launches()
    for kw in [dict(rank=3), dict(chunk=5), dict(exchange=7)]:
        args = dict(rank=0, exchange=usp.DIST_SEQ_TO_HEAD, chunk=0) | kw
        with pytest.raises(usp.UspError):
            usp.dist_attention(plan, args["rank"], args["exchange"], buf, buf, ws, 1, args["chunk"])
    with pytest.raises(usp.UspError):
        usp.dist_attention(plan, 0, usp.DIST_HEAD_TO_SEQ, buf, buf, ws)
    with pytest.raises(usp.UspError):  # too small a workspace
        usp.dist_attention(plan, 0, usp.DIST_SEQ_TO_HEAD, buf, buf, ws[:1024])
    hybrid = usp.Plan(1, 1000, 4, 128, 4, "bf16", 0, ring_size=2)
    with pytest.raises(usp.UspError) as e:
        usp.dist_pack(hybrid, 0, usp.DIST_SEQ_TO_HEAD, [buf], buf)
    assert e.value.code == usp.USP_ERR_UNSUPPORTED
    assert usp.kernel_launches() == launches
    hybrid.close()
    plan.close()


def test_process_group_of_one_runs_the_orchestration(usp, tmp_path):
    """The torch.distributed orchestration (all_to_all_single and
    all_gather_into_tensor over NCCL, the chunk pipeline) in a group of one
    rank: its result equals the one-device block bit for bit."""
    from ulysses_sequence_attention_sp_b200.dist import SequenceParallelGroup
    w = Workload("dist-group-of-one-bf16-T900-cls-H4-D128", 1, 900, 1, 4, 128, 1, "bf16", 1.0, 9405, (1, 2))
    if not dist.is_initialized():
        dist.init_process_group("nccl", init_method=f"file://{tmp_path}/pg", rank=0, world_size=1,
                                device_id=torch.device("cuda", 0))
    try:
        g = SequenceParallelGroup(w.batch, w.seq_len, w.heads, w.head_dim, w.dtype, w.prefix)
        storage = make_qkv(w)
        q, k, v = (usp.scatter_sequence(g.plan, to_device(x, w.dtype))[0] for x in storage)
        ref = _bits(usp.ulysses_attention(g.plan, [q], [k], [v])[0])
        for gather in (False, True):
            for n in w.num_chunks:
                got = g.ulysses_attention(q, k, v, num_chunks=n, prefer_all_gather=gather)
                torch.cuda.synchronize()
                np.testing.assert_array_equal(_bits(got), ref, err_msg=f"gather={gather} n={n}")
        heads = g.seq_to_head(q, k, v, num_chunks=2)
        np.testing.assert_array_equal(_bits(g.head_to_seq(heads[0], num_chunks=2)), _bits(q))
        g.close()
    finally:
        dist.destroy_process_group()

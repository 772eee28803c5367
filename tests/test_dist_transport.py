"""The multi-process transport's host logic on CPU ranks (gloo, world 2, 3 and 4).

One process per rank. Each rank builds its send blocks by the wire format the
header states (per-peer blocks of the chunk's heads for the all-to-all form,
padded whole shards for the all-gather form), asserts that the library's
split lists (usp_dist_exchange_counts, which needs no device) give exactly
those block sizes and offsets, runs the real collective
(all_to_all_single / all_gather_into_tensor), unpacks what arrived, and
compares the result bit for bit with the oracle's exchange:
seq_to_head for q, k and v (grouped-query heads, a cls prefix, ragged token
and head splits, every head-chunk count), head_to_seq on the way back, and the
all-gather form against the same. The data are random 32-bit words moved as
int32, so every bit pattern is compared.

The GPU side of the same exchanges (the pack/unpack kernels and the attention
writing into the send blocks) is checked on one device against the oracle in
tests/test_gpu_dist.py; a real multi-GPU NCCL run is not measured here.
"""

import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (batch, seq_len, heads, kv_heads, head_dim, world, prefix, chunk counts)
CASES = [
    (1, 37, 6, 6, 8, 2, 0, (1, 2, 4)),
    (2, 37, 6, 3, 4, 3, 1, (1, 2, 3)),   # grouped-query (2 q heads per kv head), cls prefix
    (1, 40, 7, 7, 4, 3, 1, (1, 2)),      # ragged heads 3,2,2; chunks 2,1 then 2,0
    (1, 29, 10, 10, 4, 4, 1, (1, 3)),    # four ranks: tokens 8,7,7,7, heads 3,3,2,2, cls prefix
    (2, 33, 8, 4, 8, 4, 0, (1, 2)),      # four ranks, grouped-query (one kv head per rank)
]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _chunk_heads(head_ranges, kv_ranges, group, lo, hi, j):
    """The wire format's heads of rank j in chunk window [lo, hi): its query
    heads in the window, and the kv heads whose first query head is in it."""
    h0, h1 = head_ranges[j]
    n = max(0, min(hi, h1 - h0) - lo)
    q0 = h0 + lo
    if n == 0:
        return q0, 0, kv_ranges[j][0], 0
    kv0 = -(-q0 // group)
    kv1 = -(-(q0 + n) // group)
    return q0, n, kv0, kv1 - kv0


def _rank_main(rank, world, port, case, out_q):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from oracle import layout as ol
    from oracle.partition import balanced_ranges, head_chunk_ranges
    from ulysses_sequence_attention_sp_b200 import usp
    from ulysses_sequence_attention_sp_b200.synth import make_bits

    B, T, H, HKV, D, P, pre, chunk_counts = case
    assert P == world
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    failures = []
    try:
        tr = balanced_ranges(T, P)
        hr = balanced_ranges(H, P)
        kr = balanced_ranges(HKV, P)
        group = H // HKV
        full = [make_bits((B, pre + T, h, D), 4, 500 + i).view(np.int32) for i, h in enumerate((H, HKV, HKV))]
        seq = [ol.scatter_sequence(x, tr, prefix=pre) for x in full]        # [tensor][rank]
        mine = [seq[t][rank] for t in range(3)]
        ref_heads = [ol.seq_to_head(seq[0], tr, hr, prefix=pre), ol.seq_to_head(seq[1], tr, kr, prefix=pre),
                     ol.seq_to_head(seq[2], tr, kr, prefix=pre)]
        rows = lambda i: pre + tr[i][1] - tr[i][0]  # noqa: E731

        def check(cond, what):
            if not cond:
                failures.append(what)

        def a2a(send, sc, rc):
            recv = torch.empty(sum(rc), dtype=torch.int32)
            dist.all_to_all_single(recv, torch.from_numpy(send), output_split_sizes=rc, input_split_sizes=sc)
            return recv.numpy()

        def counts(kind, nt, n, c):
            return usp.dist_exchange_counts(B, T, H, D, P, rank, kind, nt, n, c, pre, HKV)

        for n in chunk_counts:
            chunks = head_chunk_ranges(hr[0][1] - hr[0][0], n)
            # ---- seq -> head, all-to-all form
            got = [np.full((B, pre + T, hr[rank][1] - hr[rank][0], D), -1, np.int32),
                   np.full((B, pre + T, kr[rank][1] - kr[rank][0], D), -1, np.int32),
                   np.full((B, pre + T, kr[rank][1] - kr[rank][0], D), -1, np.int32)]
            for c, (lo, hi) in enumerate(chunks):
                sc, sd, rc, rd = counts(usp.DIST_SEQ_TO_HEAD, 3, n, c)
                blocks = []
                for j in range(P):
                    q0, nq, kv0, nkv = _chunk_heads(hr, kr, group, lo, hi, j)
                    blocks.append(np.concatenate([mine[0][:, :, q0:q0 + nq].ravel(), mine[1][:, :, kv0:kv0 + nkv].ravel(),
                                                  mine[2][:, :, kv0:kv0 + nkv].ravel()]))
                check([b.size for b in blocks] == list(sc), f"n={n} c={c} send counts {sc}")
                check(list(np.cumsum([0] + [b.size for b in blocks])[:-1]) == list(sd), f"n={n} c={c} send displs")
                recv = a2a(np.concatenate(blocks), sc, rc)
                q0r, nqr, kv0r, nkvr = _chunk_heads(hr, kr, group, lo, hi, rank)
                off = 0
                for i in range(P):
                    check(rd[i] == off, f"n={n} c={c} recv displ {i}")
                    parts = []
                    for t, (h0, nh) in enumerate(((q0r, nqr), (kv0r, nkvr), (kv0r, nkvr))):
                        size = B * rows(i) * nh * D
                        parts.append(recv[off:off + size].reshape(B, rows(i), nh, D))
                        off += size
                    check(off - rd[i] == rc[i], f"n={n} c={c} recv count {i}")
                    for t, (h0, nh) in enumerate(((q0r, nqr), (kv0r, nkvr), (kv0r, nkvr))):
                        local0 = h0 - (hr[rank][0] if t == 0 else kr[rank][0])
                        dst = got[t][:, :, local0:local0 + nh]
                        if i == 0 and pre:
                            dst[:, :pre] = parts[t][:, :pre]  # the prefix rows from rank 0
                        dst[:, pre + tr[i][0]:pre + tr[i][1]] = parts[t][:, pre:]
            for t in range(3):
                check(np.array_equal(got[t], ref_heads[t][rank]), f"n={n} seq_to_head tensor {t}")

            # ---- head -> seq, all-to-all form: the q head shard back to the q sequence shard
            o = ref_heads[0][rank]
            back = np.full(mine[0].shape, -1, np.int32)
            for c, (lo, hi) in enumerate(chunks):
                sc, sd, rc, rd = counts(usp.DIST_HEAD_TO_SEQ, 1, n, c)
                q0r, nqr, _, _ = _chunk_heads(hr, kr, group, lo, hi, rank)
                l0 = q0r - hr[rank][0]
                blocks = []
                for j in range(P):
                    rows_j = np.concatenate([np.arange(pre), pre + np.arange(tr[j][0], tr[j][1])]).astype(int)
                    blocks.append(np.ascontiguousarray(o[:, rows_j, l0:l0 + nqr]).ravel())
                check([b.size for b in blocks] == list(sc), f"n={n} c={c} head_to_seq send counts")
                recv = a2a(np.concatenate(blocks), sc, rc)
                for i in range(P):
                    qi0, nqi, _, _ = _chunk_heads(hr, kr, group, lo, hi, i)
                    check(rc[i] == B * rows(rank) * nqi * D, f"n={n} c={c} head_to_seq recv count {i}")
                    back[:, :, qi0:qi0 + nqi] = recv[rd[i]:rd[i] + rc[i]].reshape(B, rows(rank), nqi, D)
            check(np.array_equal(back, mine[0]), f"n={n} head_to_seq round trip")

        # ---- the all-gather form (prefer_all_gather): padded whole shards
        sc, sd, rc, rd = counts(usp.DIST_GATHER_SEQ, 3, 1, 0)
        block = sc[0]
        check(block == max(B * rows(i) * D * (H + 2 * HKV) for i in range(P)), "gather block size")
        check(list(rd) == [i * block for i in range(P)], "gather displs")
        mine_block = np.concatenate([x.ravel() for x in mine])
        send = np.zeros(block, np.int32)
        send[:mine_block.size] = mine_block
        recv = torch.empty(block * P, dtype=torch.int32)
        dist.all_gather_into_tensor(recv, torch.from_numpy(send))
        recv = recv.numpy()
        shards = [[], [], []]
        for i in range(P):
            off = rd[i]
            for t, h in enumerate((H, HKV, HKV)):
                size = B * rows(i) * h * D
                shards[t].append(recv[off:off + size].reshape(B, rows(i), h, D))
                off += size
        for t, ranges in enumerate((hr, kr, kr)):
            gathered = ol.gather_sequence(shards[t], tr, prefix=pre)
            check(np.array_equal(ol.sp_head_slice(gathered, ranges)[rank], ref_heads[t][rank]), f"gather form {t}")
        out_q.put((rank, failures))
        dist.barrier()
    except Exception as e:  # reported to the parent
        out_q.put((rank, [repr(e)]))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}-T{c[1]}-H{c[2]}-KV{c[3]}-P{c[5]}-pre{c[6]}")
def test_transport_over_gloo_matches_oracle(case):
    world = case[5]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(world):
        rank, failures = q.get(timeout=180)
        results[rank] = failures
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(not f for f in results.values()), results


def test_exchange_counts_need_no_device_and_reject_bad_arguments():
    sys.path.insert(0, ROOT)
    from ulysses_sequence_attention_sp_b200 import usp
    sc, sd, rc, rd = usp.dist_exchange_counts(1, 10, 3, 4, 3, 1, usp.DIST_SEQ_TO_HEAD, 1)
    # rank 1 of 3 (tokens 4,3,3; heads 1,1,1): sends [3 rows][1 head][4] to each peer
    assert sc == [12, 12, 12] and sd == [0, 12, 24]
    assert rc == [16, 12, 12] and rd == [0, 16, 28]
    for bad in [dict(rank=3), dict(exchange=9), dict(ntensors=2), dict(num_chunks=0), dict(chunk=1)]:
        kw = dict(rank=1, exchange=usp.DIST_SEQ_TO_HEAD, ntensors=1, num_chunks=1, chunk=0) | bad
        with pytest.raises(usp.UspError) as e:
            usp.dist_exchange_counts(1, 10, 3, 4, 3, kw["rank"], kw["exchange"], kw["ntensors"], kw["num_chunks"],
                                     kw["chunk"])
        assert e.value.code == usp.USP_ERR_INVALID_ARG

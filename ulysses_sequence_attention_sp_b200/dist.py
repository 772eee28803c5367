"""The Ulysses block across processes: one process per GPU and per
sequence-parallel rank, the exchanges run by torch.distributed (NCCL).

"h3_blackwell_runtime/distributed.py -- Ragged Ulysses sequence-parallel
transport", seq_to_heads / heads_to_seq: every rank packs one block per peer
(the library's pack kernels), the blocks travel in one ragged
``all_to_all_single`` whose split lists come from the library
(``usp_dist_exchange_counts``), and every rank unpacks what it receives.
"maxdiffusion PR #428": with head chunks, the exchange of chunk c+1 is in
flight while chunk c is attended. API page "mstar.model.components.
distributed.sequence_parallel", ulysses_attention(prefer_all_gather=True):
the same result through equal-size all-gathers, which a captured CUDA graph can
replay.

Every computation is a call into libusp (packs, unpacks, the attention with
its output written straight into the send blocks of the way back); this module
only allocates the flat send/receive buffers and issues the collectives. It
needs CUDA tensors and a process group whose backend moves CUDA tensors
(NCCL); there is no CPU path.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from . import usp


class SequenceParallelGroup:
    """This process's rank of a sequence-parallel group.

    Sizes are those of the whole sequence (every rank passes the same); the
    token and head splits follow the balanced rule, as in the one-device plan.
    `rank` and `world` default to the group's."""

    def __init__(self, batch: int, seq_len: int, heads: int, head_dim: int, dtype="bf16", prefix: int = 0,
                 kv_heads: int | None = None, group=None, rank: int | None = None, world: int | None = None):
        self.group = group
        self.rank = dist.get_rank(group) if rank is None else rank
        self.world = dist.get_world_size(group) if world is None else world
        self.plan = usp.Plan(batch, seq_len, heads, head_dim, self.world, dtype, prefix, kv_heads=kv_heads)
        self.dtype = self.plan.torch_dtype
        self._ws = None

    # ------------------------------------------------------------ buffers
    def _flat(self, n: int):
        return torch.empty(max(int(n), 1), dtype=self.dtype, device="cuda")

    def _workspace(self):
        need = usp.dist_workspace_bytes(self.plan, self.rank)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        return self._ws

    def counts(self, exchange: int, ntensors: int = 1, num_chunks: int = 1, chunk: int = 0):
        return usp.dist_counts(self.plan, self.rank, exchange, ntensors, num_chunks, chunk)

    # -------------------------------------------------------- collectives
    def _all_to_all(self, send, counts, async_op=False):
        sc, _sd, rc, _rd = counts
        recv = self._flat(sum(rc))
        work = dist.all_to_all_single(recv[:sum(rc)], send[:sum(sc)], output_split_sizes=list(rc),
                                      input_split_sizes=list(sc), group=self.group, async_op=async_op)
        return recv, work

    def _all_gather(self, send, counts, async_op=False):
        block = counts[0][0]
        recv = self._flat(block * self.world)
        work = dist.all_gather_into_tensor(recv[:block * self.world], send[:block], group=self.group,
                                          async_op=async_op)
        return recv, work

    # ------------------------------------------------------------- layout
    def seq_to_head(self, q, k=None, v=None, num_chunks: int = 1, prefer_all_gather: bool = False):
        """Transport page, seq_to_heads: this rank's sequence shards
        [B, p+T_r, H(kv), D] -> its head shards [B, T', H_r(kv), D]."""
        ins = [t for t in (q, k, v) if t is not None]
        nt = len(ins)
        plan, r = self.plan, self.rank
        shapes = [plan.head_shard_shape(r)] + [plan.kv_head_shard_shape(r)] * (nt - 1)
        outs = [torch.empty(s, dtype=self.dtype, device="cuda") for s in shapes]
        kind = usp.DIST_GATHER_SEQ if prefer_all_gather else usp.DIST_SEQ_TO_HEAD
        if prefer_all_gather:
            cnt = self.counts(kind, nt)
            send = self._flat(cnt[0][0])
            usp.dist_pack(plan, r, kind, ins, send)
            recv, _ = self._all_gather(send, cnt)
            for c in range(len(self._chunks(num_chunks))):
                usp.dist_unpack(plan, r, kind, recv, outs, num_chunks, c)
            return outs
        for c in range(len(self._chunks(num_chunks))):
            cnt = self.counts(kind, nt, num_chunks, c)
            send = self._flat(sum(cnt[0]))
            usp.dist_pack(plan, r, kind, ins, send, num_chunks, c)
            recv, _ = self._all_to_all(send, cnt)
            usp.dist_unpack(plan, r, kind, recv, outs, num_chunks, c)
        return outs

    def head_to_seq(self, o_heads, num_chunks: int = 1, prefer_all_gather: bool = False):
        """Transport page, heads_to_seq: this rank's head shard [B, T', H_r, D]
        -> its sequence shard [B, p+T_r, H, D]."""
        plan, r = self.plan, self.rank
        out = torch.empty(plan.seq_shard_shape(r), dtype=self.dtype, device="cuda")
        kind = usp.DIST_GATHER_HEADS if prefer_all_gather else usp.DIST_HEAD_TO_SEQ
        for c in range(len(self._chunks(num_chunks))):
            cnt = self.counts(kind, 1, num_chunks, c)
            send = self._flat(cnt[0][0] if prefer_all_gather else sum(cnt[0]))
            usp.dist_pack(plan, r, kind, [o_heads], send, num_chunks, c)
            recv, _ = (self._all_gather if prefer_all_gather else self._all_to_all)(send, cnt)
            usp.dist_unpack(plan, r, kind, recv, [out], num_chunks, c)
        return out

    def _chunks(self, num_chunks: int):
        return usp.head_chunk_ranges(self.plan.head_ranges[0][1] - self.plan.head_ranges[0][0], num_chunks)

    # ---------------------------------------------------------- attention
    def ulysses_attention(self, q, k, v, num_chunks: int = 1, prefer_all_gather: bool = False, scale: float = 0.0,
                          out=None):
        """API page, ulysses_attention, across processes: this rank's sequence
        shards of q [B, p+T_r, H, D] and k, v [B, p+T_r, Hkv, D] in, its
        sequence shard of the attention output out. With num_chunks > 1 the
        exchange of head chunk c+1 is in flight while chunk c is attended
        (cap the attention's CTAs with plan.set_attention_ctas to leave SMs
        to the collective's kernels)."""
        plan, r = self.plan, self.rank
        out = torch.empty(plan.seq_shard_shape(r), dtype=self.dtype, device="cuda") if out is None else out
        ws = self._workspace()
        nchunks = len(self._chunks(num_chunks))
        if prefer_all_gather:
            cnt = self.counts(usp.DIST_GATHER_SEQ, 3)
            send = self._flat(cnt[0][0])
            usp.dist_pack(plan, r, usp.DIST_GATHER_SEQ, [q, k, v], send)
            recv, _ = self._all_gather(send, cnt)
            for c in range(nchunks):
                cnt_o = self.counts(usp.DIST_GATHER_HEADS, 1, num_chunks, c)
                send_o = self._flat(cnt_o[0][0])
                usp.dist_attention(plan, r, usp.DIST_GATHER_SEQ, recv, send_o, ws, num_chunks, c, scale)
                recv_o, _ = self._all_gather(send_o, cnt_o)
                usp.dist_unpack(plan, r, usp.DIST_GATHER_HEADS, recv_o, [out], num_chunks, c)
            return out
        # all-to-all form: chunk c+1's q/k/v are exchanged while chunk c is attended
        pending = []

        def start(c):
            cnt = self.counts(usp.DIST_SEQ_TO_HEAD, 3, num_chunks, c)
            send = self._flat(sum(cnt[0]))
            usp.dist_pack(plan, r, usp.DIST_SEQ_TO_HEAD, [q, k, v], send, num_chunks, c)
            recv, work = self._all_to_all(send, cnt, async_op=True)
            return send, recv, work

        inflight = start(0)
        for c in range(nchunks):
            nxt = start(c + 1) if c + 1 < nchunks else None
            send, recv, work = inflight
            work.wait()
            cnt_o = self.counts(usp.DIST_HEAD_TO_SEQ, 1, num_chunks, c)
            send_o = self._flat(sum(cnt_o[0]))
            usp.dist_attention(plan, r, usp.DIST_SEQ_TO_HEAD, recv, send_o, ws, num_chunks, c, scale)
            recv_o, work_o = self._all_to_all(send_o, cnt_o, async_op=True)
            pending.append((c, send_o, recv_o, work_o, send, recv))
            inflight = nxt
        for c, _send_o, recv_o, work_o, _send, _recv in pending:
            work_o.wait()
            usp.dist_unpack(plan, r, usp.DIST_HEAD_TO_SEQ, recv_o, [out], num_chunks, c)
        return out

    def close(self):
        self.plan.close()

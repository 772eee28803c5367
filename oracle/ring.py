"""The Ulysses + Ring hybrid block (oracle; test infrastructure only).

Sources:

* "maxdiffusion PR #428: experimental two-phase (head-chunked) Ulysses
  all-to-all": the context axis runs Ulysses and Ring together (the PR applies
  the same head-chunked passes to plain Ulysses and to Ulysses+Ring, the last
  chunk carrying the remainder).
* "mstar.model.components.distributed.sequence_parallel", ulysses_attention:
  the Ulysses exchange (sequence shards -> head shards and back) around an
  unchanged attention.
* "h3_blackwell_runtime/distributed.py -- Ragged Ulysses sequence-parallel
  transport": the ragged token and head splits (``balanced_ranges``).

The pages name the hybrid but print none of its steps, so this module takes
the plainest reading that the rest supports (each point is also listed in
the design notes):

* ``P = ulysses_size * ring_size`` ranks; tokens are split over all P ranks
  by the balanced rule. Ulysses group g is the consecutive ranks
  ``g*ulysses_size .. (g+1)*ulysses_size - 1``; it owns the contiguous union
  of its members' token windows (block g of the sequence).
* Inside a group the Ulysses exchange runs as in the plain block, with heads
  split over the group's ``ulysses_size`` members by the balanced rule. Rank
  (g, u) then holds heads H_u for the tokens of block g.
* Ranks with the same u form a ring of ``ring_size``. Step s of the ring
  gives rank (g, u) the k/v of block ``(g - s) mod ring_size`` (its own block
  first, then the block of the previous ring rank, and so on). Each step
  yields a partial output normalised over that block and its log-sum-exp;
  partials merge by log-sum-exp weights.
* A replicated prefix (cls) row is a query on every rank but a key only once:
  it belongs to block 0's keys.
* The output goes back through the group's head->seq exchange.
"""

from __future__ import annotations

import numpy as np

from .attention import default_scale
from .layout import head_to_seq, seq_to_head
from .partition import balanced_ranges, check_gqa_ranges, gqa_group, head_chunk_ranges, range_lengths


def block_attention(q, k, v, scale):
    """One ring step for one head: q ``[Tq, D]`` over a k/v block ``[Tk, D]``.

    Returns ``(o, lse)``: ``o = softmax(q k^T * scale) v`` normalised over the
    block, and ``lse[i] = log sum_j exp(scale * q_i . k_j)`` (natural log).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    scores = (q @ k.T) * scale
    m = scores.max(axis=1, keepdims=True)
    w = np.exp(scores - m)
    l = w.sum(axis=1, keepdims=True)
    return (w @ v) / l, (m + np.log(l))[:, 0]


def merge_partials(o_a, lse_a, o_b, lse_b):
    """Combine two partial outputs of disjoint key sets by their log-sum-exps:
    the merged log-sum-exp is ``log(exp(lse_a) + exp(lse_b))`` and each partial
    is weighted by ``exp(lse_x - lse)``."""
    lse = np.logaddexp(lse_a, lse_b)
    return o_a * np.exp(lse_a - lse)[:, None] + o_b * np.exp(lse_b - lse)[:, None], lse


def ring_groups(token_ranges, ulysses_size: int, ring_size: int):
    """Per Ulysses group: (member ranks, (start, stop) of its token block,
    members' token windows relative to the block start)."""
    if ulysses_size < 1 or ring_size < 1 or len(token_ranges) != ulysses_size * ring_size:
        raise ValueError("world must equal ulysses_size * ring_size")
    groups = []
    for g in range(ring_size):
        members = list(range(g * ulysses_size, (g + 1) * ulysses_size))
        start, stop = token_ranges[members[0]][0], token_ranges[members[-1]][1]
        local = tuple((a - start, b - start) for a, b in (token_ranges[r] for r in members))
        groups.append((members, (start, stop), local))
    return groups


def ulysses_ring_attention(q_shards, k_shards, v_shards, token_ranges, ulysses_size: int, ring_size: int, *,
                           num_chunks=1, scale=None, prefix=0):
    """The hybrid block on per-rank sequence shards ``[B, prefix+T_i, H, D]``
    (k/v may carry fewer heads: grouped-query attention). Returns per-rank
    sequence shards of the float64 output."""
    heads_q, heads_kv = q_shards[0].shape[2], k_shards[0].shape[2]
    group = gqa_group(heads_q, heads_kv)
    hr = balanced_ranges(heads_q, ulysses_size)
    kr = balanced_ranges(heads_kv, ulysses_size)
    check_gqa_ranges(hr, kr, group)
    if scale is None:
        scale = default_scale(q_shards[0].shape[3])
    groups = ring_groups(token_ranges, ulysses_size, ring_size)

    # 1. seq -> head inside every Ulysses group
    qh, kh, vh = [], [], []
    for members, _block, local in groups:
        qh.append(seq_to_head([q_shards[r] for r in members], local, hr, prefix=prefix))
        kh.append(seq_to_head([k_shards[r] for r in members], local, kr, prefix=prefix))
        vh.append(seq_to_head([v_shards[r] for r in members], local, kr, prefix=prefix))

    def kv_block(x, gp, u, b, kv):
        rows = x[gp][u][b, prefix:, kv]
        if gp == 0 and prefix:
            rows = np.concatenate([x[gp][u][b, :prefix, kv], rows], axis=0)
        return rows

    # 2. ring attention of every rank (g, u) over each head chunk
    counts = range_lengths(hr)
    oh = [[np.full(x.shape, np.nan, dtype=np.float64) for x in qg] for qg in qh]
    for lo, hi in head_chunk_ranges(max(counts), num_chunks):
        for g in range(ring_size):
            for u, count in enumerate(counts):
                for i in range(min(lo, count), min(hi, count)):
                    kv = (hr[u][0] + i) // group - kr[u][0]
                    for b in range(q_shards[0].shape[0]):
                        q = qh[g][u][b, :, i]
                        o = lse = None
                        for s in range(ring_size):
                            gp = (g - s) % ring_size
                            o_s, lse_s = block_attention(q, kv_block(kh, gp, u, b, kv), kv_block(vh, gp, u, b, kv),
                                                         scale)
                            if o is None:
                                o, lse = o_s, lse_s
                            else:
                                o, lse = merge_partials(o, lse, o_s, lse_s)
                        oh[g][u][b, :, i] = o

    # 3. head -> seq inside every group
    out = [None] * len(token_ranges)
    for g, (members, _block, local) in enumerate(groups):
        for r, shard in zip(members, head_to_seq(oh[g], local, hr, prefix=prefix)):
            out[r] = shard
    return out

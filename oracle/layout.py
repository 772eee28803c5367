"""Layout operations of the Ulysses block (oracle; test infrastructure only).

Each virtual rank is its own numpy array; lists are indexed by rank. The
operations only move values, so any dtype works (tests feed raw bit patterns).

Tensors use the BSHD layout of the ragged transport page,
``[batch, tokens, heads, head_dim]``. ``prefix`` leading token rows (the cls
token of "deepspeed/sequence/autosp_vit.py", ``UlyssesSPViTAttention``) are
replicated on every sequence shard rather than split.

Sources:

* "mstar.model.components.distributed.sequence_parallel": ``scatter_sequence``
  (each rank narrows a replicated tensor to its window, no communication),
  ``gather_sequence`` (shards concatenated in rank order), ``sp_head_slice``
  (a rank keeps its contiguous head group), ``sp_head_gather`` (its inverse,
  an all-gather over heads).
* "h3_blackwell_runtime/distributed.py -- Ragged Ulysses sequence-parallel
  transport", ``SequenceParallelContext.seq_to_heads``: every rank cuts its
  local tokens into one chunk per destination (the destination's head
  range); every destination concatenates the chunks it receives along the
  token axis in source-rank order. ``heads_to_seq``: every rank cuts its
  full-sequence output into one chunk per destination (the destination's
  token rows); every destination concatenates what it receives along the
  head axis in source-rank order.

Readings: the scatter is materialised into separate per-rank arrays (virtual
ranks own separate memory); the cls rows are taken from rank 0 on the way in
(the replicas are equal, which :func:`seq_to_head` asserts) and written to
every rank on the way out.
"""

from __future__ import annotations

import numpy as np

TOKEN_AXIS = 1
HEAD_AXIS = 2


def _take(x, axis, start, stop):
    index = [slice(None)] * x.ndim
    index[axis] = slice(start, stop)
    return x[tuple(index)]


def scatter_sequence(x_full, token_ranges, *, axis=TOKEN_AXIS, prefix=0):
    """Per-rank copies of each rank's token window (plus the replicated prefix)."""
    shards = []
    for start, stop in token_ranges:
        parts = []
        if prefix:
            parts.append(_take(x_full, axis, 0, prefix))
        parts.append(_take(x_full, axis, prefix + start, prefix + stop))
        shards.append(np.ascontiguousarray(np.concatenate(parts, axis=axis)))
    return shards


def gather_sequence(shards, token_ranges, *, axis=TOKEN_AXIS, prefix=0):
    """Full tensor from the shards, in rank order (prefix taken from rank 0)."""
    parts = []
    if prefix:
        parts.append(_take(shards[0], axis, 0, prefix))
    for shard, (start, stop) in zip(shards, token_ranges, strict=True):
        if shard.shape[axis] != prefix + (stop - start):
            raise ValueError("shard length does not match its token range")
        parts.append(_take(shard, axis, prefix, prefix + stop - start))
    return np.ascontiguousarray(np.concatenate(parts, axis=axis))


def sp_head_slice(x_full, head_ranges, *, axis=HEAD_AXIS):
    """Per-rank copies of each rank's contiguous head group."""
    return [np.ascontiguousarray(_take(x_full, axis, h0, h1)) for h0, h1 in head_ranges]


def sp_head_gather(head_shards, *, axis=HEAD_AXIS):
    """Inverse of :func:`sp_head_slice`: concatenation over the head axis."""
    return np.ascontiguousarray(np.concatenate(head_shards, axis=axis))


def seq_to_head(seq_shards, token_ranges, head_ranges, *, prefix=0):
    """Sequence shards ``[B, prefix+T_i, H, D]`` -> head shards ``[B, prefix+T, H_r, D]``.

    Written as the exchange itself: ``send[i][r]`` is what rank ``i`` sends
    to rank ``r``; rank ``r`` concatenates ``send[i][r]`` over ``i``.
    """
    world = len(token_ranges)
    if len(seq_shards) != world or len(head_ranges) != world:
        raise ValueError("one shard and one head range per rank")
    for i, (start, stop) in enumerate(token_ranges):
        if seq_shards[i].shape[TOKEN_AXIS] != prefix + stop - start:
            raise ValueError(f"rank {i} shard has the wrong token count")
    if prefix:
        for i in range(1, world):
            if not np.array_equal(
                _take(seq_shards[i], TOKEN_AXIS, 0, prefix).view(np.uint8),
                _take(seq_shards[0], TOKEN_AXIS, 0, prefix).view(np.uint8),
            ):
                raise ValueError("replicated prefix rows differ between ranks")
    send = [
        [
            _take(_take(seq_shards[i], TOKEN_AXIS, prefix, None), HEAD_AXIS, h0, h1)
            for (h0, h1) in head_ranges
        ]
        for i in range(world)
    ]
    out = []
    for r, (h0, h1) in enumerate(head_ranges):
        parts = []
        if prefix:
            parts.append(_take(_take(seq_shards[0], TOKEN_AXIS, 0, prefix), HEAD_AXIS, h0, h1))
        parts.extend(send[i][r] for i in range(world))
        out.append(np.ascontiguousarray(np.concatenate(parts, axis=TOKEN_AXIS)))
    return out


def head_to_seq(head_shards, token_ranges, head_ranges, *, prefix=0):
    """Head shards ``[B, prefix+T, H_r, D]`` -> sequence shards ``[B, prefix+T_i, H, D]``.

    ``send[r][i]`` holds rank ``i``'s token rows of rank ``r``'s heads; rank
    ``i`` concatenates ``send[r][i]`` over ``r`` along the head axis. The
    prefix rows go to every rank.
    """
    world = len(token_ranges)
    if len(head_shards) != world or len(head_ranges) != world:
        raise ValueError("one shard and one head range per rank")
    for r, (h0, h1) in enumerate(head_ranges):
        if head_shards[r].shape[HEAD_AXIS] != h1 - h0:
            raise ValueError(f"rank {r} head shard has the wrong head count")
    send = [
        [
            _take(head_shards[r], TOKEN_AXIS, prefix + start, prefix + stop)
            for (start, stop) in token_ranges
        ]
        for r in range(world)
    ]
    out = []
    for i in range(world):
        received = np.concatenate([send[r][i] for r in range(world)], axis=HEAD_AXIS)
        if prefix:
            cls_rows = np.concatenate(
                [_take(head_shards[r], TOKEN_AXIS, 0, prefix) for r in range(world)],
                axis=HEAD_AXIS,
            )
            received = np.concatenate([cls_rows, received], axis=TOKEN_AXIS)
        out.append(np.ascontiguousarray(received))
    return out

"""Ragged row collectives of the sequence-parallel context (oracle; test
infrastructure only).

Source: "h3_blackwell_runtime/distributed.py -- Ragged Ulysses sequence-parallel
transport", ``SequenceParallelContext.all_gather_rows`` and
``SequenceParallelContext.reduce_scatter_rows``.

* ``all_gather_rows``: every rank contributes its own ``T_r`` token rows; the
  page pads each contribution with zero rows to the longest rank's count, runs
  an all-gather of the padded blocks, and every rank keeps the first ``T_i``
  rows of block ``i``, concatenated in rank order. Every rank ends up with all
  ``T`` rows; the padding never reaches the result.
* ``reduce_scatter_rows``: every rank holds a partial sum over all ``T`` rows
  (tensor-parallel partials). It cuts them into one chunk per destination (the
  destination's token rows), an all-to-all delivers chunk ``r`` of every source
  to rank ``r``, and rank ``r`` sums what it received over the source axis.

Each virtual rank is its own numpy array; lists are indexed by rank. Arrays are
``[outer, rows, ...]`` (token axis 1, like the rest of the oracle); the page
has no outer axis, which is the ``outer = 1`` case. The prefix (cls) rows of
the attention block take no part: the page's context has none.

Readings (also listed in the design notes): a one-rank group copies (the page
returns its input object; virtual ranks own separate buffers); the sum is
taken in float64 on the exact values, in source-rank order, the order the
page's ``sum(dim=0)`` runs over the received blocks.
"""

from __future__ import annotations

import numpy as np

from .partition import range_lengths

TOKEN_AXIS = 1


def _rows(x, start, stop):
    return x[:, start:stop]


def all_gather_rows(local_rows, token_ranges):
    """Per-rank full ``[outer, T, ...]`` arrays from per-rank ``[outer, T_r, ...]`` rows."""
    world = len(token_ranges)
    lengths = range_lengths(token_ranges)
    if len(local_rows) != world:
        raise ValueError("one contribution per rank")
    for r, (x, n) in enumerate(zip(local_rows, lengths)):
        if x.shape[TOKEN_AXIS] != n:
            raise ValueError(f"rank {r} must contribute {n} rows, got {x.shape[TOKEN_AXIS]}")
    if world == 1:
        return [np.array(local_rows[0], copy=True)]
    max_rows = max(lengths)
    padded = []
    for x in local_rows:
        block = np.zeros((x.shape[0], max_rows, *x.shape[2:]), dtype=x.dtype)
        block[:, : x.shape[TOKEN_AXIS]] = x
        padded.append(block)
    # all-gather: every rank receives the same list of padded blocks
    received = [list(padded) for _ in range(world)]
    out = []
    for r in range(world):
        parts = [_rows(block, 0, n) for block, n in zip(received[r], lengths, strict=True)]
        out.append(np.ascontiguousarray(np.concatenate(parts, axis=TOKEN_AXIS)))
    return out


def reduce_scatter_rows(partials, token_ranges):
    """Per-rank ``[outer, T_r, ...]`` sums (float64) of the ranks' ``[outer, T, ...]`` partials."""
    world = len(token_ranges)
    total = token_ranges[-1][1]
    if len(partials) != world:
        raise ValueError("one partial per rank")
    for r, x in enumerate(partials):
        if x.shape[TOKEN_AXIS] != total:
            raise ValueError(f"rank {r}: partial rows must cover {total} rows, got {x.shape[TOKEN_AXIS]}")
    if world == 1:
        return [np.asarray(partials[0], dtype=np.float64).copy()]
    # send[i][r]: rank i's rows of destination r
    send = [[_rows(x, start, stop) for start, stop in token_ranges] for x in partials]
    out = []
    for r in range(world):
        received = [send[i][r] for i in range(world)]
        acc = np.asarray(received[0], dtype=np.float64).copy()
        for block in received[1:]:
            acc = acc + np.asarray(block, dtype=np.float64)
        out.append(acc)
    return out

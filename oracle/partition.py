"""Partition arithmetic of the Ulysses block (oracle; test infrastructure only).

Sources:

* "h3_blackwell_runtime/distributed.py -- Ragged Ulysses sequence-parallel
  transport", ``balanced_ranges`` and ``range_lengths``: ``total`` ordered
  items are cut into ``parts`` contiguous, non-empty ranges whose lengths are
  ``total // parts`` plus one for each of the first ``total % parts`` ranks.
  Fewer items than parts, or fewer than one part, is an error.
* "mstar.model.components.distributed.sequence_parallel", ``sp_seq_split``:
  even per-rank token counts summing to the total, earlier ranks taking the
  remainder.
* "maxdiffusion PR #428: experimental two-phase (head-chunked) Ulysses
  all-to-all", description: the exchange and the attention run in
  ``num_chunks`` head-group passes, the final chunk carrying the remainder.

Readings taken where the pages leave a step open (each also listed in the
design notes):

* ``sp_seq_split`` raises, like ``balanced_ranges``, when ``total < world``
  (the API page is silent; the transport page raises).
* Head-chunk sizes: ``s = ceil(G / n)``; chunk ``c`` holds local heads
  ``[c*s, min((c+1)*s, G))``; empty chunks are dropped, so ``n > G`` behaves
  as ``n = G``. This is the reading under which 5 heads in 3 chunks split
  2, 2, 1 ("remainder last").
* Under ragged head ranges, ``G`` is the largest per-rank head count and the
  same local-head window is used on every rank, clipped to that rank's count.
"""

from __future__ import annotations


def balanced_ranges(total: int, parts: int) -> tuple[tuple[int, int], ...]:
    """Contiguous non-empty ``(start, stop)`` ranges covering ``range(total)``.

    Follows ``balanced_ranges`` of the ragged transport page: ``divmod`` gives
    the base length and the count of ranks that take one extra item; those
    ranks come first.
    """
    if int(parts) != parts or int(total) != total:
        raise ValueError("total and parts must be integers")
    if parts < 1:
        raise ValueError("parts must be positive")
    if total < parts:
        raise ValueError(f"cannot split {total} items into {parts} non-empty ranges")
    base, extra = divmod(total, parts)
    ranges = []
    start = 0
    for rank in range(parts):
        length = base + (1 if rank < extra else 0)
        ranges.append((start, start + length))
        start += length
    return tuple(ranges)


def range_lengths(ranges) -> tuple[int, ...]:
    """Length of each ``(start, stop)`` range."""
    return tuple(stop - start for start, stop in ranges)


def sp_seq_split(total: int, world_size: int) -> list[int]:
    """Per-rank token counts (``sp_seq_split`` of the API page)."""
    return list(range_lengths(balanced_ranges(total, world_size)))


def head_chunk_ranges(group_heads: int, num_chunks: int) -> list[tuple[int, int]]:
    """Local-head windows of the head-chunked passes.

    ``group_heads`` is the (largest) number of heads a rank owns; the result
    lists ``(lo, hi)`` windows of local head indices, in pass order.
    """
    if num_chunks < 1:
        raise ValueError("num_chunks must be positive")
    if group_heads < 1:
        raise ValueError("group_heads must be positive")
    size = -(-group_heads // num_chunks)  # ceil
    chunks = []
    lo = 0
    while lo < group_heads:
        hi = min(lo + size, group_heads)
        chunks.append((lo, hi))
        lo = hi
    return chunks


def rank_chunk_heads(head_ranges, num_chunks: int) -> list[list[tuple[int, int]]]:
    """Per chunk, per rank: the global head range ``[g0, g1)`` that rank
    attends to in that pass (possibly empty) under ragged head ranges."""
    counts = range_lengths(head_ranges)
    chunks = head_chunk_ranges(max(counts), num_chunks)
    out = []
    for lo, hi in chunks:
        per_rank = []
        for (h0, _h1), count in zip(head_ranges, counts):
            a = min(lo, count)
            b = min(hi, count)
            per_rank.append((h0 + a, h0 + b))
        out.append(per_rank)
    return out


def gqa_group(heads_q: int, heads_kv: int) -> int:
    """Query heads per kv head. The API page's ulysses_attention takes q with
    Hq heads and k/v with Hkv heads; each kv head serves Hq / Hkv consecutive
    query heads."""
    if heads_kv < 1 or heads_q % heads_kv != 0:
        raise ValueError(f"query heads ({heads_q}) must be a multiple of kv heads ({heads_kv})")
    return heads_q // heads_kv


def check_gqa_ranges(head_ranges, kv_head_ranges, group: int) -> None:
    """Every rank must own the kv heads its query heads use (the head split must
    keep groups whole on each rank, as a sharding divisible by the group size
    does). Raises ValueError otherwise."""
    for r, ((h0, h1), (k0, k1)) in enumerate(zip(head_ranges, kv_head_ranges, strict=True)):
        for h in range(h0, h1):
            if not k0 <= h // group < k1:
                raise ValueError(f"rank {r}: query head {h} uses kv head {h // group}, outside its kv heads [{k0}, {k1})")

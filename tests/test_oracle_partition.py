"""Pins for oracle.partition: worked splits, error cases, closed forms."""

import json
import os
import random

import pytest

from oracle.partition import (
    balanced_ranges,
    head_chunk_ranges,
    range_lengths,
    rank_chunk_heads,
    sp_seq_split,
)


def test_golden_balanced_ranges(golden_dir):
    with open(os.path.join(golden_dir, "balanced_ranges.json")) as f:
        golden = json.load(f)
    for case in golden["cases"]:
        ranges = balanced_ranges(case["total"], case["parts"])
        if "ranges" in case:
            assert [list(r) for r in ranges] == case["ranges"], case["cite"]
        assert list(range_lengths(ranges)) == case.get("lengths", list(range_lengths(ranges))), case["cite"]
        assert sp_seq_split(case["total"], case["parts"]) == list(range_lengths(ranges))
    for case in golden["errors"]:
        with pytest.raises(ValueError):
            balanced_ranges(case["total"], case["parts"])
        with pytest.raises(ValueError):
            sp_seq_split(case["total"], case["parts"])


def test_balanced_ranges_closed_form():
    # A second, independent closed form: rank r of p gets ceil((n - r) / p) items.
    rnd = random.Random(7)
    for _ in range(2000):
        parts = rnd.randint(1, 40)
        total = rnd.randint(parts, 5000)
        ranges = balanced_ranges(total, parts)
        lengths = range_lengths(ranges)
        assert list(lengths) == [-(-(total - r) // parts) for r in range(parts)]
        assert ranges[0][0] == 0 and ranges[-1][1] == total
        assert all(ranges[i][1] == ranges[i + 1][0] for i in range(parts - 1))
        assert min(lengths) >= 1 and max(lengths) - min(lengths) <= 1
        assert list(lengths) == sorted(lengths, reverse=True)


def test_balanced_ranges_edge_cases():
    assert balanced_ranges(1, 1) == ((0, 1),)
    assert balanced_ranges(7, 7) == tuple((i, i + 1) for i in range(7))
    assert balanced_ranges(8, 1) == ((0, 8),)
    with pytest.raises(ValueError):
        balanced_ranges(0, 1)
    with pytest.raises(ValueError):
        balanced_ranges(3, -1)


def test_golden_head_chunks(golden_dir):
    with open(os.path.join(golden_dir, "head_chunks.json")) as f:
        golden = json.load(f)
    for case in golden["cases"]:
        chunks = head_chunk_ranges(case["group_heads"], case["num_chunks"])
        assert [hi - lo for lo, hi in chunks] == case["sizes"], case["cite"]


def test_head_chunks_properties():
    for g in range(1, 30):
        for n in range(1, 35):
            chunks = head_chunk_ranges(g, n)
            sizes = [hi - lo for lo, hi in chunks]
            assert chunks[0][0] == 0 and chunks[-1][1] == g
            assert all(chunks[i][1] == chunks[i + 1][0] for i in range(len(chunks) - 1))
            assert all(s >= 1 for s in sizes)
            assert len(chunks) <= n
            # every chunk but the last has the same size; the last carries the remainder
            assert len(set(sizes[:-1])) <= 1 and sizes[-1] <= sizes[0]
            assert sizes[0] == -(-g // n)
    assert head_chunk_ranges(4, 3) == [(0, 2), (2, 4)]
    assert head_chunk_ranges(3, 10) == [(0, 1), (1, 2), (2, 3)]
    assert head_chunk_ranges(6, 1) == [(0, 6)]
    with pytest.raises(ValueError):
        head_chunk_ranges(4, 0)


def test_rank_chunk_heads_ragged():
    # tiny ragged block: heads 2,2,1,1 in two chunks -> 1,1,1,1 then 1,1,0,0
    hr = balanced_ranges(6, 4)
    per_chunk = rank_chunk_heads(hr, 2)
    assert [[b - a for a, b in c] for c in per_chunk] == [[1, 1, 1, 1], [1, 1, 0, 0]]
    # every head appears in exactly one chunk, on the rank that owns it
    seen = []
    for c in per_chunk:
        for r, (a, b) in enumerate(c):
            for g in range(a, b):
                assert hr[r][0] <= g < hr[r][1]
                seen.append(g)
    assert sorted(seen) == list(range(6))

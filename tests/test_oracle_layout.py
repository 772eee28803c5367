"""Pins for oracle.layout: invariants, world=1 identity, element-wise brute force."""

import itertools

import numpy as np
import pytest

from oracle.layout import (
    gather_sequence,
    head_to_seq,
    scatter_sequence,
    seq_to_head,
    sp_head_gather,
    sp_head_slice,
)
from oracle.partition import balanced_ranges
from ulysses_sequence_attention_sp_b200.synth import make_bits

SHAPES = [  # (batch, tokens, heads, head_dim, world, prefix)
    (1, 37, 6, 16, 4, 0),
    (2, 11, 5, 3, 3, 0),
    (3, 9, 4, 5, 4, 1),
    (1, 5, 7, 2, 5, 1),
    (2, 8, 3, 4, 1, 0),
    (2, 8, 3, 4, 1, 1),
]


def _bits_equal(a, b):
    return a.dtype == b.dtype and a.shape == b.shape and np.array_equal(a.view(np.uint8), b.view(np.uint8))


def _owner(ranges, index):
    for r, (a, b) in enumerate(ranges):
        if a <= index < b:
            return r
    raise AssertionError(index)


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("itemsize", [2, 4])
def test_scatter_gather_roundtrip_bits(shape, itemsize):
    batch, tokens, heads, dim, world, prefix = shape
    x = make_bits((batch, prefix + tokens, heads, dim), itemsize, seed=2001)
    tr = balanced_ranges(tokens, world)
    shards = scatter_sequence(x, tr, prefix=prefix)
    assert _bits_equal(gather_sequence(shards, tr, prefix=prefix), x)
    # brute force: shard r row j is full row prefix + t0 + j, cls rows replicated
    for r, (t0, t1) in enumerate(tr):
        assert shards[r].shape == (batch, prefix + t1 - t0, heads, dim)
        for j in range(prefix + t1 - t0):
            src = j if j < prefix else prefix + t0 + (j - prefix)
            assert _bits_equal(shards[r][:, j], x[:, src])


@pytest.mark.parametrize("shape", SHAPES)
def test_seq_to_head_elementwise(shape):
    batch, tokens, heads, dim, world, prefix = shape
    x = make_bits((batch, prefix + tokens, heads, dim), 2, seed=2002)
    tr = balanced_ranges(tokens, world)
    hr = balanced_ranges(heads, world) if heads >= world else None
    if hr is None:
        pytest.skip("fewer heads than ranks")
    seq = scatter_sequence(x, tr, prefix=prefix)
    out = seq_to_head(seq, tr, hr, prefix=prefix)
    for r, (h0, h1) in enumerate(hr):
        assert out[r].shape == (batch, prefix + tokens, h1 - h0, dim)
        for b, t, h in itertools.product(range(batch), range(prefix + tokens), range(h1 - h0)):
            if t < prefix:
                expect = seq[0][b, t, h0 + h]
            else:
                i = _owner(tr, t - prefix)
                expect = seq[i][b, prefix + (t - prefix) - tr[i][0], h0 + h]
            assert _bits_equal(out[r][b, t, h], expect)


@pytest.mark.parametrize("shape", SHAPES)
def test_head_to_seq_elementwise(shape):
    batch, tokens, heads, dim, world, prefix = shape
    if heads < world:
        pytest.skip("fewer heads than ranks")
    tr = balanced_ranges(tokens, world)
    hr = balanced_ranges(heads, world)
    head_shards = [make_bits((batch, prefix + tokens, h1 - h0, dim), 4, seed=2003 + r)
                   for r, (h0, h1) in enumerate(hr)]
    out = head_to_seq(head_shards, tr, hr, prefix=prefix)
    for i, (t0, t1) in enumerate(tr):
        assert out[i].shape == (batch, prefix + t1 - t0, heads, dim)
        for b, t, h in itertools.product(range(batch), range(prefix + t1 - t0), range(heads)):
            r = _owner(hr, h)
            src_t = t if t < prefix else prefix + t0 + (t - prefix)
            assert _bits_equal(out[i][b, t, h], head_shards[r][b, src_t, h - hr[r][0]])


@pytest.mark.parametrize("shape", SHAPES)
def test_exchange_invariants(shape):
    batch, tokens, heads, dim, world, prefix = shape
    if heads < world:
        pytest.skip("fewer heads than ranks")
    x = make_bits((batch, prefix + tokens, heads, dim), 2, seed=2004)
    tr = balanced_ranges(tokens, world)
    hr = balanced_ranges(heads, world)
    seq = scatter_sequence(x, tr, prefix=prefix)
    heads_view = seq_to_head(seq, tr, hr, prefix=prefix)
    # head_to_seq(seq_to_head(x)) == x
    back = head_to_seq(heads_view, tr, hr, prefix=prefix)
    assert all(_bits_equal(a, b) for a, b in zip(back, seq))
    # the head group the exchange routes to rank r is the head slice of the full tensor
    sliced = sp_head_slice(x, hr)
    assert all(_bits_equal(a, b) for a, b in zip(heads_view, sliced))
    # sp_head_gather(sp_head_slice(x)) == x
    assert _bits_equal(sp_head_gather(sliced), x)


def test_world_one_is_identity():
    x = make_bits((2, 1 + 9, 4, 6), 2, seed=2005)
    tr, hr = balanced_ranges(9, 1), balanced_ranges(4, 1)
    for prefix in (0, 1):
        xs = x if prefix else x[:, 1:]
        xs = np.ascontiguousarray(xs)
        t = xs.shape[1] - prefix
        tr = balanced_ranges(t, 1)
        (s,) = scatter_sequence(xs, tr, prefix=prefix)
        assert _bits_equal(s, xs)
        (hd,) = seq_to_head([xs], tr, hr, prefix=prefix)
        assert _bits_equal(hd, xs)
        (sq,) = head_to_seq([xs], tr, hr, prefix=prefix)
        assert _bits_equal(sq, xs)
        assert _bits_equal(gather_sequence([xs], tr, prefix=prefix), xs)
        (hs,) = sp_head_slice(xs, hr)
        assert _bits_equal(hs, xs)


def test_mismatched_prefix_replicas_rejected():
    x = make_bits((1, 1 + 8, 4, 2), 2, seed=2006)
    tr, hr = balanced_ranges(8, 2), balanced_ranges(4, 2)
    seq = scatter_sequence(x, tr, prefix=1)
    seq[1][0, 0, 0, 0] ^= np.uint16(1)
    with pytest.raises(ValueError):
        seq_to_head(seq, tr, hr, prefix=1)


def test_generic_token_axis_scatter():
    # the API page's scatter/gather take a token axis; a [T, hidden] residual stream
    x = make_bits((37, 12), 4, seed=2007)
    tr = balanced_ranges(37, 4)
    shards = scatter_sequence(x, tr, axis=0)
    assert [s.shape[0] for s in shards] == [10, 9, 9, 9]
    assert _bits_equal(gather_sequence(shards, tr, axis=0), x)

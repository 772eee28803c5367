"""Pins for oracle.ring: library routines (SDPA, logsumexp), the exactness of
the log-sum-exp merge, brute-force equality with full attention, and the two
degenerate hybrids (one ring rank = plain Ulysses, one Ulysses rank = pure ring)."""

import math

import numpy as np
import pytest
import torch

from oracle.attention import attention_bshd, ulysses_attention
from oracle.layout import scatter_sequence
from oracle.partition import balanced_ranges
from oracle.ring import block_attention, merge_partials, ring_groups, ulysses_ring_attention


def _rand(shape, seed, std=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * std


def test_block_attention_matches_sdpa_and_logsumexp():
    q, k, v = _rand((9, 16), 1), _rand((23, 16), 2), _rand((23, 16), 3)
    o, lse = block_attention(q, k, v, 0.3)
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq[None], tk[None], tv[None], scale=0.3)[0].numpy()
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, torch.logsumexp(tq @ tk.T * 0.3, dim=1).numpy(), rtol=1e-13)


def test_single_key_block():
    q, k, v = _rand((4, 8), 4), _rand((1, 8), 5), _rand((1, 8), 6)
    o, lse = block_attention(q, k, v, 0.5)
    np.testing.assert_array_equal(o, np.repeat(v, 4, axis=0))
    np.testing.assert_allclose(lse, (q @ k.T)[:, 0] * 0.5, rtol=1e-15)


@pytest.mark.parametrize("split", [1, 7, 15, 29])
def test_merge_of_two_blocks_is_the_whole(split):
    q, k, v = _rand((6, 8), 7, 2.0), _rand((30, 8), 8, 2.0), _rand((30, 8), 9)
    whole = block_attention(q, k, v, 0.7)
    a = block_attention(q, k[:split], v[:split], 0.7)
    b = block_attention(q, k[split:], v[split:], 0.7)
    for merged in (merge_partials(*a, *b), merge_partials(*b, *a)):
        np.testing.assert_allclose(merged[0], whole[0], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(merged[1], whole[1], rtol=1e-13)


def test_merge_closed_form_two_keys():
    # one key per block: the merge is the two-key softmax, w0 = 1 / (1 + e^(b - a))
    q = np.array([[0.4, -1.0]])
    k = np.array([[1.0, 0.5], [-0.3, 0.2]])
    v = np.array([[2.0, -1.0], [0.5, 4.0]])
    a, b = (q @ k.T)[0]
    o, lse = merge_partials(*block_attention(q, k[:1], v[:1], 1.0), *block_attention(q, k[1:], v[1:], 1.0))
    w0 = 1.0 / (1.0 + math.exp(b - a))
    np.testing.assert_allclose(o[0], w0 * v[0] + (1 - w0) * v[1], rtol=1e-14)
    np.testing.assert_allclose(lse[0], math.log(math.exp(a) + math.exp(b)), rtol=1e-14)


def test_merge_is_associative():
    q, k, v = _rand((5, 8), 10), _rand((33, 8), 11), _rand((33, 8), 12)
    parts = [block_attention(q, k[a:b], v[a:b], 0.4) for a, b in ((0, 10), (10, 11), (11, 33))]
    left = merge_partials(*merge_partials(*parts[0], *parts[1]), *parts[2])
    right = merge_partials(*parts[0], *merge_partials(*parts[1], *parts[2]))
    np.testing.assert_allclose(left[0], right[0], rtol=1e-12, atol=1e-14)


def test_ring_groups():
    tr = balanced_ranges(10, 6)  # 2,2,2,2,1,1
    groups = ring_groups(tr, 2, 3)
    assert [m for m, _, _ in groups] == [[0, 1], [2, 3], [4, 5]]
    assert [blk for _, blk, _ in groups] == [(0, 4), (4, 8), (8, 10)]
    assert [loc for _, _, loc in groups] == [((0, 2), (2, 4)), ((0, 2), (2, 4)), ((0, 1), (1, 2))]
    with pytest.raises(ValueError):
        ring_groups(tr, 4, 2)


CASES = [  # batch, tokens, Hq, Hkv, dim, ulysses, ring, prefix
    (1, 37, 4, 4, 8, 2, 2, 0),
    (2, 23, 6, 6, 8, 3, 2, 1),
    (1, 29, 4, 4, 4, 1, 4, 0),   # pure ring
    (1, 19, 6, 6, 8, 3, 1, 0),   # one ring rank
    (2, 31, 8, 4, 8, 2, 3, 1),   # grouped-query attention
    (1, 50, 5, 5, 8, 2, 5, 0),   # ragged heads and tokens
]


@pytest.mark.parametrize("case", CASES)
def test_hybrid_equals_full_attention(case):
    batch, tokens, hq, hkv, dim, pu, pr, prefix = case
    tr = balanced_ranges(tokens, pu * pr)
    q = _rand((batch, prefix + tokens, hq, dim), 21)
    k, v = _rand((batch, prefix + tokens, hkv, dim), 22), _rand((batch, prefix + tokens, hkv, dim), 23)
    qs, ks, vs = (scatter_sequence(x, tr, prefix=prefix) for x in (q, k, v))
    ref = scatter_sequence(attention_bshd(q, k, v), tr, prefix=prefix)
    for n in (1, 2, 3):
        out = ulysses_ring_attention(qs, ks, vs, tr, pu, pr, num_chunks=n, prefix=prefix)
        for a, b in zip(out, ref):
            np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_one_ring_rank_is_plain_ulysses():
    batch, tokens, heads, dim, world = 2, 27, 6, 8, 3
    tr, hr = balanced_ranges(tokens, world), balanced_ranges(heads, world)
    qs, ks, vs = (scatter_sequence(_rand((batch, tokens, heads, dim), s), tr) for s in (31, 32, 33))
    plain = ulysses_attention(qs, ks, vs, tr, hr)
    hybrid = ulysses_ring_attention(qs, ks, vs, tr, world, 1)
    for a, b in zip(plain, hybrid):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-14)


def test_cls_key_is_counted_once():
    """With a cls row, every group sees the cls query but the cls key only in
    block 0: the result equals attention over the 1 + T tokens, which a
    per-step cls key (counted ring_size times) would not give."""
    batch, tokens, heads, dim, pu, pr = 1, 12, 2, 4, 2, 3
    tr = balanced_ranges(tokens, pu * pr)
    q, k, v = (_rand((batch, 1 + tokens, heads, dim), s, 2.0) for s in (41, 42, 43))
    k[:, 0] *= 3.0  # a dominant cls key makes a double count visible
    qs, ks, vs = (scatter_sequence(x, tr, prefix=1) for x in (q, k, v))
    out = ulysses_ring_attention(qs, ks, vs, tr, pu, pr, prefix=1)
    ref = scatter_sequence(attention_bshd(q, k, v), tr, prefix=1)
    for a, b in zip(out, ref):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)

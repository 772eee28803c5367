"""Pins for oracle.attention: a library routine, closed forms, invariants, brute force."""

import math

import numpy as np
import pytest
import torch

from oracle.attention import (
    attention_bshd,
    attention_rows,
    default_scale,
    softmax_attention,
    ulysses_attention,
)
from oracle.layout import gather_sequence, scatter_sequence
from oracle.partition import balanced_ranges


def _rand(shape, seed, std=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * std


@pytest.mark.parametrize("tq,tk,d", [(1, 1, 4), (5, 7, 16), (37, 37, 16), (600, 530, 8), (3, 1100, 80)])
def test_matches_torch_sdpa_float64(tq, tk, d):
    q, k, v = _rand((tq, d), 1), _rand((tk, d), 2), _rand((tk, d), 3)
    scale = 1.0 / math.sqrt(d)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(k)[None, None],
        torch.from_numpy(v)[None, None], scale=scale)[0, 0].numpy()
    np.testing.assert_allclose(softmax_attention(q, k, v, scale), ref, rtol=1e-12, atol=1e-13)


def test_other_scale_matches_sdpa():
    q, k, v = _rand((9, 16), 4), _rand((13, 16), 5), _rand((13, 16), 6)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None],
        scale=0.37)[0].numpy()
    np.testing.assert_allclose(softmax_attention(q, k, v, 0.37), ref, rtol=1e-12, atol=1e-13)


def test_two_keys_closed_form():
    q = np.array([[0.3, -1.2, 0.5, 2.0]])
    k = np.array([[1.0, 0.0, -1.0, 0.5], [0.2, 0.4, 0.1, -0.3]])
    v = np.array([[1.0, 2.0, 3.0, 4.0], [-1.0, 0.5, 0.0, 10.0]])
    s = 0.5
    a, b = (q @ k.T)[0] * s
    w0 = 1.0 / (1.0 + math.exp(b - a))
    expect = w0 * v[0] + (1.0 - w0) * v[1]
    np.testing.assert_allclose(softmax_attention(q, k, v, s)[0], expect, rtol=1e-14)


def test_single_key_returns_v():
    q, k, v = _rand((6, 8), 7), _rand((1, 8), 8), _rand((1, 8), 9)
    np.testing.assert_array_equal(softmax_attention(q, k, v, 0.3), np.repeat(v, 6, axis=0))


def test_uniform_scores_give_mean_of_v():
    k, v = _rand((50, 16), 10), _rand((50, 16), 11)
    out = softmax_attention(np.zeros((3, 16)), k, v, 0.25)
    np.testing.assert_allclose(out, np.repeat(v.mean(axis=0, keepdims=True), 3, axis=0), rtol=1e-13)
    kk = np.repeat(_rand((1, 16), 12), 50, axis=0)
    out = softmax_attention(_rand((4, 16), 13), kk, v, 0.25)
    np.testing.assert_allclose(out, np.repeat(v.mean(axis=0, keepdims=True), 4, axis=0), rtol=1e-12)


def test_convex_combination_bounds_and_permutation():
    q, k, v = _rand((40, 16), 14, 3.0), _rand((70, 16), 15, 3.0), _rand((70, 16), 16)
    out = softmax_attention(q, k, v, 0.25)
    assert np.all(out <= v.max(axis=0) + 1e-12) and np.all(out >= v.min(axis=0) - 1e-12)
    perm = np.random.default_rng(17).permutation(70)
    np.testing.assert_allclose(softmax_attention(q, k[perm], v[perm], 0.25), out, rtol=1e-12, atol=1e-14)


def test_large_scores_stay_finite():
    q, k, v = _rand((4, 8), 18, 40.0), _rand((20, 8), 19, 40.0), _rand((20, 8), 20)
    out = softmax_attention(q, k, v, 1.0)
    assert np.all(np.isfinite(out))


def test_rows_match_full():
    q, k, v = (_rand((2, 30, 3, 8), s) for s in (21, 22, 23))
    full = attention_bshd(q, k, v)
    rows = [0, 7, 29]
    np.testing.assert_array_equal(attention_rows(q, k, v, 1, 2, rows), full[1, rows, 2])


CASES = [  # (batch, tokens, heads, dim, world, prefix)
    (1, 37, 6, 16, 4, 0),
    (2, 23, 5, 8, 3, 0),
    (3, 16, 4, 10, 4, 1),
    (1, 9, 3, 4, 1, 0),
]


@pytest.mark.parametrize("case", CASES)
def test_ulysses_equals_full_attention(case):
    """The sharded block equals single-device attention on the gathered tensors."""
    batch, tokens, heads, dim, world, prefix = case
    tr, hr = balanced_ranges(tokens, world), balanced_ranges(heads, world)
    q, k, v = (_rand((batch, prefix + tokens, heads, dim), s) for s in (31, 32, 33))
    qs, ks, vs = (scatter_sequence(x, tr, prefix=prefix) for x in (q, k, v))
    out = ulysses_attention(qs, ks, vs, tr, hr, prefix=prefix)
    brute = scatter_sequence(attention_bshd(q, k, v), tr, prefix=prefix)
    for a, b in zip(out, brute):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
    assert np.array_equal(gather_sequence(out, tr, prefix=prefix).shape, q.shape)


@pytest.mark.parametrize("case", CASES)
def test_chunk_counts_bit_identical(case):
    batch, tokens, heads, dim, world, prefix = case
    tr, hr = balanced_ranges(tokens, world), balanced_ranges(heads, world)
    q, k, v = (_rand((batch, prefix + tokens, heads, dim), s) for s in (41, 42, 43))
    qs, ks, vs = (scatter_sequence(x, tr, prefix=prefix) for x in (q, k, v))
    g = max(b - a for a, b in hr)
    ref = ulysses_attention(qs, ks, vs, tr, hr, prefix=prefix, num_chunks=1)
    for n in sorted({2, 3, g, g + 3}):
        out = ulysses_attention(qs, ks, vs, tr, hr, prefix=prefix, num_chunks=n)
        for a, b in zip(out, ref):
            assert np.array_equal(a, b)


def test_cls_prefix_matches_gather_compute_scatter():
    """The ViT wrapper's form: all-gather patches, prepend the replicated cls,
    full non-causal attention, keep this rank's patch slice and re-prepend cls."""
    batch, patches, heads, dim, world = 2, 12, 4, 8, 4
    tr, hr = balanced_ranges(patches, world), balanced_ranges(heads, world)
    q, k, v = (_rand((batch, 1 + patches, heads, dim), s, 0.5) for s in (51, 52, 53))
    qs, ks, vs = (scatter_sequence(x, tr, prefix=1) for x in (q, k, v))
    out = ulysses_attention(qs, ks, vs, tr, hr, prefix=1)
    for r, (t0, t1) in enumerate(tr):
        full_q = np.concatenate([qs[r][:, :1]] + [s[:, 1:] for s in qs], axis=1)
        full_k = np.concatenate([ks[r][:, :1]] + [s[:, 1:] for s in ks], axis=1)
        full_v = np.concatenate([vs[r][:, :1]] + [s[:, 1:] for s in vs], axis=1)
        full_out = attention_bshd(full_q, full_k, full_v)
        local = np.concatenate([full_out[:, :1], full_out[:, 1 + t0:1 + t1]], axis=1)
        np.testing.assert_allclose(out[r], local, rtol=0, atol=1e-12)


def test_default_scale():
    assert default_scale(128) == 1.0 / math.sqrt(128)
    q, k, v = (_rand((1, 7, 2, 16), s) for s in (61, 62, 63))
    np.testing.assert_array_equal(attention_bshd(q, k, v), attention_bshd(q, k, v, scale=0.25))


# ---------------------------------------------------------------- grouped-query attention
def test_gqa_matches_torch_sdpa_float64():
    q, k, v = _rand((1, 37, 6, 16), 71), _rand((1, 37, 2, 16), 72), _rand((1, 37, 2, 16), 73)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q).permute(0, 2, 1, 3), torch.from_numpy(k).permute(0, 2, 1, 3),
        torch.from_numpy(v).permute(0, 2, 1, 3), enable_gqa=True).permute(0, 2, 1, 3).numpy()
    np.testing.assert_allclose(attention_bshd(q, k, v), ref, rtol=1e-12, atol=1e-13)


def test_gqa_equals_mha_with_repeated_kv_heads():
    q, k, v = _rand((2, 21, 8, 8), 74), _rand((2, 21, 2, 8), 75), _rand((2, 21, 2, 8), 76)
    mha = attention_bshd(q, np.repeat(k, 4, axis=2), np.repeat(v, 4, axis=2))
    np.testing.assert_array_equal(attention_bshd(q, k, v), mha)


@pytest.mark.parametrize("case", [(1, 37, 8, 4, 16, 4, 0), (2, 23, 12, 4, 8, 2, 1), (1, 19, 6, 6, 8, 3, 0),
                                  (3, 16, 16, 8, 8, 4, 1)])
def test_ulysses_gqa_equals_full_attention(case):
    batch, tokens, hq, hkv, dim, world, prefix = case
    tr, hr, kr = balanced_ranges(tokens, world), balanced_ranges(hq, world), balanced_ranges(hkv, world)
    q = _rand((batch, prefix + tokens, hq, dim), 81)
    k, v = _rand((batch, prefix + tokens, hkv, dim), 82), _rand((batch, prefix + tokens, hkv, dim), 83)
    qs, ks, vs = (scatter_sequence(x, tr, prefix=prefix) for x in (q, k, v))
    ref = scatter_sequence(attention_bshd(q, k, v), tr, prefix=prefix)
    for n in (1, 2, 5):
        out = ulysses_attention(qs, ks, vs, tr, hr, kv_head_ranges=kr, prefix=prefix, num_chunks=n)
        for a, b in zip(out, ref):
            np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_gqa_split_that_breaks_groups_is_rejected():
    # 6 query heads over 4 ranks -> 2,2,1,1; 3 kv heads -> 1,1,1,0 is impossible
    # (fewer kv heads than ranks); 12 q / 4 kv over 3 ranks -> q 4,4,4 with kv 2,1,1:
    # rank 0's query heads 0..3 use kv heads 0,1 (owned), rank 1's 4..7 use 2,3 but owns only 2.
    tr, hr, kr = balanced_ranges(9, 3), balanced_ranges(12, 3), balanced_ranges(4, 3)
    x = [np.zeros((1, 3, 4, 2))] * 3
    kv = [np.zeros((1, 3, b - a, 2)) for a, b in kr]
    with pytest.raises(ValueError):
        ulysses_attention(x, kv, kv, tr, hr, kv_head_ranges=kr)

"""Plant plausible mistakes in copies of oracle functions (on the CPU) and check
that the pins used above reject each one. This shows the pins can fail."""

import json
import math
import os

import numpy as np
import torch

from oracle.layout import _take, scatter_sequence, seq_to_head
from oracle.partition import balanced_ranges, range_lengths


def _golden_partition_ok(fn, golden_dir):
    with open(os.path.join(golden_dir, "balanced_ranges.json")) as f:
        golden = json.load(f)
    for case in golden["cases"]:
        r = fn(case["total"], case["parts"])
        if "ranges" in case and [list(x) for x in r] != case["ranges"]:
            return False
        if "lengths" in case and list(range_lengths(r)) != case["lengths"]:
            return False
    return True


def test_remainder_on_last_ranks_is_caught(golden_dir):
    def wrong(total, parts):
        base, extra = divmod(total, parts)
        lengths = [base + (r >= parts - extra) for r in range(parts)]
        out, s = [], 0
        for n in lengths:
            out.append((s, s + n))
            s += n
        return tuple(out)

    assert _golden_partition_ok(balanced_ranges, golden_dir)
    assert not _golden_partition_ok(wrong, golden_dir)


def test_floor_chunks_are_caught(golden_dir):
    def wrong(g, n):
        s = g // n
        chunks = [(c * s, (c + 1) * s) for c in range(n - 1)]
        return chunks + [((n - 1) * s, g)]

    with open(os.path.join(golden_dir, "head_chunks.json")) as f:
        case = json.load(f)["cases"][0]
    sizes = [hi - lo for lo, hi in wrong(case["group_heads"], case["num_chunks"])]
    assert sizes != case["sizes"]


def test_reversed_source_order_is_caught():
    def wrong_seq_to_head(seq_shards, token_ranges, head_ranges, prefix=0):
        out = []
        for (h0, h1) in head_ranges:
            parts = [_take(_take(s, 1, prefix, None), 2, h0, h1) for s in reversed(seq_shards)]
            out.append(np.concatenate(parts, axis=1))
        return out

    x = np.arange(1 * 10 * 4 * 2, dtype=np.uint32).reshape(1, 10, 4, 2)
    tr, hr = balanced_ranges(10, 3), balanced_ranges(4, 3)
    seq = scatter_sequence(x, tr)
    good = seq_to_head(seq, tr, hr)
    bad = wrong_seq_to_head(seq, tr, hr)
    # the element-wise definition (source rank = owner of the token) holds only for the oracle
    def holds(out):
        for r, (h0, h1) in enumerate(hr):
            if not np.array_equal(out[r], x[:, :, h0:h1]):
                return False
        return True
    assert holds(good) and not holds(bad)


def _sdpa_ok(fn):
    rng = np.random.default_rng(3)
    q, k, v = rng.standard_normal((7, 16)), rng.standard_normal((9, 16)), rng.standard_normal((9, 16))
    scale = 1.0 / math.sqrt(16)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None], scale=scale)[0].numpy()
    return np.allclose(fn(q, k, v, scale), ref, rtol=1e-12, atol=1e-13)


def test_attention_mistakes_are_caught():
    from oracle.attention import softmax_attention

    def no_scale(q, k, v, scale):
        s = q @ k.T
        p = np.exp(s - s.max(axis=1, keepdims=True))
        return (p @ v) / p.sum(axis=1, keepdims=True)

    def wrong_axis(q, k, v, scale):
        s = (q @ k.T) * scale
        p = np.exp(s - s.max(axis=0, keepdims=True))
        return (p @ v) / p.sum(axis=0)[:, None][: q.shape[0]]

    def transposed_v(q, k, v, scale):
        s = (q @ k.T) * scale
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p = p / p.sum(axis=1, keepdims=True)
        return p @ v[::-1]

    assert _sdpa_ok(softmax_attention)
    for bad in (no_scale, wrong_axis, transposed_v):
        try:
            ok = _sdpa_ok(bad)
        except ValueError:
            ok = False
        assert not ok, bad.__name__


def test_row_collective_mistakes_are_caught():
    """A reduce-scatter that forgets the destination's row offset (reads rows
    0..T_r of every partial for every destination), or an all-gather that drops the zero-padding
    strip (keeps max_rows per rank), fails the adjointness pin or the shape."""
    from oracle.rows import all_gather_rows, reduce_scatter_rows

    tr = balanced_ranges(10, 4)
    rng = np.random.default_rng(3)
    x = [rng.standard_normal((1, 10, 2)) for _ in range(4)]
    y = [rng.standard_normal((1, b - a, 2)) for a, b in tr]

    def wrong_rs(partials, token_ranges):
        out = []
        for r, (start, stop) in enumerate(token_ranges):
            acc = np.zeros_like(partials[0][:, start:stop])
            for p in partials:
                acc = acc + p[:, 0:stop - start]  # mistake: destination offset dropped
            out.append(acc)
        return out

    def adjoint_gap(rs, ag):
        lhs = sum(float(np.sum(a * b)) for a, b in zip(rs(x, tr), y))
        rhs = sum(float(np.sum(a * b)) for a, b in zip(x, ag(y, tr)))
        return abs(lhs - rhs)

    assert adjoint_gap(reduce_scatter_rows, all_gather_rows) < 1e-10
    assert adjoint_gap(wrong_rs, all_gather_rows) > 1e-3

    def wrong_ag(local, token_ranges):
        m = max(b - a for a, b in token_ranges)
        blocks = []
        for v in local:
            pad = np.zeros((v.shape[0], m, *v.shape[2:]))
            pad[:, : v.shape[1]] = v
            blocks.append(pad)
        full = np.concatenate(blocks, axis=1)  # mistake: padding rows kept
        return [full] * len(local)

    assert wrong_ag(y, tr)[0].shape != all_gather_rows(y, tr)[0].shape


def test_ring_merge_mistakes_are_caught():
    """A merge that averages the partials, or one that weights them by exp(lse)
    without renormalising, fails the two-block pin; a cls key that every ring
    step sees fails the full-attention pin."""
    from oracle.attention import attention_bshd
    from oracle.ring import block_attention, merge_partials

    rng = np.random.default_rng(5)
    q, k, v = rng.standard_normal((6, 8)) * 2, rng.standard_normal((30, 8)) * 2, rng.standard_normal((30, 8))
    whole = block_attention(q, k, v, 0.7)
    a, b = block_attention(q, k[:11], v[:11], 0.7), block_attention(q, k[11:], v[11:], 0.7)

    def averaged(o_a, lse_a, o_b, lse_b):
        return (o_a + o_b) / 2, np.logaddexp(lse_a, lse_b)

    def unnormalised(o_a, lse_a, o_b, lse_b):
        return o_a * np.exp(lse_a)[:, None] + o_b * np.exp(lse_b)[:, None], np.logaddexp(lse_a, lse_b)

    assert np.allclose(merge_partials(*a, *b)[0], whole[0], rtol=1e-12, atol=1e-13)
    for wrong in (averaged, unnormalised):
        assert not np.allclose(wrong(*a, *b)[0], whole[0], rtol=1e-6, atol=1e-6)

    # cls key in every block: attention over [cls, block] per step, merged
    tokens, ring = 12, 3
    x = [rng.standard_normal((1 + tokens, 4)) * 2 for _ in range(3)]
    x[1][0] *= 3.0
    qq, kk, vv = x
    blocks = [(1 + 4 * g, 1 + 4 * (g + 1)) for g in range(ring)]
    o = lse = None
    for s0, s1 in blocks:
        kb = np.concatenate([kk[:1], kk[s0:s1]])
        vb = np.concatenate([vv[:1], vv[s0:s1]])
        part = block_attention(qq, kb, vb, 0.5)
        o, lse = part if o is None else merge_partials(o, lse, *part)
    ref = attention_bshd(qq[None, :, None], kk[None, :, None], vv[None, :, None], scale=0.5)[0, :, 0]
    assert not np.allclose(o, ref, rtol=1e-6, atol=1e-6)

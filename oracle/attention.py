"""Float64 softmax attention and the Ulysses block (oracle; test infrastructure only).

Sources:

* "mstar.model.components.distributed.sequence_parallel",
  ``ulysses_attention``: exchange sequence shards for head shards, run the
  unchanged single-device attention on the full sequence of this rank's
  heads, exchange back. A trivial group is byte-identical to the non-SP path.
* "deepspeed/sequence/autosp_vit.py", module notes: the attention is
  non-causal (every token attends to every token) and the sharded result is
  identical to single-device execution; the cls token is replicated.
* "maxdiffusion PR #428: experimental two-phase (head-chunked) Ulysses
  all-to-all": the head-chunked passes compute the same result as the
  single-shot pass because heads are independent.
* API page, ulysses_attention: q carries Hq heads and k/v carry Hkv heads
  (grouped-query attention); each kv head serves Hq / Hkv query heads.

Readings: the attention is ``softmax(Q K^T * scale) V`` per (batch, head)
with ``scale = 1/sqrt(D)`` unless given, no mask, no dropout; it is computed
in float64 on the exact upcast of the inputs. Batch elements never attend to
each other.
"""

from __future__ import annotations

import math

import numpy as np

from .layout import head_to_seq, seq_to_head
from .partition import check_gqa_ranges, gqa_group, head_chunk_ranges, range_lengths

# Query rows per matmul. Rows are independent, so this only bounds memory.
_ROW_BLOCK = 512


def default_scale(head_dim: int) -> float:
    return 1.0 / math.sqrt(head_dim)


def softmax_attention(q, k, v, scale):
    """``softmax(q k^T * scale) v`` for one head: q ``[Tq, D]``, k/v ``[Tk, D]``.

    The row maximum is subtracted before ``exp`` (this changes nothing
    mathematically and keeps ``exp`` finite).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if k.shape[0] != v.shape[0] or q.shape[1] != k.shape[1]:
        raise ValueError("incompatible q/k/v shapes")
    out = np.empty((q.shape[0], v.shape[1]), dtype=np.float64)
    for r0 in range(0, q.shape[0], _ROW_BLOCK):
        r1 = min(r0 + _ROW_BLOCK, q.shape[0])
        scores = (q[r0:r1] @ k.T) * scale
        scores -= scores.max(axis=1, keepdims=True)
        weights = np.exp(scores)
        out[r0:r1] = (weights @ v) / weights.sum(axis=1, keepdims=True)
    return out


def attention_bshd(q, k, v, scale=None):
    """Attention over ``[B, T, Hs, D]`` head-layout arrays; float64 result.

    k and v may carry fewer heads than q (grouped-query attention, the API
    page's Hkv <= Hq): query head h then uses kv head h // (Hq / Hkv).
    """
    if k.shape != v.shape or q.shape[:2] != k.shape[:2] or q.shape[3] != k.shape[3]:
        raise ValueError("incompatible q/k/v shapes")
    batch, _tokens, heads, head_dim = q.shape
    group = heads // k.shape[2]
    if group * k.shape[2] != heads:
        raise ValueError("query heads must be a multiple of kv heads")
    if scale is None:
        scale = default_scale(head_dim)
    out = np.empty(q.shape, dtype=np.float64)
    for b in range(batch):
        for h in range(heads):
            out[b, :, h, :] = softmax_attention(q[b, :, h, :], k[b, :, h // group, :], v[b, :, h // group, :], scale)
    return out


def attention_rows(q_full, k_full, v_full, b, h, rows, scale=None):
    """Output rows ``rows`` of head ``h``, batch ``b`` of full-sequence BSHD
    arrays; used to check sampled rows of a full-size run one by one."""
    head_dim = q_full.shape[3]
    if scale is None:
        scale = default_scale(head_dim)
    rows = np.asarray(rows, dtype=np.int64)
    return softmax_attention(q_full[b, rows, h, :], k_full[b, :, h, :], v_full[b, :, h, :], scale)


def ulysses_attention(q_shards, k_shards, v_shards, token_ranges, head_ranges, *,
                      kv_head_ranges=None, num_chunks=1, scale=None, prefix=0):
    """The Ulysses block on per-rank sequence shards ``[B, prefix+T_i, H, D]``.

    Returns per-rank sequence shards of the float64 attention output. The
    steps are the block's: seq->head exchange of q, k and v; for each head
    chunk, attention of every rank over its heads of that chunk; head->seq
    exchange of the output. With grouped-query attention k and v carry Hkv
    heads split by ``kv_head_ranges``; query head h uses kv head
    h // (Hq / Hkv), which must be one of its rank's kv heads.
    """
    if kv_head_ranges is None:
        kv_head_ranges = head_ranges
    heads_q = head_ranges[-1][1]
    heads_kv = kv_head_ranges[-1][1]
    group = gqa_group(heads_q, heads_kv)
    check_gqa_ranges(head_ranges, kv_head_ranges, group)
    qh = seq_to_head(q_shards, token_ranges, head_ranges, prefix=prefix)
    kh = seq_to_head(k_shards, token_ranges, kv_head_ranges, prefix=prefix)
    vh = seq_to_head(v_shards, token_ranges, kv_head_ranges, prefix=prefix)
    head_dim = q_shards[0].shape[3]
    if scale is None:
        scale = default_scale(head_dim)
    counts = range_lengths(head_ranges)
    oh = [np.full(x.shape, np.nan, dtype=np.float64) for x in qh]
    for lo, hi in head_chunk_ranges(max(counts), num_chunks):
        for r, count in enumerate(counts):
            h0, k0 = head_ranges[r][0], kv_head_ranges[r][0]
            for i in range(min(lo, count), min(hi, count)):
                kv = (h0 + i) // group - k0   # this rank's local kv head for local query head i
                oh[r][:, :, i:i + 1, :] = attention_bshd(
                    qh[r][:, :, i:i + 1, :], kh[r][:, :, kv:kv + 1, :], vh[r][:, :, kv:kv + 1, :], scale
                )
    return head_to_seq(oh, token_ranges, head_ranges, prefix=prefix)

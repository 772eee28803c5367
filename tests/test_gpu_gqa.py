"""GPU parity of grouped-query attention (k/v with fewer heads than q).

The API page's ulysses_attention takes q with Hq heads and k/v with Hkv heads;
query head h attends with kv head h // (Hq / Hkv). Each virtual rank owns a
contiguous query-head group and the kv heads that group uses, so the k/v
exchange moves Hkv / Hq of the bytes the q exchange moves. The block is
compared element by element with the float64 oracle; the k/v exchange alone
is compared bit for bit."""

import numpy as np
import pytest
import torch

from oracle import attention as oa
from oracle import layout as ol
from tests.gpu_util import assert_close, bits_to_device, device_bits, to_device, to_f64
from ulysses_sequence_attention_sp_b200.synth import make_bits, make_qkv, storage_to_f64
from ulysses_sequence_attention_sp_b200.workloads import Workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def usp():
    from ulysses_sequence_attention_sp_b200 import usp as mod
    assert torch.cuda.is_available()
    mod.device_status(reset=True)
    return mod


GQA = [  # name, batch, seq_len, prefix, Hq, D, world, dtype, std, seed, chunks, Hkv
    Workload("g1", 1, 300, 0, 8, 128, 2, "bf16", 1.0, 31, (1, 2, 3), 2),
    Workload("g2", 2, 200, 1, 12, 80, 4, "bf16", 1.0, 32, (1, 2), 4),
    Workload("g3", 1, 1000, 0, 16, 64, 2, "bf16", 1.0, 33, (1, 3, 8), 4),
    Workload("g4", 1, 129, 0, 8, 128, 1, "bf16", 1.0, 34, (1, 3), 1),   # multi-query
    Workload("g5", 3, 40, 1, 24, 96, 8, "bf16", 1.0, 35, (1, 2), 8),
    Workload("g6", 2, 77, 0, 6, 16, 3, "fp32", 1.0, 36, (1, 2), 3),
    Workload("g7", 1, 260, 0, 8, 128, 2, "bf16", 1.0, 37, (1,), 8),     # Hkv == Hq through the GQA entry
]


def _plan(usp, w):
    return usp.Plan(w.batch, w.seq_len, w.heads, w.head_dim, w.world, w.dtype, w.prefix, kv_heads=w.heads_kv)


def _oracle(w, storage, plan, num_chunks=1):
    q, k, v = (storage_to_f64(x, w.dtype) for x in storage)
    tr = plan.token_ranges
    qs, ks, vs = (ol.scatter_sequence(x, tr, prefix=w.prefix) for x in (q, k, v))
    return oa.ulysses_attention(qs, ks, vs, tr, plan.head_ranges, kv_head_ranges=plan.kv_head_ranges,
                                prefix=w.prefix, num_chunks=num_chunks)


def _run(usp, w, num_chunks):
    storage = make_qkv(w)
    plan = _plan(usp, w)
    shards = [usp.scatter_sequence(plan, to_device(x, w.dtype)) for x in storage]
    out = plan.empty_seq_shards(fill=float("nan"))
    usp.ulysses_attention(plan, *shards, out=out, num_chunks=num_chunks)
    torch.cuda.synchronize()
    assert usp.device_status() == 0
    return storage, plan, out


def test_plan_kv_ranges(usp):
    plan = usp.Plan(1, 64, 12, 64, 4, "bf16", 0, kv_heads=4)
    assert plan.kv_heads == 4
    assert plan.head_ranges == ((0, 3), (3, 6), (6, 9), (9, 12))
    assert plan.kv_head_ranges == ((0, 1), (1, 2), (2, 3), (3, 4))
    plan.close()


@pytest.mark.parametrize("w", GQA, ids=lambda w: w.name)
def test_gqa_block_elementwise(usp, w):
    for n in w.num_chunks:
        storage, plan, out = _run(usp, w, n)
        ref = _oracle(w, storage, plan)
        for r in range(plan.world):
            assert_close(to_f64(out[r], w.dtype), ref[r], w.dtype, f"{w.name} chunks={n} rank={r}")
        plan.close()


@pytest.mark.parametrize("w", GQA[:3], ids=lambda w: w.name)
def test_gqa_chunk_counts_bit_identical(usp, w):
    base = None
    g = max(b - a for a, b in usp.balanced_ranges(w.heads, w.world))
    for n in [1, 2, 3, g, g + 2]:
        _, plan, out = _run(usp, w, n)
        bits = [o.view(torch.int16).cpu() for o in out]
        if base is None:
            base = bits
        else:
            assert all(torch.equal(a, b) for a, b in zip(bits, base)), f"num_chunks={n}"
        plan.close()


def test_gqa_equals_mha_with_repeated_kv(usp):
    """Bit identity with the dense-head block on k/v repeated group times."""
    w = GQA[0]
    storage = make_qkv(w)
    group = w.heads // w.heads_kv
    plan = _plan(usp, w)
    shards = [usp.scatter_sequence(plan, to_device(x, w.dtype)) for x in storage]
    out = usp.ulysses_attention(plan, *shards)
    mha = usp.Plan(w.batch, w.seq_len, w.heads, w.head_dim, w.world, w.dtype, w.prefix)
    rep = [storage[0]] + [np.repeat(x, group, axis=2) for x in storage[1:]]
    mshards = [usp.scatter_sequence(mha, to_device(x, w.dtype)) for x in rep]
    mout = usp.ulysses_attention(mha, *mshards)
    torch.cuda.synchronize()
    for a, b in zip(out, mout):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    plan.close()
    mha.close()


@pytest.mark.parametrize("w", [GQA[0], GQA[1], GQA[5]], ids=lambda w: w.name)
def test_gqa_head_attention(usp, w):
    q, k, v = make_qkv(w)
    plan = _plan(usp, w)
    hr, kr = plan.head_ranges, plan.kv_head_ranges
    qh = [to_device(np.ascontiguousarray(q[:, :, h0:h1]), w.dtype) for h0, h1 in hr]
    kh = [to_device(np.ascontiguousarray(k[:, :, h0:h1]), w.dtype) for h0, h1 in kr]
    vh = [to_device(np.ascontiguousarray(v[:, :, h0:h1]), w.dtype) for h0, h1 in kr]
    out = plan.empty_head_shards(fill=float("nan"))
    usp.head_attention(plan, qh, kh, vh, out=out)
    torch.cuda.synchronize()
    qf, kf, vf = (storage_to_f64(x, w.dtype) for x in (q, k, v))
    for r, ((h0, h1), (k0, k1)) in enumerate(zip(hr, kr)):
        ref = oa.attention_bshd(qf[:, :, h0:h1], kf[:, :, k0:k1], vf[:, :, k0:k1])
        assert_close(to_f64(out[r], w.dtype), ref, w.dtype, f"{w.name} rank {r}")
    plan.close()


@pytest.mark.parametrize("w", [GQA[1], GQA[4], GQA[5]], ids=lambda w: w.name)
def test_seq_to_head_kv_bit_exact(usp, w):
    plan = _plan(usp, w)
    itemsize = 2 if w.dtype == "bf16" else 4
    shape = (w.batch, w.tokens, w.heads_kv, w.head_dim)
    full = [make_bits(shape, itemsize, 500 + i) for i in range(2)]
    tr, kr = plan.token_ranges, plan.kv_head_ranges
    seq = [[bits_to_device(s) for s in ol.scatter_sequence(x, tr, prefix=w.prefix)] for x in full]
    seq = [[t.view(plan.torch_dtype) for t in group] for group in seq]
    out = usp.ulysses_seq_to_head(plan, seq, kv=True)
    torch.cuda.synchronize()
    for x, got in zip(full, out):
        ref = ol.seq_to_head(ol.scatter_sequence(x, tr, prefix=w.prefix), tr, kr, prefix=w.prefix)
        for r in range(plan.world):
            assert np.array_equal(device_bits(got[r]), ref[r]), f"{w.name} rank {r}"
    plan.close()


def test_gqa_rejects_q_shaped_kv(usp):
    w = GQA[0]
    plan = _plan(usp, w)
    q = plan.empty_seq_shards(fill=0.0)
    with pytest.raises(usp.UspError):
        usp.ulysses_attention(plan, q, q, q)
    plan.close()

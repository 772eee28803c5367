"""GPU parity of the two-query-tile attention kernel (attn_pp.cu).

The automatic choice takes it only above 16 key tiles of 256 (the full-size
workloads, checked in test_gpu_attention.py and test_gpu_ring.py); here the
plan forces it on small shapes that reach every ragged case: a last key tile
of a few keys, a query-tile pair whose second tile is partly or wholly
beyond the sequence, fewer tokens than one tile, every head_dim it is built
for, grouped-query heads, a cls prefix, batch > 1, fp16, the Ulysses + Ring
key-block walk, and scores spread wide enough that the O rescale runs. Each is
compared with the float64 oracle element by element, and with the one-tile
kernel."""

import numpy as np
import pytest
import torch

from oracle import attention as oa
from oracle import layout as ol
from oracle import ring as oring
from tests.gpu_util import assert_close, to_device, to_f64
from ulysses_sequence_attention_sp_b200.synth import bf16_bits_to_f32, f32_to_bf16_bits, make_qkv, storage_to_f64
from ulysses_sequence_attention_sp_b200.workloads import Workload

pytestmark = pytest.mark.gpu

CASES = [
    Workload("tt-bf16-T1000-H6-D128-P3", 1, 1000, 0, 6, 128, 3, "bf16", 1.0, 9501, (1, 2)),
    Workload("tt-bf16-B2-T300-cls-H5-D80-P2", 2, 300, 1, 5, 80, 2, "bf16", 0.5, 9502, (1, 3)),
    Workload("tt-bf16-T777-H8-KV4-D64-P4", 1, 777, 0, 8, 64, 4, "bf16", 1.0, 9503, (1, 2), kv_heads=4),
    Workload("tt-fp16-T513-H4-D96-P4", 1, 513, 0, 4, 96, 4, "fp16", 1.0, 9504, (1,)),
    Workload("tt-bf16-T129-H2-D112-P2", 1, 129, 0, 2, 112, 2, "bf16", 1.0, 9505, (1, 2)),
    Workload("tt-bf16-T50-H3-D128-P3", 1, 50, 0, 3, 128, 3, "bf16", 1.0, 9506, (1,)),
    Workload("tt-bf16-T256-cls-H4-D64-P4", 1, 256, 1, 4, 64, 4, "bf16", 1.0, 9507, (1,)),
    Workload("tt-bf16-spread-T900-H4-D128-P2", 1, 900, 0, 4, 128, 2, "bf16", 1.0, 9508, (1,)),
]
RING_CASES = [
    (Workload("tt-ring-bf16-T1000-H4-D128-U2xR2", 1, 1000, 0, 4, 128, 4, "bf16", 1.0, 9511, (1, 2)), 2),
    (Workload("tt-ring-bf16-T700-cls-H6-D80-U3xR2", 1, 700, 1, 6, 80, 6, "bf16", 1.0, 9512, (1,)), 2),
    (Workload("tt-ring-bf16-T999-H8-KV4-D64-U2xR2", 1, 999, 0, 8, 64, 4, "bf16", 1.0, 9513, (1,), 4), 2),
]


@pytest.fixture(scope="module")
def usp():
    from ulysses_sequence_attention_sp_b200 import usp as mod
    assert torch.cuda.is_available()
    mod.device_status(reset=True)
    return mod


def _storage(w):
    if w.dtype == "fp16":
        rng = np.random.default_rng(w.seed)
        shape = (w.batch, w.tokens, w.heads, w.head_dim)
        kv = (w.batch, w.tokens, w.heads_kv, w.head_dim)
        return tuple(rng.standard_normal(s, dtype=np.float32).astype(np.float16) for s in (shape, kv, kv))
    q, k, v = make_qkv(w)
    if "spread" in w.name:
        # scores spread wide enough that row maxima keep growing across key tiles
        q = f32_to_bf16_bits(bf16_bits_to_f32(q) * np.float32(4.0))
        k = f32_to_bf16_bits(bf16_bits_to_f32(k) * np.float32(4.0))
    return q, k, v


def _dev(x, w):
    return torch.from_numpy(x).cuda() if w.dtype == "fp16" else to_device(x, w.dtype)


def _f64(x, w):
    return x.astype(np.float64) if w.dtype == "fp16" else storage_to_f64(x, w.dtype)


def _out64(t, w):
    return t.double().cpu().numpy() if w.dtype == "fp16" else to_f64(t, w.dtype)


def _run(usp, w, kernel, num_chunks, ring=1, lse=None, ctas=0):
    plan = usp.Plan(w.batch, w.seq_len, w.heads, w.head_dim, w.world, w.dtype, w.prefix, kv_heads=w.heads_kv,
                    ring_size=ring)
    plan.set_attention_kernel(kernel)
    plan.set_attention_ctas(ctas)
    storage = _storage(w)
    shards = [usp.scatter_sequence(plan, _dev(x, w)) for x in storage]
    out = plan.empty_seq_shards(fill=float("nan"))
    usp.ulysses_attention(plan, *shards, out=out, num_chunks=num_chunks, lse=lse)
    torch.cuda.synchronize()
    assert usp.device_status() == 0
    return storage, plan, out


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_two_tile_matches_oracle(usp, w):
    for n in w.num_chunks:
        storage, plan, out = _run(usp, w, "two_tile", n)
        f64 = [_f64(x, w) for x in storage]
        sh = [ol.scatter_sequence(x, plan.token_ranges, prefix=w.prefix) for x in f64]
        ref = oa.ulysses_attention(*sh, plan.token_ranges, plan.head_ranges, kv_head_ranges=plan.kv_head_ranges,
                                   prefix=w.prefix)
        for r in range(plan.world):
            assert_close(_out64(out[r], w), ref[r], "bf16", f"{w.name} chunks={n} rank={r}")
        plan.close()


@pytest.mark.parametrize("w", CASES[:3], ids=lambda w: w.name)
def test_two_tile_agrees_with_one_tile(usp, w):
    _, p2, o2 = _run(usp, w, "two_tile", 1)
    _, p1, o1 = _run(usp, w, "one_tile", 1)
    for r in range(p2.world):
        assert_close(_out64(o2[r], w), _out64(o1[r], w), "bf16", f"rank {r}")
    p1.close()
    p2.close()


@pytest.mark.parametrize("w", [CASES[0], CASES[2]], ids=lambda w: w.name)
def test_two_tile_chunk_counts_bit_identical(usp, w):
    base = None
    g = max(b - a for a, b in usp.balanced_ranges(w.heads, w.world))
    for n in [1, 2, 3, g, g + 2]:
        _, plan, out = _run(usp, w, "two_tile", n)
        bits = [o.view(torch.int16).cpu() for o in out]
        if base is None:
            base = bits
        else:
            assert all(torch.equal(a, b) for a, b in zip(bits, base)), f"num_chunks={n}"
        plan.close()


@pytest.mark.parametrize("case", RING_CASES, ids=lambda c: c[0].name)
def test_two_tile_ring_matches_oracle(usp, case):
    w, ring = case
    for n in w.num_chunks:
        storage, plan, out = _run(usp, w, "two_tile", n, ring=ring)
        tr = plan.token_ranges
        qs, ks, vs = (ol.scatter_sequence(_f64(x, w), tr, prefix=w.prefix) for x in storage)
        ref = oring.ulysses_ring_attention(qs, ks, vs, tr, w.world // ring, ring, prefix=w.prefix)
        for r in range(plan.world):
            assert_close(_out64(out[r], w), ref[r], "bf16", f"{w.name} chunks={n} rank={r}")
        plan.close()


TWO_CTA_CASES = [w for w in CASES if w.head_dim in (64, 80)] + [
    Workload("tc-bf16-B3-T576-cls-H4-D80-P4", 3, 576, 1, 4, 80, 4, "bf16", 1.0, 9521, (1, 2)),
    Workload("tc-fp16-T300-H2-D64-P2", 1, 300, 0, 2, 64, 2, "fp16", 1.0, 9522, (1,)),
]


@pytest.mark.parametrize("w", TWO_CTA_CASES, ids=lambda w: w.name)
def test_two_cta_matches_oracle(usp, w):
    """One query tile per CTA, two CTAs per SM: the same kernel at QT=1."""
    for n in w.num_chunks:
        storage, plan, out = _run(usp, w, "two_cta", n)
        f64 = [_f64(x, w) for x in storage]
        sh = [ol.scatter_sequence(x, plan.token_ranges, prefix=w.prefix) for x in f64]
        ref = oa.ulysses_attention(*sh, plan.token_ranges, plan.head_ranges, kv_head_ranges=plan.kv_head_ranges,
                                   prefix=w.prefix)
        for r in range(plan.world):
            assert_close(_out64(out[r], w), ref[r], "bf16", f"{w.name} chunks={n} rank={r}")
        plan.close()


@pytest.mark.parametrize("case", [c for c in RING_CASES if c[0].head_dim in (64, 80)], ids=lambda c: c[0].name)
def test_two_cta_ring_matches_oracle(usp, case):
    w, ring = case
    storage, plan, out = _run(usp, w, "two_cta", 1, ring=ring)
    tr = plan.token_ranges
    qs, ks, vs = (ol.scatter_sequence(_f64(x, w), tr, prefix=w.prefix) for x in storage)
    ref = oring.ulysses_ring_attention(qs, ks, vs, tr, w.world // ring, ring, prefix=w.prefix)
    for r in range(plan.world):
        assert_close(_out64(out[r], w), ref[r], "bf16", f"{w.name} rank={r}")
    plan.close()


@pytest.mark.parametrize("w", TWO_CTA_CASES[:3] + TWO_CTA_CASES[-2:], ids=lambda w: w.name)
def test_two_cta_walk_is_bit_identical(usp, w):
    """Capped so that each CTA walks several items (item hand-off through
    q_empty and o_free): the same bits as one item per CTA."""
    _, p0, base = _run(usp, w, "two_cta", 1, ctas=1 << 20)
    bits = [o.view(torch.int16).cpu() for o in base]
    p0.close()
    for ctas in (1, 2, 5):
        _, pc, out = _run(usp, w, "two_cta", 1, ctas=ctas)
        for r, o in enumerate(out):
            assert torch.equal(o.view(torch.int16).cpu(), bits[r]), f"ctas={ctas} rank={r}"
        pc.close()


@pytest.mark.parametrize("case", [c for c in RING_CASES if c[0].head_dim in (64, 80)], ids=lambda c: c[0].name)
def test_two_cta_ring_walk_is_bit_identical(usp, case):
    w, ring = case
    _, p0, base = _run(usp, w, "two_cta", 1, ring=ring, ctas=1 << 20)
    bits = [o.view(torch.int16).cpu() for o in base]
    p0.close()
    _, pc, out = _run(usp, w, "two_cta", 1, ring=ring, ctas=3)
    for r, o in enumerate(out):
        assert torch.equal(o.view(torch.int16).cpu(), bits[r]), f"rank={r}"
    pc.close()


def test_two_cta_agrees_bitwise_with_two_tile(usp):
    """Both run the same per-tile arithmetic in the same order: identical bits."""
    w = TWO_CTA_CASES[0]
    _, p1, o1 = _run(usp, w, "two_cta", 1)
    _, p2, o2 = _run(usp, w, "two_tile", 1)
    for r in range(p1.world):
        assert torch.equal(o1[r].view(torch.int16).cpu(), o2[r].view(torch.int16).cpu()), f"rank {r}"
    p1.close()
    p2.close()


@pytest.mark.parametrize("kernel", ["two_tile", "two_cta"])
def test_two_tile_lse(usp, kernel):
    w = CASES[1]
    lse = torch.full((w.heads, w.batch, w.tokens), float("nan"), dtype=torch.float32, device="cuda")
    storage, plan, _ = _run(usp, w, kernel, 1, lse=lse)
    q, k, _v = (_f64(x, w) for x in storage)
    scale = 1.0 / np.sqrt(w.head_dim)
    got = lse.cpu().numpy()
    for h in range(w.heads):
        for b in range(w.batch):
            s = (q[b, :, h] @ k[b, :, h].T) * scale
            mx = s.max(axis=1)
            ref = mx + np.log(np.exp(s - mx[:, None]).sum(axis=1))
            np.testing.assert_allclose(got[h, b], ref, rtol=0, atol=2e-3)
    plan.close()


def test_two_tile_refused_where_not_built(usp):
    plan = usp.Plan(1, 100, 4, 48, 2, "bf16", 0)
    with pytest.raises(usp.UspError) as e:
        plan.set_attention_kernel("two_tile")
    assert e.value.code == usp.USP_ERR_UNSUPPORTED
    with pytest.raises(usp.UspError) as e:
        plan.set_attention_kernel("two_cta")
    assert e.value.code == usp.USP_ERR_UNSUPPORTED
    plan.close()
    plan = usp.Plan(1, 100, 4, 128, 2, "bf16", 0)
    with pytest.raises(usp.UspError) as e:
        plan.set_attention_kernel("two_cta")
    assert e.value.code == usp.USP_ERR_UNSUPPORTED
    with pytest.raises(usp.UspError) as e:
        plan.set_attention_kernel("fastest")
    assert e.value.code == usp.USP_ERR_INVALID_ARG
    plan.close()

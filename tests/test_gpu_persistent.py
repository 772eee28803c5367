"""Persistent attention CTAs of the one-tile kernel: with fewer CTAs than
(query tile, batch, head) items, each CTA walks several items and overlaps one
item's loads and first Q K^T with the previous item's last key tiles. Every
item is computed the same way, so a capped launch must give the same bits as
the one-CTA-per-item launch of that kernel (which the other attention tests
pin to the float64 oracle). The ViT workload (577-token items) is also
compared with the oracle directly, through the automatic choice and through
the persistent launch."""

import numpy as np
import pytest
import torch

from oracle import layout as ol
from oracle import ring as oring
from oracle.attention import attention_bshd
from tests.gpu_util import assert_close, to_device, to_f64
from ulysses_sequence_attention_sp_b200.synth import make_qkv, storage_to_f64
from ulysses_sequence_attention_sp_b200.workloads import VIT, Workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def usp():
    from ulysses_sequence_attention_sp_b200 import usp as mod
    assert torch.cuda.is_available()
    mod.device_status(reset=True)
    return mod


def _dev(x, w):
    if w.dtype == "fp16":
        return torch.from_numpy(x).cuda()
    return to_device(x, w.dtype)


def _storage(w):
    if w.dtype != "fp16":
        return make_qkv(w)
    rng = np.random.default_rng(w.seed)
    shape = (w.batch, w.tokens, w.heads, w.head_dim)
    return tuple(rng.standard_normal(shape, dtype=np.float32).astype(np.float16) for _ in range(3))


def _block(usp, w, storage, ring=1, ctas=0, num_chunks=1, lse=None, kernel="one_tile"):
    plan = usp.Plan(w.batch, w.seq_len, w.heads, w.head_dim, w.world, w.dtype, w.prefix, kv_heads=w.heads_kv,
                    ring_size=ring)
    plan.set_attention_kernel(kernel)
    plan.set_attention_ctas(ctas)
    shards = [usp.scatter_sequence(plan, _dev(x, w)) for x in storage]
    out = plan.empty_seq_shards(fill=float("nan"))
    usp.ulysses_attention(plan, *shards, out=out, num_chunks=num_chunks, lse=lse)
    torch.cuda.synchronize()
    assert usp.device_status() == 0
    bits = [o.view(torch.int16).cpu() for o in out]
    tr = plan.token_ranges
    plan.close()
    return bits, out, tr


# (workload, ring size): item counts from a handful to a few hundred per launch
CASES = [
    (Workload("p1", 1, 600, 0, 4, 128, 4, "bf16", 1.0, 81, (1,)), 1),              # 5 q tiles x 4 heads, 3 key tiles
    (Workload("p2", 8, 200, 0, 8, 64, 2, "bf16", 1.0, 82, (1,)), 1),               # one key tile per item
    (Workload("p3", 3, 257, 1, 6, 80, 3, "bf16", 0.5, 83, (1,)), 1),               # cls, 2 key tiles, ragged
    (Workload("p4", 2, 517, 0, 8, 128, 2, "bf16", 1.0, 84, (1,), 2), 1),           # grouped-query attention
    (Workload("p5", 2, 260, 0, 4, 48, 4, "fp16", 1.0, 85, (1,)), 1),
    (Workload("p6", 1, 1000, 0, 6, 96, 6, "bf16", 1.0, 86, (1,)), 2),              # Ulysses 3 x Ring 2
    (Workload("p7", 2, 700, 0, 8, 112, 8, "bf16", 1.0, 87, (1,)), 4),              # Ulysses 2 x Ring 4
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0].name}-ring{c[1]}")
def test_capped_launch_is_bit_identical(usp, case):
    w, ring = case
    storage = _storage(w)
    base, _, _ = _block(usp, w, storage, ring=ring)
    for ctas in (1, 3, 7, 148):
        got, _, _ = _block(usp, w, storage, ring=ring, ctas=ctas)
        for r, (a, b) in enumerate(zip(got, base)):
            assert torch.equal(a, b), f"{w.name} ctas={ctas} rank={r}"


@pytest.mark.parametrize("case", [CASES[0], CASES[3], CASES[5]], ids=lambda c: c[0].name)
def test_capped_chunked_block_against_oracle(usp, case):
    """Head-chunked passes (one attention launch per chunk) with 2 CTAs each."""
    w, ring = case
    storage = _storage(w)
    _, out, tr = _block(usp, w, storage, ring=ring, ctas=2, num_chunks=2)
    f64 = [x.astype(np.float64) if w.dtype == "fp16" else storage_to_f64(x, w.dtype) for x in storage]
    qs, ks, vs = (ol.scatter_sequence(x, tr, prefix=w.prefix) for x in f64)
    ref = oring.ulysses_ring_attention(qs, ks, vs, tr, w.world // ring, ring, prefix=w.prefix)
    for r in range(w.world):
        assert_close(to_f64(out[r], w.dtype), ref[r], w.dtype, f"{w.name} rank={r}")


def test_capped_lse_is_bit_identical(usp):
    w, ring = CASES[5]
    storage = _storage(w)
    lse = [torch.full((w.heads, w.batch, w.tokens), float("nan"), dtype=torch.float32, device="cuda")
           for _ in range(2)]
    _block(usp, w, storage, ring=ring, lse=lse[0])
    _block(usp, w, storage, ring=ring, ctas=5, lse=lse[1])
    assert torch.equal(lse[0].view(torch.int32), lse[1].view(torch.int32))


def test_vit_workload_persistent_against_oracle(usp):
    """B=16, cls + 576 patches, H=16, D=80, P=4: 1280 items of 3 key tiles of
    256. The automatic launch (the 128-key kernel, two CTAs per SM) and the
    persistent one-tile launch (one CTA per SM) are both compared with the
    oracle; the persistent launch also with the one-CTA-per-item launch."""
    w = VIT
    storage = make_qkv(w)
    ref = attention_bshd(*(storage_to_f64(x, w.dtype) for x in storage))
    for kernel, ctas in (("auto", 0), ("one_tile", 148)):
        bits, out, tr = _block(usp, w, storage, ctas=ctas, kernel=kernel)
        full = np.concatenate([to_f64(o, w.dtype)[:, (w.prefix if r else 0):] for r, o in enumerate(out)], axis=1)
        assert_close(full, ref, w.dtype, f"vit {kernel}")
        # every rank's copy of the cls row is the same row
        for o in out[1:]:
            assert torch.equal(o[:, 0].view(torch.int16), out[0][:, 0].view(torch.int16))
    # the one-CTA-per-item launch gives the persistent launch's bits
    got, _, _ = _block(usp, w, storage, ctas=1 << 30)
    for a, b in zip(got, bits):
        assert torch.equal(a, b)


def test_attention_cta_cap_rejects_negative(usp):
    plan = usp.Plan(1, 64, 2, 64, 2, "bf16")
    with pytest.raises(usp.UspError) as e:
        plan.set_attention_ctas(-1)
    assert e.value.code == usp.USP_ERR_INVALID_ARG
    plan.close()

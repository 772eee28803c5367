"""Seeded random sweep over the block's configuration space, each case
against the float64 oracle.

Every case draws:
- batch, sequence length and a cls prefix;
- head_dim and dtype (bf16 and fp16 run the tcgen05 kernels, fp32 the SIMT kernel);
- grouped-query attention;
- world and ring size;
- the head-chunk count and an attention CTA cap.

Shapes are small enough for the float64 oracle but span several 128-row query tiles and
256-key tiles with ragged tails. The same case also checks that scatter and gather of its
inputs round-trip bit for bit. A plan the library refuses (some rank's query heads would use
k/v heads another rank owns) must be one the oracle's own check refuses too."""

import numpy as np
import pytest
import torch

from oracle import layout as ol
from oracle import ring as oring
from oracle.partition import balanced_ranges, check_gqa_ranges
from tests.gpu_util import assert_close, to_device, to_f64
from ulysses_sequence_attention_sp_b200.synth import make_qkv, storage_to_f64
from ulysses_sequence_attention_sp_b200.workloads import Workload

pytestmark = pytest.mark.gpu

N_CASES = 120


@pytest.fixture(scope="module")
def usp():
    from ulysses_sequence_attention_sp_b200 import usp as mod
    assert torch.cuda.is_available()
    mod.device_status(reset=True)
    return mod


def _draw(i):
    rng = np.random.default_rng(5000 + i)
    ulysses = int(rng.integers(1, 5))
    ring = int(rng.choice([1, 1, 2, 3]))
    world = ulysses * ring
    kv = ulysses * int(rng.integers(1, 3)) + int(rng.integers(0, 2))  # sometimes not a multiple
    group = int(rng.choice([1, 1, 2, 3]))
    dtype = str(rng.choice(["bf16", "bf16", "fp16", "fp32"]))
    head_dim = int(rng.choice([16, 32, 48, 64, 80, 96, 112, 128]))
    seq_len = int(rng.integers(world, 700 if dtype != "fp32" else 300))
    w = Workload(f"fz{i}", int(rng.integers(1, 4)), seq_len, int(rng.integers(0, 2)), kv * group, head_dim, world,
                 dtype, float(rng.choice([0.5, 1.0])), 6000 + i, (1,), kv, ring)
    return w, int(rng.integers(1, 5)), int(rng.choice([0, 0, 1, 3, 7]))


def _storage(w):
    if w.dtype != "fp16":
        return make_qkv(w)
    rng = np.random.default_rng(w.seed)
    q = (w.std * rng.standard_normal((w.batch, w.tokens, w.heads, w.head_dim), dtype=np.float32)).astype(np.float16)
    kv = [(w.std * rng.standard_normal((w.batch, w.tokens, w.heads_kv, w.head_dim), dtype=np.float32))
          .astype(np.float16) for _ in range(2)]
    return (q, *kv)


def _dev(x, w):
    return torch.from_numpy(x).cuda() if w.dtype == "fp16" else to_device(x, w.dtype)


def _f64(x, w):
    return x.astype(np.float64) if w.dtype == "fp16" else storage_to_f64(x, w.dtype)


def _oracle_refuses(w):
    hr = balanced_ranges(w.heads, w.world // w.ring)
    kr = balanced_ranges(w.heads_kv, w.world // w.ring)
    try:
        check_gqa_ranges(hr, kr, w.heads // w.heads_kv)
    except ValueError:
        return True
    return False


@pytest.mark.parametrize("i", range(N_CASES))
def test_random_configuration(usp, i):
    w, num_chunks, ctas = _draw(i)
    try:
        plan = usp.Plan(w.batch, w.seq_len, w.heads, w.head_dim, w.world, w.dtype, w.prefix, kv_heads=w.heads_kv,
                        ring_size=w.ring)
    except usp.UspError as e:
        assert e.code in (usp.USP_ERR_SHAPE, usp.USP_ERR_INVALID_ARG), e
        assert _oracle_refuses(w), f"{w}: the library refused a plan the oracle accepts ({e})"
        return
    assert not _oracle_refuses(w), f"{w}: the library accepted a plan the oracle refuses"
    plan.set_attention_ctas(ctas)
    storage = _storage(w)
    shards = [usp.scatter_sequence(plan, _dev(x, w)) for x in storage]
    # scatter then gather gives back the same bits
    for x, sh in zip(storage, shards):
        back = usp.gather_sequence(plan, sh)
        assert torch.equal(back.view(torch.int16 if back.element_size() == 2 else torch.int32),
                           _dev(x, w).view(torch.int16 if back.element_size() == 2 else torch.int32))
    out = plan.empty_seq_shards(fill=float("nan"))
    usp.ulysses_attention(plan, *shards, out=out, num_chunks=num_chunks)
    torch.cuda.synchronize()
    assert usp.device_status() == 0
    tr = plan.token_ranges
    qs, ks, vs = (ol.scatter_sequence(_f64(x, w), tr, prefix=w.prefix) for x in storage)
    ref = oring.ulysses_ring_attention(qs, ks, vs, tr, w.world // w.ring, w.ring, prefix=w.prefix)
    tol = "bf16" if w.dtype == "fp16" else w.dtype
    got = (lambda t: t.double().cpu().numpy()) if w.dtype == "fp16" else (lambda t: to_f64(t, w.dtype))
    for r in range(w.world):
        assert_close(got(out[r]), ref[r], tol, f"{w} chunks={num_chunks} ctas={ctas} rank={r}")
    plan.close()

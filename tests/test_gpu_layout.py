"""GPU parity of the layout kernels against the oracle: bit-exact on random bit
patterns (NaN payloads, -0 and Inf included), outputs pre-filled with 0xFF so
an unwritten element shows. Full workload sizes and small ragged cases."""

import numpy as np
import pytest
import torch

from oracle import layout as ol
from tests.gpu_util import bits_to_device, device_bits
from ulysses_sequence_attention_sp_b200.synth import make_bits
from ulysses_sequence_attention_sp_b200.workloads import ALL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def usp():
    from ulysses_sequence_attention_sp_b200 import usp as mod
    assert torch.cuda.is_available()
    return mod


def _filled(shape, itemsize):
    dt = {2: torch.int16, 4: torch.int32}[itemsize]
    return torch.full(shape, -1, dtype=dt, device="cuda")


def _same(t, ref):
    got = device_bits(t)
    return got.shape == ref.shape and np.array_equal(got, ref)


def _run_layout_checks(usp, plan, itemsize, seed, ntensors=1):
    P = plan.world
    shape = plan.full_shape()
    xs = [make_bits(shape, itemsize, seed + i) for i in range(ntensors)]
    xd = [bits_to_device(x) for x in xs]
    tr, hr, pre = plan.token_ranges, plan.head_ranges, plan.prefix

    # scatter / gather
    shards = [_filled(plan.seq_shard_shape(r), itemsize) for r in range(P)]
    usp.scatter_sequence(plan, xd[0], out=shards)
    ref_shards = ol.scatter_sequence(xs[0], tr, prefix=pre)
    assert all(_same(a, b) for a, b in zip(shards, ref_shards)), "scatter_sequence"
    full = _filled(shape, itemsize)
    usp.gather_sequence(plan, shards, out=full)
    assert _same(full, xs[0]), "gather_sequence"

    # seq -> head (ntensors at once) and back
    seq = [[bits_to_device(s) for s in ol.scatter_sequence(x, tr, prefix=pre)] for x in xs]
    heads = [[_filled(plan.head_shard_shape(r), itemsize) for r in range(P)] for _ in range(ntensors)]
    usp.ulysses_seq_to_head(plan, seq, out=heads)
    for i, x in enumerate(xs):
        ref_heads = ol.seq_to_head(ol.scatter_sequence(x, tr, prefix=pre), tr, hr, prefix=pre)
        assert all(_same(a, b) for a, b in zip(heads[i], ref_heads)), f"seq_to_head tensor {i}"
    back = [[_filled(plan.seq_shard_shape(r), itemsize) for r in range(P)] for _ in range(ntensors)]
    usp.ulysses_head_to_seq(plan, heads, out=back)
    for i, x in enumerate(xs):
        ref_back = ol.head_to_seq(ol.seq_to_head(ol.scatter_sequence(x, tr, prefix=pre), tr, hr, prefix=pre),
                                  tr, hr, prefix=pre)
        assert all(_same(a, b) for a, b in zip(back[i], ref_back)), f"head_to_seq tensor {i}"
        assert all(_same(a, b) for a, b in zip(back[i], ol.scatter_sequence(x, tr, prefix=pre)))

    # head slice / gather
    sl = [_filled(plan.head_shard_shape(r), itemsize) for r in range(P)]
    usp.sp_head_slice(plan, xd[0], out=sl)
    assert all(_same(a, b) for a, b in zip(sl, ol.sp_head_slice(xs[0], hr))), "sp_head_slice"
    g = _filled(shape, itemsize)
    usp.sp_head_gather(plan, sl, out=g)
    assert _same(g, xs[0]), "sp_head_gather"
    torch.cuda.synchronize()
    assert usp.device_status() == 0


MODES = ["vector", "tma"]  # how sequence -> head moves run (16-byte vectors or TMA tile copies)


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("w", ALL, ids=[w.name for w in ALL])
def test_layout_full_size(usp, w, mode):
    with usp.Plan(w.batch, w.seq_len, w.heads, w.head_dim, w.world, w.dtype, w.prefix) as plan:
        plan.set_pack_mode(mode)
        _run_layout_checks(usp, plan, w.elem_bytes, seed=2000 + w.seed % 1000)


SMALL = [  # batch, seq_len, heads, head_dim, world, dtype, prefix, ntensors
    (1, 37, 6, 16, 4, "fp32", 0, 3),
    (2, 11, 5, 8, 3, "bf16", 0, 3),
    (3, 9, 4, 40, 4, "bf16", 1, 2),
    (1, 5, 7, 24, 5, "bf16", 1, 3),
    (2, 8, 3, 4, 1, "bf16", 0, 1),      # world 1: every op is a copy
    (2, 8, 3, 4, 1, "fp32", 1, 3),
    (1, 33, 8, 2, 8, "bf16", 0, 3),     # 4-byte head units
    (1, 33, 8, 3, 4, "fp32", 0, 2),     # 12-byte head units
    (1, 17, 16, 1, 4, "bf16", 0, 1),    # 2-byte head units
    (1, 10, 5, 3, 2, "bf16", 1, 3),     # 30-byte token rows: exchanges only
    (4, 32, 32, 128, 32, "bf16", 1, 3), # largest world
]


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("case", SMALL)
def test_layout_small_ragged(usp, case, mode):
    batch, seq_len, heads, dim, world, dtype, prefix, nt = case
    with usp.Plan(batch, seq_len, heads, dim, world, dtype, prefix) as plan:
        plan.set_pack_mode(mode)
        itemsize = 4 if dtype == "fp32" else 2
        if (heads * dim * itemsize) % 16:
            # scatter/gather need 16-byte rows; the exchanges do not
            x = [make_bits(plan.full_shape(), itemsize, 77 + i) for i in range(nt)]
            seq = [[bits_to_device(s) for s in ol.scatter_sequence(xx, plan.token_ranges, prefix=prefix)] for xx in x]
            heads_out = usp.ulysses_seq_to_head(plan, seq)
            for i, xx in enumerate(x):
                ref = ol.seq_to_head(ol.scatter_sequence(xx, plan.token_ranges, prefix=prefix), plan.token_ranges,
                                     plan.head_ranges, prefix=prefix)
                assert all(_same(a, b) for a, b in zip(heads_out[i], ref))
            back = usp.ulysses_head_to_seq(plan, heads_out)
            for i, xx in enumerate(x):
                ref = ol.scatter_sequence(xx, plan.token_ranges, prefix=prefix)
                assert all(_same(a, b) for a, b in zip(back[i], ref))
            with pytest.raises(usp.UspError):
                usp.scatter_sequence(plan, bits_to_device(x[0]))
        else:
            _run_layout_checks(usp, plan, itemsize, seed=300 + seq_len, ntensors=nt)


def test_layout_rejects_bad_tensors(usp):
    with usp.Plan(1, 16, 4, 16, 2, "bf16") as plan:
        x = torch.zeros(plan.full_shape(), dtype=torch.bfloat16, device="cuda")
        with pytest.raises(usp.UspError):
            usp.scatter_sequence(plan, x[:, :8])                       # wrong shape
        with pytest.raises(usp.UspError):
            usp.scatter_sequence(plan, x.float())                      # wrong element size
        bad = [torch.zeros(plan.seq_shard_shape(r), dtype=torch.bfloat16, device="cuda") for r in range(2)]
        with pytest.raises(usp.UspError):
            usp.gather_sequence(plan, [b.transpose(1, 2) for b in bad])  # not contiguous

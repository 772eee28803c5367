"""GPU parity of the Ulysses + Ring hybrid block and of the log-sum-exp output.

The hybrid plan groups consecutive virtual ranks into Ulysses groups; the
kernel takes every group's queries over the k/v blocks of the ring in ring
order, carrying the online-softmax state (the factored log-sum-exp) from one
block to the next. Compared element by element with the float64 oracle,
which runs the ring steps one by one and merges them by log-sum-exp."""

import numpy as np
import pytest
import torch

from oracle import layout as ol
from oracle import ring as oring
from tests.gpu_util import assert_close, to_device, to_f64
from oracle.attention import default_scale
from ulysses_sequence_attention_sp_b200.synth import bf16_bits_to_f32, make_qkv, storage_to_f64
from ulysses_sequence_attention_sp_b200.workloads import HYBRID, Workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def usp():
    from ulysses_sequence_attention_sp_b200 import usp as mod
    assert torch.cuda.is_available()
    mod.device_status(reset=True)
    return mod


# (workload with world = ulysses * ring, ring size)
CASES = [
    (Workload("r1", 1, 600, 0, 4, 128, 4, "bf16", 1.0, 41, (1, 2)), 2),
    (Workload("r2", 2, 333, 1, 6, 64, 6, "bf16", 1.0, 42, (1, 3)), 2),
    (Workload("r3", 1, 1000, 0, 4, 128, 4, "bf16", 1.0, 43, (1,)), 4),           # pure ring
    (Workload("r4", 1, 517, 0, 8, 128, 6, "bf16", 1.0, 44, (1, 2), 2), 3),       # grouped-query attention
    (Workload("r5", 1, 260, 0, 5, 80, 4, "fp16", 1.0, 45, (1, 2)), 2),
    (Workload("r6", 2, 77, 1, 4, 16, 4, "fp32", 1.0, 46, (1, 2)), 2),
    (Workload("r7", 1, 2000, 0, 6, 96, 12, "bf16", 1.0, 47, (1, 2, 3)), 4),
    (Workload("r8", 1, 300, 0, 3, 128, 3, "bf16", 1.0, 48, (1,)), 1),            # ring of one
]


def _storage(w):
    if w.dtype != "fp16":
        return make_qkv(w)
    rng = np.random.default_rng(w.seed)
    shape = (w.batch, w.tokens, w.heads, w.head_dim)
    return tuple(rng.standard_normal(shape, dtype=np.float32).astype(np.float16) for _ in range(3))


def _dev(x, w):
    if w.dtype == "fp16":
        return torch.from_numpy(x).cuda()
    return to_device(x, w.dtype)


def _f64(x, w):
    return x.astype(np.float64) if w.dtype == "fp16" else storage_to_f64(x, w.dtype)


def _plan(usp, w, ring):
    return usp.Plan(w.batch, w.seq_len, w.heads, w.head_dim, w.world, w.dtype, w.prefix, kv_heads=w.heads_kv,
                    ring_size=ring)


def _run(usp, w, ring, num_chunks, lse=None):
    storage = _storage(w)
    plan = _plan(usp, w, ring)
    shards = [usp.scatter_sequence(plan, _dev(x, w)) for x in storage]
    out = plan.empty_seq_shards(fill=float("nan"))
    usp.ulysses_attention(plan, *shards, out=out, num_chunks=num_chunks, lse=lse)
    torch.cuda.synchronize()
    assert usp.device_status() == 0
    return storage, plan, out


def _out_f64(t, w):
    return t.double().cpu().numpy() if w.dtype == "fp16" else to_f64(t, w.dtype)


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0].name}-ring{c[1]}")
def test_hybrid_block_elementwise(usp, case):
    w, ring = case
    for n in w.num_chunks:
        storage, plan, out = _run(usp, w, ring, n)
        assert (plan.ulysses_size, plan.ring_size) == (w.world // ring, ring)
        tr = plan.token_ranges
        qs, ks, vs = (ol.scatter_sequence(_f64(x, w), tr, prefix=w.prefix) for x in storage)
        ref = oring.ulysses_ring_attention(qs, ks, vs, tr, w.world // ring, ring, prefix=w.prefix)
        tol = "bf16" if w.dtype == "fp16" else w.dtype
        for r in range(plan.world):
            assert_close(_out_f64(out[r], w), ref[r], tol, f"{w.name} ring={ring} chunks={n} rank={r}")
        plan.close()


@pytest.mark.parametrize("case", [CASES[0], CASES[3], CASES[6]], ids=lambda c: c[0].name)
def test_hybrid_chunk_counts_bit_identical(usp, case):
    w, ring = case
    base = None
    g = max(b - a for a, b in usp.balanced_ranges(w.heads, w.world // ring))
    for n in sorted({1, 2, 3, g, g + 2}):
        _, plan, out = _run(usp, w, ring, n)
        bits = [o.view(torch.int16).cpu() for o in out]
        if base is None:
            base = bits
        else:
            assert all(torch.equal(a, b) for a, b in zip(bits, base)), f"num_chunks={n}"
        plan.close()


def test_ring_of_one_is_the_plain_block_bit_for_bit(usp):
    w, _ = CASES[7]
    _, plan, hybrid = _run(usp, w, 1, 1)
    plain_plan = usp.Plan(w.batch, w.seq_len, w.heads, w.head_dim, w.world, w.dtype, w.prefix)
    shards = [usp.scatter_sequence(plain_plan, _dev(x, w)) for x in _storage(w)]
    plain = usp.ulysses_attention(plain_plan, *shards)
    torch.cuda.synchronize()
    for a, b in zip(hybrid, plain):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    plan.close()
    plain_plan.close()


@pytest.mark.parametrize("case", [CASES[0], CASES[1], CASES[5]], ids=lambda c: c[0].name)
def test_lse_output(usp, case):
    """The log-sum-exp of every row over all keys, against float64
    log(sum exp(scale q.k)); the ring path and the plain block agree on it."""
    w, ring = case
    lse = torch.full((w.heads, w.batch, w.tokens), float("nan"), dtype=torch.float32, device="cuda")
    storage, plan, _ = _run(usp, w, ring, 1, lse=lse)
    q, k, _v = (_f64(x, w) for x in storage)
    group = w.heads // w.heads_kv
    scale = 1.0 / np.sqrt(w.head_dim)
    got = lse.cpu().numpy()
    for h in range(w.heads):
        for b in range(w.batch):
            s = (q[b, :, h] @ k[b, :, h // group].T) * scale
            m = s.max(axis=1)
            ref = m + np.log(np.exp(s - m[:, None]).sum(axis=1))
            np.testing.assert_allclose(got[h, b], ref, rtol=0, atol=2e-3 if w.dtype != "fp32" else 1e-4)
    plain = usp.Plan(w.batch, w.seq_len, w.heads, w.head_dim, w.world, w.dtype, w.prefix)
    shards = [usp.scatter_sequence(plain, _dev(x, w)) for x in storage]
    lse2 = torch.full_like(lse, float("nan"))
    usp.ulysses_attention(plain, *shards, lse=lse2)
    torch.cuda.synchronize()
    assert torch.allclose(lse, lse2, rtol=0, atol=1e-4)
    plan.close()
    plain.close()


def test_hybrid_plan_refuses_head_shard_calls(usp):
    w, ring = CASES[0]
    plan = _plan(usp, w, ring)
    x = [torch.zeros(plan.seq_shard_shape(r), dtype=torch.bfloat16, device="cuda") for r in range(plan.world)]
    with pytest.raises(usp.UspError) as e:
        usp.ulysses_seq_to_head(plan, [x])
    assert e.value.code == usp.USP_ERR_UNSUPPORTED
    plan.close()


@pytest.mark.parametrize("mode", ["vector", "tma"])
def test_hybrid_replays_from_a_cuda_graph(usp, mode):
    """The hybrid block (ring walk, chunk overlap on the auxiliary stream, either
    pack) captured once into a CUDA graph and replayed on new inputs written
    into the same buffers gives the same bits as a direct call."""
    w, ring = CASES[6]
    plan = _plan(usp, w, ring)
    plan.set_pack_mode(mode)
    ins = [plan.empty_seq_shards() for _ in range(3)]
    out = plan.empty_seq_shards(fill=float("nan"))
    ws = torch.empty(plan.workspace_bytes(3), dtype=torch.uint8, device="cuda")

    def load(seed):
        for x, dst in zip(make_qkv(w, seed), ins):
            usp.scatter_sequence(plan, _dev(x, w), out=dst)

    load(11)
    usp.ulysses_attention(plan, *ins, out=out, num_chunks=3, workspace=ws)  # warm-up
    torch.cuda.synchronize()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(cap):
        with torch.cuda.graph(graph, stream=cap):
            usp.ulysses_attention(plan, *ins, out=out, num_chunks=3, workspace=ws)
    torch.cuda.current_stream().wait_stream(cap)
    for seed in (12, 13):
        load(seed)
        for o in out:
            o.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        ref = usp.ulysses_attention(plan, *ins, num_chunks=3)
        torch.cuda.synchronize()
        for a, b in zip(out, ref):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert usp.device_status() == 0
    del graph
    plan.close()


def _hybrid_sample_rows(plan, groups, rng, n_random=24):
    """Every rank boundary, both edges of every ring block, first and last
    rows, and seeded random rows (full-sequence row numbers)."""
    rows = {0, 1, plan.tokens - 1, plan.tokens - 2}
    for t0, t1 in plan.token_ranges:
        rows.update(plan.prefix + t for t in (t0 - 1, t0, t1 - 1) if 0 <= t < plan.seq_len)
    for _members, (b0, b1), _local in groups:
        rows.update(plan.prefix + t for t in (b0 - 1, b0, b0 + 1, b1 - 2, b1 - 1, b1) if 0 <= t < plan.seq_len)
    rows.update(int(x) for x in rng.integers(0, plan.tokens, size=n_random))
    return sorted(rows)


def test_full_size_hybrid_sampled_rows(usp):
    """The video latent as Ulysses 4 x Ring 2 (T=75600, H=24, D=128, two ring
    blocks of 37,800 keys, each ending in a ragged 256-key tile), in the
    launch configuration the benchmark times. Sampled rows of every head are
    computed by the oracle's ring steps: the row's own block first, then the
    previous ring block, each normalised over its keys with its log-sum-exp,
    merged by log-sum-exp weights."""
    w = HYBRID
    ring, uly = w.ring, w.world // w.ring
    storage, plan, out = _run(usp, w, ring, w.num_chunks[0])
    for o in out:
        assert not torch.isnan(o).any().item(), "an output element was never written"
    q, k, v = storage
    groups = oring.ring_groups(plan.token_ranges, uly, ring)
    rows = _hybrid_sample_rows(plan, groups, np.random.default_rng(8))
    assert 37799 in rows and 37800 in rows

    def block_rows(gp):
        b0, b1 = groups[gp][1]
        keys = np.arange(plan.prefix + b0, plan.prefix + b1)
        return np.concatenate([np.arange(plan.prefix), keys]) if gp == 0 else keys

    def group_of(t):
        tok = t - plan.prefix
        return 0 if tok < 0 else next(g for g, (_m, (b0, b1), _l) in enumerate(groups) if b0 <= tok < b1)

    scale = default_scale(w.head_dim)
    got_all, ref_all = [], []
    for b in range(w.batch):
        for h in range(w.heads):
            kh = storage_to_f64(k[b, :, h], w.dtype)
            vh = storage_to_f64(v[b, :, h], w.dtype)
            for g in range(ring):
                rows_g = [t for t in rows if group_of(t) == g]
                qh = storage_to_f64(q[b, rows_g, h], w.dtype)
                o = lse = None
                for step in range(ring):
                    keys = block_rows((g - step) % ring)
                    o_s, lse_s = oring.block_attention(qh, kh[keys], vh[keys], scale)
                    o, lse = (o_s, lse_s) if o is None else oring.merge_partials(o, lse, o_s, lse_s)
                for i, t in enumerate(rows_g):
                    tok = t - plan.prefix
                    owners = range(w.world) if tok < 0 else [
                        next(r for r, (a, c) in enumerate(plan.token_ranges) if a <= tok < c)]
                    for r in owners:
                        local = t if tok < 0 else plan.prefix + tok - plan.token_ranges[r][0]
                        got_all.append(to_f64(out[r][b, local, h], w.dtype))
                        ref_all.append(o[i])
    st = assert_close(np.stack(got_all), np.stack(ref_all), w.dtype, w.name)
    print(w.name, len(rows), "rows x", w.heads, "heads", st)
    plan.close()


def test_full_size_hybrid_every_element_against_fp32_kernel(usp):
    """Secondary signal at full size: every output element of the hybrid block
    against the fp32 CUDA-core kernel's ring walk on the same values (the bf16
    inputs upcast exactly), with the bf16 tolerances."""
    w = HYBRID
    storage, plan, out = _run(usp, w, w.ring, w.num_chunks[0])
    plan32 = usp.Plan(w.batch, w.seq_len, w.heads, w.head_dim, w.world, "fp32", w.prefix, ring_size=w.ring)
    shards32 = [usp.scatter_sequence(plan32, torch.from_numpy(bf16_bits_to_f32(x)).cuda()) for x in storage]
    del storage
    out32 = usp.ulysses_attention(plan32, *shards32)
    torch.cuda.synchronize()
    assert usp.device_status() == 0
    for r in range(w.world):
        got, ref = out[r].double(), out32[r].double()
        diff = (got - ref).abs()
        st = {"max_abs": diff.max().item(), "mean_abs": diff.mean().item(),
              "rel_l2": ((got - ref).norm() / ref.norm()).item(), "nan": int(torch.isnan(got).sum().item())}
        assert st["nan"] == 0 and st["max_abs"] <= 2e-2 and st["mean_abs"] <= 2e-3 and st["rel_l2"] <= 1e-2, (r, st)
    print(w.name, "rank", w.world - 1, st)
    plan.close()
    plan32.close()

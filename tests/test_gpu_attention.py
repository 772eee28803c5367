"""GPU parity of the attention block against the float64 oracle.

Small cases (several tiles, ragged tails, cls prefix, ragged heads, chunking)
are compared element by element; the full-size workloads run in the launch
configuration the benchmark times and are compared on sampled rows that the
oracle computes one by one (every rank boundary, first and last rows, the cls
row, and seeded random rows), plus a check that every output element was
written."""

import numpy as np
import pytest
import torch

from oracle import attention as oa
from oracle import layout as ol
from tests.gpu_util import assert_close, to_device, to_f64
from ulysses_sequence_attention_sp_b200.synth import bf16_bits_to_f32, f32_to_bf16_bits, make_qkv, storage_to_f64
from ulysses_sequence_attention_sp_b200.workloads import CHUNKED, TINY, VIDEO, VIT, Workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def usp():
    from ulysses_sequence_attention_sp_b200 import usp as mod
    assert torch.cuda.is_available()
    mod.device_status(reset=True)
    return mod


def _plan(usp, w):
    return usp.Plan(w.batch, w.seq_len, w.heads, w.head_dim, w.world, w.dtype, w.prefix)


def _nan_shards(plan):
    return plan.empty_seq_shards(fill=float("nan"))


def _times4(bits):
    """Exact multiplication of bf16 values by 4 (exponent + 2)."""
    x = bf16_bits_to_f32(bits) * np.float32(4.0)
    return f32_to_bf16_bits(x)


def _run_block(usp, w, num_chunks, seed=None):
    """Full-sequence q/k/v -> device, scatter on the GPU, Ulysses block; returns
    (host storage, plan, output shards)."""
    q, k, v = make_qkv(w, seed)
    if w.name == "s8":
        # scores with a spread of ~16: row maxima keep growing across key
        # tiles, so the O rescale in tensor memory runs
        q, k = _times4(q), _times4(k)
    plan = _plan(usp, w)
    shards = [usp.scatter_sequence(plan, to_device(x, w.dtype)) for x in (q, k, v)]
    out = _nan_shards(plan)
    usp.ulysses_attention(plan, *shards, out=out, num_chunks=num_chunks)
    torch.cuda.synchronize()
    assert usp.device_status() == 0
    return (q, k, v), plan, out


def _oracle_block(w, storage, plan, num_chunks=1):
    q, k, v = (storage_to_f64(x, w.dtype) for x in storage)
    tr, hr = plan.token_ranges, plan.head_ranges
    qs, ks, vs = (ol.scatter_sequence(x, tr, prefix=w.prefix) for x in (q, k, v))
    return oa.ulysses_attention(qs, ks, vs, tr, hr, prefix=w.prefix, num_chunks=num_chunks)


SMALL = [
    Workload("s1", 1, 300, 0, 6, 128, 4, "bf16", 1.0, 11, (1,)),
    Workload("s2", 2, 200, 1, 5, 80, 3, "bf16", 0.5, 12, (1,)),
    Workload("s3", 1, 1000, 0, 3, 64, 3, "bf16", 1.0, 13, (1,)),
    Workload("s4", 1, 77, 0, 4, 16, 2, "bf16", 1.0, 14, (1,)),
    Workload("s5", 1, 128, 0, 2, 32, 2, "bf16", 1.0, 15, (1,)),
    Workload("s6", 1, 129, 0, 2, 48, 1, "bf16", 1.0, 16, (1,)),
    Workload("s7", 1, 260, 0, 4, 128, 4, "fp16", 1.0, 17, (1,)),
    Workload("s8", 1, 700, 0, 2, 128, 2, "bf16", 1.0, 18, (1,)),   # q, k scaled by 4 below: rescale path
    Workload("s9", 3, 40, 1, 8, 96, 8, "bf16", 1.0, 19, (1,)),
    Workload("s10", 1, 384, 0, 9, 112, 4, "bf16", 1.0, 20, (1,)),
    Workload("s11", 2, 333, 0, 5, 16, 5, "fp32", 1.0, 21, (1,)),
    Workload("s12", 1, 50, 1, 3, 80, 3, "fp32", 1.0, 22, (1,)),
]


@pytest.mark.parametrize("w", [TINY] + [w for w in SMALL if w.dtype != "fp16"], ids=lambda w: w.name)
def test_block_small_elementwise(usp, w):
    """bf16 and fp32 cases (the fp16 case has its own storage: test_fp16_block)."""
    for n in sorted(set(w.num_chunks) | {1, 2}):
        storage, plan, out = _run_block(usp, w, n)
        ref = _oracle_block(w, storage, plan)
        for r in range(plan.world):
            assert_close(to_f64(out[r], w.dtype), ref[r], w.dtype, f"{w.name} chunks={n} rank={r}")
        plan.close()


def test_fp16_block(usp):
    w = SMALL[6]
    rng = np.random.default_rng(w.seed)
    shape = (w.batch, w.tokens, w.heads, w.head_dim)
    host = [rng.standard_normal(shape, dtype=np.float32).astype(np.float16) for _ in range(3)]
    plan = usp.Plan(w.batch, w.seq_len, w.heads, w.head_dim, w.world, "fp16", w.prefix)
    dev = [usp.scatter_sequence(plan, torch.from_numpy(x).cuda()) for x in host]
    out = _nan_shards(plan)
    usp.ulysses_attention(plan, *dev, out=out)
    torch.cuda.synchronize()
    tr, hr = plan.token_ranges, plan.head_ranges
    qs, ks, vs = (ol.scatter_sequence(x.astype(np.float64), tr) for x in host)
    ref = oa.ulysses_attention(qs, ks, vs, tr, hr)
    for r in range(plan.world):
        assert_close(out[r].double().cpu().numpy(), ref[r], "fp16", f"fp16 rank={r}")
    plan.close()


@pytest.mark.parametrize("w", SMALL[:4] + SMALL[8:10], ids=lambda w: w.name)
def test_chunk_counts_bit_identical(usp, w):
    base = None
    g = max(b - a for a, b in usp.balanced_ranges(w.heads, w.world))
    for n in [1, 2, 3, g, g + 2]:
        _, plan, out = _run_block(usp, w, n)
        bits = [o.view(torch.int16).cpu() for o in out]
        if base is None:
            base = bits
        else:
            assert all(torch.equal(a, b) for a, b in zip(bits, base)), f"num_chunks={n}"
        plan.close()


@pytest.mark.parametrize("w", SMALL[:3] + [SMALL[10]], ids=lambda w: w.name)
def test_head_attention_matches_oracle(usp, w):
    q, k, v = make_qkv(w)
    plan = _plan(usp, w)
    hr = plan.head_ranges
    heads = [[to_device(np.ascontiguousarray(x[:, :, h0:h1]), w.dtype) for h0, h1 in hr] for x in (q, k, v)]
    out = plan.empty_head_shards(fill=float("nan"))
    usp.head_attention(plan, *heads, out=out)
    torch.cuda.synchronize()
    qf, kf, vf = (storage_to_f64(x, w.dtype) for x in (q, k, v))
    for r, (h0, h1) in enumerate(hr):
        ref = oa.attention_bshd(qf[:, :, h0:h1], kf[:, :, h0:h1], vf[:, :, h0:h1])
        assert_close(to_f64(out[r], w.dtype), ref, w.dtype, f"rank {r}")
    plan.close()


def _sample_rows(plan, rng, n_random=24):
    rows = {0, 1, plan.tokens - 1, plan.tokens - 2}
    for t0, t1 in plan.token_ranges:
        for t in (t0 - 1, t0, t1 - 1):
            if 0 <= t < plan.seq_len:
                rows.add(plan.prefix + t)
    rows.update(int(x) for x in rng.integers(0, plan.tokens, size=n_random))
    return sorted(rows)


def _owner(plan, t):
    if t < plan.prefix:
        return list(range(plan.world)), t
    tok = t - plan.prefix
    for r, (a, b) in enumerate(plan.token_ranges):
        if a <= tok < b:
            return [r], plan.prefix + tok - a
    raise AssertionError(t)


@pytest.mark.parametrize("w", [VIDEO, CHUNKED], ids=lambda w: w.name)
def test_full_size_sampled_rows(usp, w):
    """Full workload size, launch configuration of the benchmark; sampled rows."""
    n = w.num_chunks[0]
    storage, plan, out = _run_block(usp, w, n)
    for o in out:
        assert not torch.isnan(o).any().item(), "an output element was never written"
    q, k, v = storage
    rng = np.random.default_rng(7)
    rows = _sample_rows(plan, rng)
    got_all, ref_all = [], []
    for b in range(w.batch):
        for h in range(w.heads):
            qh = storage_to_f64(q[b, rows, h], w.dtype)
            kh = storage_to_f64(k[b, :, h], w.dtype)
            vh = storage_to_f64(v[b, :, h], w.dtype)
            ref = oa.softmax_attention(qh, kh, vh, oa.default_scale(w.head_dim))
            for i, t in enumerate(rows):
                ranks, local = _owner(plan, t)
                for r in ranks:
                    got_all.append(to_f64(out[r][b, local, h], w.dtype))
                    ref_all.append(ref[i])
    st = assert_close(np.stack(got_all), np.stack(ref_all), w.dtype, w.name)
    print(w.name, st)
    plan.close()


@pytest.mark.parametrize("w", [VIDEO, CHUNKED], ids=lambda w: w.name)
def test_full_size_every_row_against_fp32_kernel(usp, w):
    """Secondary signal at full size: every output element of the tensor-core
    block against the fp32 CUDA-core kernel run on the same values (the bf16
    inputs upcast exactly), with the bf16 tolerances. The float64 oracle
    checks sampled rows of the same workloads above."""
    storage, plan, out = _run_block(usp, w, w.num_chunks[0])
    plan32 = usp.Plan(w.batch, w.seq_len, w.heads, w.head_dim, w.world, "fp32", w.prefix)
    shards32 = [usp.scatter_sequence(plan32, torch.from_numpy(bf16_bits_to_f32(x)).cuda()) for x in storage]
    del storage
    out32 = usp.ulysses_attention(plan32, *shards32)
    torch.cuda.synchronize()
    assert usp.device_status() == 0
    for r in range(w.world):
        got = out[r].double()
        ref = out32[r].double()
        diff = (got - ref).abs()
        st = {"max_abs": diff.max().item(), "mean_abs": diff.mean().item(),
              "rel_l2": ((got - ref).norm() / ref.norm()).item(), "nan": int(torch.isnan(got).sum().item())}
        assert st["nan"] == 0 and st["max_abs"] <= 2e-2 and st["mean_abs"] <= 2e-3 and st["rel_l2"] <= 1e-2, (r, st)
    print(w.name, "rank", w.world - 1, st)
    plan.close()
    plan32.close()


def test_vit_full_elementwise(usp):
    """The ViT workload is small enough for the full float64 oracle."""
    storage, plan, out = _run_block(usp, VIT, 1)
    ref = _oracle_block(VIT, storage, plan)
    for r in range(plan.world):
        st = assert_close(to_f64(out[r], VIT.dtype), ref[r], VIT.dtype, f"vit rank {r}")
    print("vit", st)
    plan.close()


def test_chunked_workload_equals_single_shot(usp):
    """Head-chunked workload: num_chunks=3 equals num_chunks=1 (bit for bit:
    heads are independent and each is computed by the same kernel)."""
    _, plan3, out3 = _run_block(usp, CHUNKED, 3)
    _, plan1, out1 = _run_block(usp, CHUNKED, 1)
    for a, b in zip(out3, out1):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    plan3.close()
    plan1.close()


def test_scale_argument(usp):
    w = SMALL[0]
    q, k, v = make_qkv(w)
    plan = _plan(usp, w)
    shards = [usp.scatter_sequence(plan, to_device(x, w.dtype)) for x in (q, k, v)]
    out = usp.ulysses_attention(plan, *shards, scale=0.05)
    torch.cuda.synchronize()
    qf, kf, vf = (storage_to_f64(x, w.dtype) for x in (q, k, v))
    ref = ol.scatter_sequence(oa.attention_bshd(qf, kf, vf, scale=0.05), plan.token_ranges)
    for r in range(plan.world):
        assert_close(to_f64(out[r], w.dtype), ref[r], w.dtype)
    plan.close()


def test_wait_timeout_is_reported_not_hung(usp):
    """A device-side wait on a barrier nothing arrives on gives up after its
    limit, records its site, and leaves the context usable."""
    usp.device_status(reset=True)
    usp.debug_wait_timeout(2000)
    assert usp.device_status(reset=True) == 99
    assert usp.device_status(reset=True) == 0
    # the library still computes correctly afterwards
    storage, plan, out = _run_block(usp, TINY, 1)
    ref = _oracle_block(TINY, storage, plan)
    for r in range(plan.world):
        assert_close(to_f64(out[r], "fp32"), ref[r], "fp32")
    plan.close()


def test_invalid_attention_arguments(usp):
    with usp.Plan(1, 64, 4, 72, 2, "bf16") as plan:   # 72 is not a multiple of 16
        shards = plan.empty_seq_shards(fill=0.0)
        with pytest.raises(usp.UspError) as e:
            usp.ulysses_attention(plan, shards, shards, shards)
        assert e.value.code == usp.USP_ERR_UNSUPPORTED
    with usp.Plan(1, 64, 4, 64, 2, "bf16") as plan:
        shards = plan.empty_seq_shards(fill=0.0)
        with pytest.raises(usp.UspError):
            usp.ulysses_attention(plan, shards, shards, shards, num_chunks=0)
        ws = torch.empty(16, dtype=torch.uint8, device="cuda")
        with pytest.raises(usp.UspError):
            usp.ulysses_attention(plan, shards, shards, shards, workspace=ws)


@pytest.mark.parametrize("num_chunks", [1, 3])
def test_block_replays_from_a_cuda_graph(usp, num_chunks):
    """The block's launches are stream-ordered and synchronise nothing, so the
    whole call (with the auxiliary-stream chunk overlap) can be captured into a
    CUDA graph and replayed on new inputs written into the same buffers."""
    w = SMALL[0]
    plan = _plan(usp, w)
    ins = [plan.empty_seq_shards() for _ in range(3)]
    out = plan.empty_seq_shards(fill=float("nan"))
    ws = torch.empty(plan.workspace_bytes(num_chunks), dtype=torch.uint8, device="cuda")

    def load(seed):
        for x, dst in zip(make_qkv(w, seed), ins):
            usp.scatter_sequence(plan, to_device(x, w.dtype), out=dst)

    load(101)
    usp.ulysses_attention(plan, *ins, out=out, num_chunks=num_chunks, workspace=ws)  # warm-up
    torch.cuda.synchronize()
    ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    for e in ev:
        e.record()
    torch.cuda.synchronize()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(cap):
        plan.set_timing_events(*ev)  # recorded as graph event nodes: every replay records them
        with torch.cuda.graph(graph, stream=cap):
            usp.ulysses_attention(plan, *ins, out=out, num_chunks=num_chunks, workspace=ws)
        plan.set_timing_events(None, None)
    torch.cuda.current_stream().wait_stream(cap)
    for seed in (202, 303):
        load(seed)
        for o in out:
            o.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        ref = usp.ulysses_attention(plan, *ins, num_chunks=num_chunks)
        torch.cuda.synchronize()
        for a, b in zip(out, ref):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16))
        assert ev[0].elapsed_time(ev[1]) > 0.0
    assert usp.device_status() == 0
    del graph
    plan.close()


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_trivial_group_is_byte_identical_to_single_device(usp, dtype):
    """API page, ulysses_attention: a one-rank group gives exactly the non-SP
    result. With P = 1 the block's output equals, bit for bit, the unchanged
    attention run on the full tensors (usp_head_attention on one head shard
    holding every head)."""
    w = Workload("p1", 2, 333, 0, 5, 64 if dtype == "bf16" else 48, 1, dtype, 1.0, 77, (1,))
    q, k, v = (to_device(x, dtype) for x in make_qkv(w))
    plan = _plan(usp, w)
    block = usp.ulysses_attention(plan, [q], [k], [v], num_chunks=2)
    direct = usp.head_attention(plan, [q], [k], [v])
    torch.cuda.synchronize()
    bits = torch.int16 if dtype == "bf16" else torch.int32
    assert torch.equal(block[0].view(bits), direct[0].view(bits))
    plan.close()


def test_largest_world_and_head_count(usp):
    """32 virtual ranks (the largest world) over 256 heads (the largest head
    count), ragged tokens, elementwise against the oracle."""
    w = Workload("max", 1, 97, 1, 256, 16, 32, "bf16", 1.0, 78, (1,))
    storage, plan, out = _run_block(usp, w, 3)
    ref = _oracle_block(w, storage, plan)
    for r in range(plan.world):
        assert_close(to_f64(out[r], w.dtype), ref[r], w.dtype, f"rank {r}")
    plan.close()


def test_fp32_largest_head_dim(usp):
    """fp32 attention at head_dim 256, the largest the fp32 kernel is built for."""
    w = Workload("fp32-d256", 1, 70, 0, 3, 256, 3, "fp32", 1.0, 79, (1,))
    storage, plan, out = _run_block(usp, w, 1)
    ref = _oracle_block(w, storage, plan)
    for r in range(plan.world):
        assert_close(to_f64(out[r], w.dtype), ref[r], w.dtype, f"rank {r}")
    plan.close()

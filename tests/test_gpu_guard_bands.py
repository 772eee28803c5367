"""Guard bands: every output buffer sits between 64 KiB margins filled with a
sentinel byte pattern, and each operation must leave the margins untouched
(an out-of-bounds write anywhere in a kernel shows up here even when the
values inside the buffer are right). Ragged splits, a cls prefix and chunked
passes make the edge offsets irregular."""

import pytest
import torch

from ulysses_sequence_attention_sp_b200.workloads import Workload

pytestmark = pytest.mark.gpu

PAD = 64 * 1024
SENTINEL = 0xA5


@pytest.fixture(scope="module")
def usp():
    from ulysses_sequence_attention_sp_b200 import usp as mod
    assert torch.cuda.is_available()
    mod.device_status(reset=True)
    return mod


class Guarded:
    """Flat byte buffer [PAD | body | PAD]; `body` is the output view."""

    def __init__(self, shape, dtype):
        nbytes = torch.empty((), dtype=dtype).element_size()
        for s in shape:
            nbytes *= s
        self.raw = torch.full((PAD + nbytes + PAD,), SENTINEL, dtype=torch.uint8, device="cuda")
        self.body = self.raw[PAD:PAD + nbytes].view(dtype).view(shape)
        self.nbytes = nbytes

    def margins_intact(self) -> bool:
        head = self.raw[:PAD]
        tail = self.raw[PAD + self.nbytes:]
        return bool((head == SENTINEL).all().item() and (tail == SENTINEL).all().item())


def _guarded_list(shapes, dtype):
    return [Guarded(s, dtype) for s in shapes]


def _check(guards, what):
    torch.cuda.synchronize()
    bad = [i for i, g in enumerate(guards) if not g.margins_intact()]
    assert not bad, f"{what}: margins written around outputs {bad}"


CASES = [  # batch, seq_len, prefix, heads, head_dim, world, dtype, kv_heads, ring
    (1, 37, 0, 6, 16, 4, "fp32", 6, 1),
    (2, 101, 1, 5, 80, 3, "bf16", 5, 1),
    (3, 9, 1, 4, 48, 4, "bf16", 4, 1),
    (1, 517, 0, 8, 64, 2, "bf16", 2, 1),
    (1, 600, 0, 4, 128, 4, "bf16", 4, 2),
]


@pytest.mark.parametrize("mode", ["vector", "tma"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}-T{c[1]}-P{c[5]}-{c[6]}-kv{c[7]}-ring{c[8]}")
def test_no_write_outside_outputs(usp, case, mode):
    batch, seq_len, prefix, heads, dim, world, dtype, kv_heads, ring = case
    plan = usp.Plan(batch, seq_len, heads, dim, world, dtype, prefix, kv_heads=kv_heads, ring_size=ring)
    plan.set_pack_mode(mode)
    tdt = plan.torch_dtype
    gen = torch.Generator(device="cuda").manual_seed(seq_len + world)

    def rand(shape):
        return torch.randn(shape, generator=gen, device="cuda", dtype=torch.float32).to(tdt)

    full = rand(plan.full_shape())
    kv_full = [rand(plan.kv_full_shape()) for _ in range(2)]

    # scatter / gather
    g = _guarded_list([plan.seq_shard_shape(r) for r in range(world)], tdt)
    usp.scatter_sequence(plan, full, out=[x.body for x in g])
    _check(g, "scatter_sequence")
    q = [x.body for x in g]
    gf = Guarded(plan.full_shape(), tdt)
    usp.gather_sequence(plan, q, out=gf.body)
    _check([gf], "gather_sequence")
    assert torch.equal(gf.body, full)
    k, v = (usp.scatter_sequence(plan, x) for x in kv_full)

    if ring == 1:
        # exchanges (q-shaped and kv-shaped), head slice / gather, per-rank attention
        gh = [_guarded_list([plan.head_shard_shape(r) for r in range(world)], tdt) for _ in range(3)]
        usp.ulysses_seq_to_head(plan, [q, q, q], out=[[x.body for x in gg] for gg in gh])
        _check([x for gg in gh for x in gg], "seq_to_head")
        gkv = [_guarded_list([plan.kv_head_shard_shape(r) for r in range(world)], tdt) for _ in range(2)]
        usp.ulysses_seq_to_head(plan, [k, v], out=[[x.body for x in gg] for gg in gkv], kv=True)
        _check([x for gg in gkv for x in gg], "seq_to_head_kv")
        gb = _guarded_list([plan.seq_shard_shape(r) for r in range(world)], tdt)
        usp.ulysses_head_to_seq(plan, [[x.body for x in gh[0]]], out=[[x.body for x in gb]])
        _check(gb, "head_to_seq")
        go = _guarded_list([plan.head_shard_shape(r) for r in range(world)], tdt)
        usp.head_attention(plan, [x.body for x in gh[0]], [x.body for x in gkv[0]], [x.body for x in gkv[1]],
                           out=[x.body for x in go])
        _check(go, "head_attention")
        if (heads * dim * full.element_size()) % 16 == 0:
            gs = _guarded_list([plan.head_shard_shape(r) for r in range(world)], tdt)
            usp.sp_head_slice(plan, full, out=[x.body for x in gs])
            _check(gs, "sp_head_slice")
            gg2 = Guarded(plan.full_shape(), tdt)
            usp.sp_head_gather(plan, [x.body for x in gs], out=gg2.body)
            _check([gg2], "sp_head_gather")

    # row collectives (rows of the plan's split tokens, no prefix)
    row = (heads, dim)
    local = [rand((batch, t1 - t0, *row)) for t0, t1 in plan.token_ranges]
    gfull = _guarded_list([(batch, seq_len, *row)] * world, tdt)
    usp.all_gather_rows(plan, local, out=[x.body for x in gfull])
    _check(gfull, "all_gather_rows")
    glocal = _guarded_list([(batch, t1 - t0, *row) for t0, t1 in plan.token_ranges], tdt)
    usp.reduce_scatter_rows(plan, [x.body for x in gfull], out=[x.body for x in glocal])
    _check(glocal, "reduce_scatter_rows")

    # the block, one and two chunks, with the log-sum-exp output
    for n in (1, 2):
        gout = _guarded_list([plan.seq_shard_shape(r) for r in range(world)], tdt)
        glse = Guarded((heads, batch, plan.tokens), torch.float32)
        gws = Guarded((plan.workspace_bytes(n),), torch.uint8)
        usp.ulysses_attention(plan, q, k, v, out=[x.body for x in gout], num_chunks=n, workspace=gws.body,
                              lse=glse.body)
        _check(gout + [glse, gws], f"ulysses_attention chunks={n}")
    assert usp.device_status() == 0
    plan.close()

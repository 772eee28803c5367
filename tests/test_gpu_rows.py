"""GPU parity of the ragged row collectives (all_gather_rows, reduce_scatter_rows).

all_gather_rows only moves bytes, so it is compared bit for bit with the
oracle on random bit patterns. reduce_scatter_rows sums P partials in fp32 in
rank order and rounds once to the storage type; the oracle sums exactly in
float64. The bound follows from that arithmetic: each of the P-1 fp32 adds
errs by at most 2^-24 of a partial sum no larger than sum_i |x_i|, and the
final rounding by half an ulp of the output type (2^-8 relative for bf16,
2^-11 for fp16, none for fp32). Sums of small integers are exact on both
sides and are compared bit for bit."""

import numpy as np
import pytest
import torch

from oracle import rows as orows
from tests.gpu_util import bits_to_device, device_bits
from ulysses_sequence_attention_sp_b200.synth import f32_to_bf16_bits, make_bits, storage_to_f64

pytestmark = pytest.mark.gpu

TORCH = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32}
ROUND_REL = {"bf16": 2.0 ** -8, "fp16": 2.0 ** -11, "fp32": 0.0}


@pytest.fixture(scope="module")
def usp():
    from ulysses_sequence_attention_sp_b200 import usp as mod
    assert torch.cuda.is_available()
    mod.device_status(reset=True)
    return mod


CASES = [  # batch, seq_len, world, row shape, dtype (rows need not be the plan's H x D)
    (1, 37, 4, (6, 16), "bf16"),
    (2, 101, 7, (3, 40), "bf16"),   # 240-byte rows: 16-byte vectors, ragged split
    (3, 50, 5, (1, 3), "bf16"),     # 6-byte rows: 2-byte vectors
    (1, 64, 8, (2, 2), "fp16"),     # 8-byte rows
    (2, 33, 32, (5, 12), "fp32"),   # 32 ranks, 240-byte rows
    (1, 19, 1, (1, 1), "fp32"),     # one rank; 4-byte rows
    (4, 1000, 3, (8, 64), "bf16"),  # several tiles per segment
]


def _plan(usp, case):
    b, t, p, _row, dt = case
    return usp.Plan(b, t, p, 8, p, dt, 0)


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}-T{c[1]}-P{c[2]}-row{'x'.join(map(str, c[3]))}-{c[4]}")
def test_all_gather_rows_bit_exact(usp, case):
    b, t, p, row, dt = case
    plan = _plan(usp, case)
    itemsize = 4 if dt == "fp32" else 2
    tr = plan.token_ranges
    local = [make_bits((b, t1 - t0, *row), itemsize, 700 + r) for r, (t0, t1) in enumerate(tr)]
    dev = [bits_to_device(x).view(TORCH[dt]) for x in local]
    out = [torch.full((b, t, *row), float("nan"), dtype=TORCH[dt], device="cuda") for _ in range(p)]
    usp.all_gather_rows(plan, dev, out=out)
    torch.cuda.synchronize()
    ref = orows.all_gather_rows(local, tr)
    for r in range(p):
        assert np.array_equal(device_bits(out[r]), ref[r]), f"rank {r}"
    plan.close()


def _draw(shape, dt, rng):
    x = rng.standard_normal(shape, dtype=np.float32)
    if dt == "bf16":
        bits = f32_to_bf16_bits(x)
        return bits, storage_to_f64(bits, "bf16")
    if dt == "fp16":
        h = x.astype(np.float16)
        return h.view(np.uint16), h.astype(np.float64)
    return x.view(np.uint32), x.astype(np.float64)


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}-T{c[1]}-P{c[2]}-row{'x'.join(map(str, c[3]))}-{c[4]}")
def test_reduce_scatter_rows_within_bound(usp, case):
    b, t, p, row, dt = case
    plan = _plan(usp, case)
    rng = np.random.default_rng(900 + p)
    drawn = [_draw((b, t, *row), dt, rng) for _ in range(p)]
    dev = [bits_to_device(bits).view(TORCH[dt]) for bits, _ in drawn]
    out = usp.reduce_scatter_rows(plan, dev)
    torch.cuda.synchronize()
    tr = plan.token_ranges
    exact = orows.reduce_scatter_rows([v for _, v in drawn], tr)
    mag = orows.reduce_scatter_rows([np.abs(v) for _, v in drawn], tr)
    for r in range(p):
        got = out[r].double().cpu().numpy()
        e = (p - 1) * 2.0 ** -24 * mag[r]
        tol = ROUND_REL[dt] * (np.abs(exact[r]) + e) + e + (2.0 ** -24 if dt == "fp16" else 0.0)
        err = np.abs(got - exact[r])
        assert np.all(err <= tol), f"rank {r}: worst excess {float(np.max(err - tol))}"
        if dt != "fp32":  # 16 spare fp32 bits: nearly every sum rounds like the exact one
            rounded = torch.from_numpy(exact[r]).to(TORCH[dt]).double().numpy()
            assert np.mean(got == rounded) > 0.99, f"rank {r}: {np.mean(got == rounded)} equal the rounded sum"
    plan.close()


@pytest.mark.parametrize("dt", ["bf16", "fp16", "fp32"])
def test_reduce_scatter_rows_integer_sums_bit_exact(usp, dt):
    b, t, h, d, p = 2, 45, 6, 8, 6
    plan = usp.Plan(b, t, h, d, p, dt, 0)
    rng = np.random.default_rng(17)
    ints = [rng.integers(-20, 21, size=(b, t, h, d)).astype(np.float64) for _ in range(p)]
    dev = [torch.from_numpy(x).to(TORCH[dt]).cuda() for x in ints]
    out = usp.reduce_scatter_rows(plan, dev)
    torch.cuda.synchronize()
    exact = orows.reduce_scatter_rows(ints, plan.token_ranges)
    for r in range(p):
        assert np.array_equal(out[r].double().cpu().numpy(), exact[r])
    plan.close()


def test_gather_then_reduce_scatter(usp):
    """AG followed by RS of the replicas gives P times each rank's rows."""
    plan = usp.Plan(1, 77, 4, 32, 4, "bf16", 0)
    local = [torch.randint(-8, 8, (1, t1 - t0, 4, 32), device="cuda").to(torch.bfloat16)
             for t0, t1 in plan.token_ranges]
    back = usp.reduce_scatter_rows(plan, usp.all_gather_rows(plan, local))
    torch.cuda.synchronize()
    for x, y in zip(local, back):
        assert torch.equal(y, 4 * x)
    plan.close()


def test_rows_reject_bad_tensors(usp):
    plan = usp.Plan(1, 20, 4, 8, 4, "bf16", 0)
    local = [torch.zeros((1, t1 - t0, 2, 8), dtype=torch.bfloat16, device="cuda") for t0, t1 in plan.token_ranges]
    with pytest.raises(usp.UspError):
        usp.all_gather_rows(plan, local[:3])
    with pytest.raises(usp.UspError):
        usp.reduce_scatter_rows(plan, local)  # local rows are not full-length partials
    full = [torch.zeros((1, 20, 2, 8), dtype=torch.float16, device="cuda") for _ in range(4)]
    with pytest.raises(usp.UspError):
        usp.reduce_scatter_rows(plan, full)  # fp16 partials on a bf16 plan
    plan.close()

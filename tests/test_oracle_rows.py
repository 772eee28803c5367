"""Pins for oracle.rows: brute force on tiny inputs, closed forms, adjointness,
the one-rank case and the page's argument checks."""

import numpy as np
import pytest

from oracle.partition import balanced_ranges
from oracle.rows import all_gather_rows, reduce_scatter_rows

SPLITS = [(10, 4), (7, 7), (9, 2), (13, 5), (5, 1), (33, 8)]


def _owner(t, token_ranges):
    for i, (start, stop) in enumerate(token_ranges):
        if start <= t < stop:
            return i, t - start
    raise AssertionError(t)


@pytest.mark.parametrize("total,world", SPLITS)
def test_all_gather_brute_force(total, world):
    tr = balanced_ranges(total, world)
    rng = np.random.default_rng(total * 31 + world)
    local = [rng.standard_normal((2, b - a, 3)) for a, b in tr]
    out = all_gather_rows(local, tr)
    assert len(out) == world
    for r in range(world):
        assert out[r].shape == (2, total, 3)
        for b in range(2):
            for t in range(total):
                i, k = _owner(t, tr)
                for c in range(3):
                    assert out[r][b, t, c] == local[i][b, k, c]


@pytest.mark.parametrize("total,world", SPLITS)
def test_reduce_scatter_brute_force(total, world):
    tr = balanced_ranges(total, world)
    rng = np.random.default_rng(total * 37 + world)
    partials = [rng.standard_normal((2, total, 2, 2)) for _ in range(world)]
    out = reduce_scatter_rows(partials, tr)
    for r, (start, stop) in enumerate(tr):
        assert out[r].shape == (2, stop - start, 2, 2)
        for b in range(2):
            for t in range(stop - start):
                for h in range(2):
                    for d in range(2):
                        s = 0.0
                        for i in range(world):
                            s += partials[i][b, start + t, h, d]
                        assert out[r][b, t, h, d] == s


def test_reduce_scatter_closed_form():
    """Partial i is the constant i + 1: every output element is P(P+1)/2."""
    tr = balanced_ranges(23, 6)
    partials = [np.full((1, 23, 4), i + 1, dtype=np.float32) for i in range(6)]
    for r, x in enumerate(reduce_scatter_rows(partials, tr)):
        assert x.shape == (1, tr[r][1] - tr[r][0], 4)
        assert np.all(x == 21.0)


def test_rows_keep_their_token_index():
    """Row t carries the value t: the gather puts every row back at its index,
    and the reduce-scatter of P copies gives P * t on the owner of t."""
    total, world = 19, 4
    tr = balanced_ranges(total, world)
    local = [np.arange(a, b, dtype=np.float64).reshape(1, -1, 1) for a, b in tr]
    for x in all_gather_rows(local, tr):
        np.testing.assert_array_equal(x[0, :, 0], np.arange(total))
    full = np.arange(total, dtype=np.float64).reshape(1, -1, 1)
    for (a, b), x in zip(tr, reduce_scatter_rows([full] * world, tr)):
        np.testing.assert_array_equal(x[0, :, 0], world * np.arange(a, b))


@pytest.mark.parametrize("total,world", SPLITS)
def test_reduce_scatter_is_adjoint_of_all_gather(total, world):
    """sum_r <RS(X)_r, y_r> == sum_i <X_i, AG(y)_i>: the two collectives are
    transposes of each other, which fails for any mismatched row index."""
    tr = balanced_ranges(total, world)
    rng = np.random.default_rng(total + 101 * world)
    x = [rng.standard_normal((3, total, 5)) for _ in range(world)]
    y = [rng.standard_normal((3, b - a, 5)) for a, b in tr]
    lhs = sum(float(np.sum(a * b)) for a, b in zip(reduce_scatter_rows(x, tr), y))
    rhs = sum(float(np.sum(a * b)) for a, b in zip(x, all_gather_rows(y, tr)))
    assert abs(lhs - rhs) <= 1e-10 * max(1.0, abs(lhs))


def test_one_rank_is_a_copy():
    x = np.random.default_rng(5).standard_normal((2, 6, 3))
    tr = balanced_ranges(6, 1)
    g = all_gather_rows([x], tr)[0]
    np.testing.assert_array_equal(g, x)
    assert g is not x
    s = reduce_scatter_rows([x], tr)[0]
    np.testing.assert_array_equal(s, x)


def test_gather_then_reduce_scatter_scales_by_world():
    """AG then RS of the same replicated rows gives P times each rank's rows."""
    tr = balanced_ranges(17, 5)
    rng = np.random.default_rng(9)
    local = [rng.integers(-50, 50, size=(2, b - a, 3)).astype(np.float64) for a, b in tr]
    back = reduce_scatter_rows(all_gather_rows(local, tr), tr)
    for x, y in zip(local, back):
        np.testing.assert_array_equal(y, 5 * x)


def test_wrong_row_counts_raise():
    tr = balanced_ranges(10, 4)  # 3, 3, 2, 2
    with pytest.raises(ValueError):
        all_gather_rows([np.zeros((1, 3, 2))] * 4, tr)
    with pytest.raises(ValueError):
        reduce_scatter_rows([np.zeros((1, 9, 2))] * 4, tr)
    with pytest.raises(ValueError):
        reduce_scatter_rows([np.zeros((1, 10, 2))] * 3, tr)

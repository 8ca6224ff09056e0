"""Pins of the oracle's dense projection (a linear layer, y = x w^T) against
facts that do not come from the oracle itself: exact integer arithmetic done
with Python integers, a selection weight whose output is known column by
column, and the stacking order of the input projection's four outputs."""

import numpy as np
import pytest

import oracle
from linear_attention_recurrence_deltanet_b200 import inputs as gi


def test_project_matches_exact_integer_products():
    """Small integers make every product and sum exact in float64, so the
    result must equal the same sums done with Python integers.  M, K and N
    all differ, so a transposed operand or a swapped index fails."""
    rng = np.random.default_rng(11)
    M, K, N = 5, 7, 3
    x = rng.integers(-9, 10, (M, K))
    w = rng.integers(-9, 10, (N, K))
    want = [[sum(int(x[r, k]) * int(w[c, k]) for k in range(K)) for c in range(N)] for r in range(M)]
    got = oracle.project(x.astype(np.float32), w.astype(np.float32))
    assert got.shape == (M, N)
    assert np.array_equal(got, np.array(want, np.float64))


def test_project_row_sampling():
    rng = np.random.default_rng(12)
    x = rng.standard_normal((9, 16)).astype(np.float32)
    w = rng.standard_normal((4, 16)).astype(np.float32)
    full = oracle.project(x, w)
    rows = [8, 0, 3]
    assert np.array_equal(oracle.project(x, w, rows=rows), full[rows])


def test_project_in_split_follows_weight_row_order():
    """A weight whose row c picks input feature p(c) turns the projection into
    a column gather; qkv, z, a and b must then hold exactly the features the
    rows stacked in that order select."""
    geo = gi.Geometry(num_k_heads=2, num_v_heads=4, head_k_dim=8, head_v_dim=8)
    C, V, H = geo.conv_dim, geo.value_dim, geo.num_v_heads
    n = C + V + 2 * H
    hidden = n + 3
    perm = np.random.default_rng(13).permutation(hidden)[:n]
    w = np.zeros((n, hidden), np.float32)
    w[np.arange(n), perm] = 1.0
    x = np.random.default_rng(14).standard_normal((6, hidden)).astype(np.float32)
    qkv, z, a, b = oracle.split_projection(geo, oracle.project(x, w))
    assert qkv.shape == (6, C) and z.shape == (6, V) and a.shape == (6, H) and b.shape == (6, H)
    assert np.array_equal(qkv, x[:, perm[:C]].astype(np.float64))
    assert np.array_equal(z, x[:, perm[C:C + V]].astype(np.float64))
    assert np.array_equal(a, x[:, perm[C + V:C + V + H]].astype(np.float64))
    assert np.array_equal(b, x[:, perm[C + V + H:]].astype(np.float64))


@pytest.mark.parametrize("K", [1, 64, 333])
def test_project_is_linear_in_the_weight(K):
    rng = np.random.default_rng(15)
    x = rng.integers(-4, 5, (3, K)).astype(np.float32)
    w1 = rng.integers(-4, 5, (5, K)).astype(np.float32)
    w2 = rng.integers(-4, 5, (5, K)).astype(np.float32)
    assert np.array_equal(oracle.project(x, w1 + w2), oracle.project(x, w1) + oracle.project(x, w2))

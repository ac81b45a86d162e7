"""Pins for the adaptive-rank pieces of the oracle (CPU): the kurtosis of a
weight matrix and the split of a rank budget by score.

"MiLo: Efficient Quantized MoE Inference with Mixture of Low-Rank
Compensators", section "MiLo Algorithm: Mixture of Low-Rank Compensators",
adaptive rank selection: higher kurtosis (strategy 3) or higher activation
frequency (strategy 2) gets a higher rank.  The budget split is a reading:
shares proportional to the scores in units of 8 ranks, capped, largest
remainder for the leftover units.
"""
import numpy as np
import pytest
from scipy import stats

import oracle
import workloads as wl


def _bits(a):
    return np.asarray(a, np.float32).astype(np.float16).view(np.uint16)


def test_kurtosis_matches_scipy():
    rng = np.random.default_rng(61)
    for W in (wl.gen_weight(rng, 64, 256), _bits(rng.standard_normal((32, 128))),
              _bits(rng.laplace(size=(16, 128)))):
        ref = stats.kurtosis(W.view(np.float16).astype(np.float64).ravel(), fisher=False)
        assert abs(oracle.kurtosis(W) - ref) <= 1e-12 * ref


def test_kurtosis_closed_forms():
    assert oracle.kurtosis(_bits([0.5, -0.5] * 64)) == pytest.approx(1.0, abs=1e-15)   # two-point: 1
    assert oracle.kurtosis(_bits([0.25] * 128)) == 0.0                                  # constant
    # one outlier of size a among n zeros: m4 / m2^2 = n - 3 + 3/n ... exactly (n^2 - 3n + 3) / (n - 1)
    n = 128
    x = np.zeros(n)
    x[0] = 2.0
    assert oracle.kurtosis(_bits(x)) == pytest.approx((n * n - 3 * n + 3) / (n - 1), rel=1e-12)


def test_assign_ranks_hand_examples():
    # budget 4 * 16 = 64 ranks = 8 units; shares 8 * (5, 3, 3, 1) / 12 = 3.33, 2, 2, 0.67;
    # floors 3, 2, 2, 0 use 7 units, the eighth goes to the largest fraction (0.67)
    assert oracle.assign_ranks([5, 3, 3, 1], 16) == [24, 16, 16, 8]
    # exact proportions: 12 units over scores 1, 1, 2
    assert oracle.assign_ranks([1, 1, 2], 32) == [24, 24, 48]
    # cap: 12 units, 100/102 of them would exceed 8 -> 8 (64 ranks), the other 4 split evenly
    assert oracle.assign_ranks([100, 1, 1], 32) == [64, 16, 16]
    # all zero or negative scores -> equal shares; leftover by lower index
    assert oracle.assign_ranks([0, 0, 0], 16) == [16, 16, 16]
    assert oracle.assign_ranks([-1, -2, -3, -4], 12) == [16, 16, 8, 8]
    # 3 units over scores 1, 3, 2: shares 0.5, 1.5, 1; floors 0, 1, 1; the
    # leftover unit: fractions 0.5 and 0.5 tie, the higher score (3) takes it
    assert oracle.assign_ranks([1, 3, 2], 8) == [0, 16, 8]
    # a budget below one unit per matrix goes to the highest share first
    assert oracle.assign_ranks([1, 3, 2], 4) == [0, 8, 0]
    # one positive score, capped: 12 units, cap 4; the other three share 8 units
    # equally (2.67 each), floors 2 + 2 + 2, the two leftover units by lower index
    # (equal fractions, equal clipped scores 0)
    assert oracle.assign_ranks([-1, 5, 0, -2], 24, max_rank=32) == [24, 32, 24, 16]


def test_assign_ranks_properties():
    rng = np.random.default_rng(62)
    for _ in range(500):
        n = int(rng.integers(1, 30))
        sc = (rng.standard_normal(n) * rng.choice([0.1, 1.0, 50.0]) + rng.choice([0.0, 3.0])).tolist()
        avg = int(rng.integers(0, 72))
        mx = int(rng.choice([8, 32, 64]))
        r = oracle.assign_ranks(sc, avg, mx)
        assert all(x % 8 == 0 and 0 <= x <= mx for x in r)
        assert sum(r) == 8 * min(n * avg // 8, n * (mx // 8))          # the whole budget is used
        for i in range(n):
            for j in range(n):
                if max(sc[i], 0) > max(sc[j], 0):
                    assert r[i] >= r[j]                                 # monotone in the score
        assert oracle.assign_ranks([2 * x for x in sc], avg, mx) == r  # invariant to scaling by 2

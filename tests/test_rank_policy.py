"""Host logic of the library: milo_assign_ranks (a host function of the C
ABI) against the oracle's budget split, and its argument checks.  No GPU."""
import numpy as np
import pytest

import oracle


@pytest.fixture(scope="module")
def milo():
    from int3_gemm_rank_b200 import build
    build.build()
    import int3_gemm_rank_b200 as m
    return m


def test_assign_ranks_matches_oracle(milo):
    rng = np.random.default_rng(63)
    for _ in range(1000):
        n = int(rng.integers(1, 50))
        sc = (rng.standard_normal(n) * rng.choice([0.01, 1.0, 100.0]) + rng.choice([0.0, 3.0])).tolist()
        if rng.random() < 0.2:
            sc = [float(round(x)) for x in sc]                 # ties
        avg, mx = int(rng.integers(0, 80)), int(rng.choice([0, 8, 24, 64]))
        assert milo.milo_assign_ranks(sc, avg, mx) == oracle.assign_ranks(sc, avg, mx)


def test_assign_ranks_rejects_bad_arguments(milo):
    with pytest.raises(milo.MiloError):
        milo.milo_assign_ranks([1.0, float("nan")], 16)
    with pytest.raises(milo.MiloError):
        milo.milo_assign_ranks([1.0], 16, max_rank=12)
    with pytest.raises(milo.MiloError):
        milo.milo_assign_ranks([1.0], 16, max_rank=72)
    with pytest.raises(milo.MiloError):
        milo.milo_assign_ranks([], 16)

"""GPU parity of the kurtosis reduction (adaptive compensator ranks) through
the C ABI, against the oracle's fp64 centred moments.

"MiLo: Efficient Quantized MoE Inference with Mixture of Low-Rank
Compensators", adaptive rank selection, strategy 3 (kurtosis).  Both sides are
fp64; the GPU sums raw power sums over a fixed grid and converts them to
central moments, the oracle centres first, so they agree to about 1e-12
relative for weight-like data (mean near zero); the bar is 1e-9.
"""
import numpy as np
import pytest

import oracle
import workloads as wl
from parity_util import f16_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def milo():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import int3_gemm_rank_b200 as m
    m.lib()
    return m


@pytest.mark.parametrize("shape", [(1, 128), (130, 384), (1001,), (7, 5), (14336, 4096)])
def test_kurtosis_matches_oracle(milo, shape):
    rng = np.random.default_rng(int(np.prod(shape)) % 1000)
    if len(shape) == 2 and shape[1] % 64 == 0:
        W = wl.gen_weight(rng, *shape)
    else:
        W = wl.gen_normal_f16(rng, shape, 0.02)
    st = milo.new_status()
    k = milo.milo_kurtosis(f16_dev(W), dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = oracle.kurtosis(W)
    assert abs(float(k.item()) - ref) <= 1e-9 * ref


def test_kurtosis_deterministic_and_flags_nonfinite(milo):
    W = wl.gen_weight(np.random.default_rng(64), 256, 512)
    a = milo.milo_kurtosis(f16_dev(W))
    b = milo.milo_kurtosis(f16_dev(W))
    assert torch.equal(a, b)
    W[3, 7] = 0x7E00
    st = milo.new_status()
    milo.milo_kurtosis(f16_dev(W), dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & milo.MILO_DEV_NONFINITE


def test_kurtosis_of_a_constant_matrix_is_zero(milo):
    W = np.full((64, 128), 0x3800, np.uint16)
    assert float(milo.milo_kurtosis(f16_dev(W)).item()) == 0.0


def test_ranks_from_kurtosis_match_the_oracle(milo):
    """Strategy 3 end to end: kurtosis of eight matrices with different
    outlier weights on the GPU, ranks from the library's budget split; the
    oracle's kurtosis and split give the same ranks, and heavier tails get
    more rank."""
    rng = np.random.default_rng(65)
    mats = [wl.gen_weight(rng, 256, 512, outlier_mul=s) for s in (1, 2, 4, 8, 12, 16, 20, 30)]
    kg = [float(milo.milo_kurtosis(f16_dev(W)).item()) for W in mats]
    kr = [oracle.kurtosis(W) for W in mats]
    ranks = milo.milo_assign_ranks(kg, 24)
    assert ranks == oracle.assign_ranks(kr, 24)
    assert ranks == sorted(ranks) and ranks[0] < ranks[-1]

"""Failure detection on the GPU without a fault: a bounded wait that runs out.

The kernels wait on mbarriers with an iteration limit; past it they flag
MILO_DEV_TIMEOUT in the caller's status word and return.  The self-test
entry point makes such a wait run out (a barrier that nothing completes);
the host reads the flag, and the same context then runs a checked call.
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


def test_bounded_wait_times_out_and_the_context_stays_usable(milo):
    import ctypes as C
    st = milo.new_status()
    s = torch.cuda.current_stream()
    assert milo.lib().milo_selftest_wait_timeout(C.c_void_p(st.data_ptr()), C.c_void_p(s.cuda_stream)) == 0
    torch.cuda.synchronize()
    assert int(st.item()) & milo.MILO_DEV_TIMEOUT
    # the context still works: a packing call matches the oracle bit for bit
    W = wl.gen_weight(np.random.default_rng(70), 64, 256)
    blob = milo.milo_pack(f16_dev(W))
    q, sc, z, _ = oracle.quantize(W)
    assert np.array_equal(blob.cpu().numpy(), oracle.tile_pack(oracle.pack(q), sc, z, 256))

"""milo_grouped_linear_noalloc: the grouped linear for callers that cannot
allocate device memory (for example code behind a plugin or custom-operator
interface that is handed only its input and output buffers, or a path that
must not call cudaMalloc because it can synchronise the device).  Its scratch
is a buffer built into the library instead of a caller workspace.

The test calls it through the C ABI twice in a row and checks each result
against the ordinary entry point, milo_grouped_linear, with a caller-provided
workspace.  Both run the same kernels with the same launch plan, so the
results must be identical bit for bit; a stale value left in the shared
buffer by the previous call (for example a slice counter of the compensator's
K-split down-projection, which the single-expert case uses) would show.  This
file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes as C

import numpy as np
import pytest

import workloads as wl
from parity_util import act_dev, f16_dev, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def milo():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import int3_gemm_rank_b200 as m
    m.lib()
    return m


def _lin(milo, projs):
    return milo.GroupedLinear([milo.QWeight.quantize(f16_dev(p.W), f16_dev(p.U) if p.rank else None,
                                                     f16_dev(p.V) if p.rank else None) for p in projs])


def _call_noalloc(milo, lin, x, r, k, T, out_dtype=torch.float32):
    """Direct C-ABI call of milo_grouped_linear_noalloc."""
    y = torch.empty((T * k, lin.cs.N), dtype=out_dtype, device="cuda")
    st = milo.new_status()
    status = milo.lib().milo_grouped_linear_noalloc(
        C.byref(lin.cs), C.c_void_p(x.data_ptr()), milo._dt(x), T, k,
        C.c_void_p(r["offsets"].data_ptr()), C.c_void_p(r["perm"].data_ptr()),
        C.c_void_p(y.data_ptr()), milo._dt(y), C.c_void_p(st.data_ptr()),
        C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert status == milo.MILO_OK, milo.lib().milo_last_error()
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return y


@pytest.mark.parametrize("case", ["single_expert_decode", "three_experts_top2"])
def test_noalloc_matches_workspace_entry_point_on_two_calls(milo, case):
    if case == "single_expert_decode":
        x0, P = wl.single(seed_workload="t_noalloc1")
        projs, T, k, E, dt = [P], 1, 1, 1, "f16"
        xs = [x0, wl.gen_activations(np.random.default_rng(21), 1, 1024, "f16")]
        ids = [np.zeros((1, 1), np.int32)] * 2
    else:
        projs = [wl.make_projection("t_noalloc2", "w", e, 256, 512, r) for e, r in enumerate((16, 0, 8))]
        T, k, E, dt = 7, 2, 3, "bf16"
        rng = np.random.default_rng(22)
        xs = [wl.gen_activations(rng, T, 512, dt) for _ in range(2)]
        ids = [np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32) for _ in range(2)]
    lin = _lin(milo, projs)
    for call in range(2):
        x = act_dev(xs[call], dt)
        r = milo.milo_route(None, k, False, E=E, ids=to_dev(ids[call]))
        out = torch.float32 if call == 0 else torch.float16
        y_ref = lin(x, r["offsets"], r["perm"], k=k, out_dtype=out)
        y = _call_noalloc(milo, lin, x, r, k, T, out_dtype=out)
        assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16)), (case, call)


def test_noalloc_rejects_calls_beyond_its_buffer(milo):
    projs = [wl.make_projection("t_noalloc3", "w", 0, 4096, 1024, 0)]
    lin = _lin(milo, projs)
    T = 4096
    need = lin.workspace_bytes(T, 1)
    L = milo.lib()
    x = torch.zeros((T, 1024), dtype=torch.float16, device="cuda")
    y = torch.empty((T, 4096), dtype=torch.float32, device="cuda")
    off = torch.tensor([0, T], dtype=torch.int32, device="cuda")
    status = L.milo_grouped_linear_noalloc(C.byref(lin.cs), C.c_void_p(x.data_ptr()), milo.MILO_F16, T, 1,
                                           C.c_void_p(off.data_ptr()), None, C.c_void_p(y.data_ptr()),
                                           milo.MILO_F32, None,
                                           C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert need > 16 * 1024 * 1024
    assert status == milo.MILO_ERR_WORKSPACE
    assert b"scratch" in L.milo_last_error()

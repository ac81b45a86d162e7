"""GPU parity at activation scales far from 1.

The GEMMs take FP16 activations ("MiLo Kernel: Efficient Int3 Quantized GEMM
Backend": int3 weights times FP16 activations).  Before rounding an
activation row to fp16 the kernels multiply it by the power of two 2^a that
brings its largest magnitude into [1, 2), and multiply the row's result by
2^-a; the int3 fields' own powers of two are applied upwards.  So the results
must stay within REL_TOL of the oracle whatever the scale of the rows: tiny
inputs (fp16 subnormals, bf16 values below the fp16 range), inputs beyond the
fp16 range (bf16), and a SwiGLU output h small enough that, multiplied by
the largest field factor, it would become an fp16 subnormal.

References: the oracle computes in fp64 and takes x exactly, so for bf16 rows
scaled by 2^a (exact in bf16) its result is exactly 2^a times its result on
the unscaled rows -- that scaled result is the reference.  Where the scaled
input is not exact (fp16 subnormals) or the layer is not linear (SwiGLU), the
oracle runs on the scaled bits themselves.  Both GEMM kernels are checked.
"""
import numpy as np
import pytest

import oracle
import workloads as wl
from parity_util import REL_TOL, act_dev, act_f64, f16_dev, rel_err, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def milo():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import int3_gemm_rank_b200 as m
    m.lib()
    return m


@pytest.fixture(params=["mma", "tc"])
def gemm_path(request, milo):
    milo.milo_set_gemm_path(request.param)
    yield request.param
    milo.milo_set_gemm_path("auto")


def scaled_bits(bits: np.ndarray, dtype: str, a: int) -> np.ndarray:
    """Activation bits times 2^a, rounded back to the same format."""
    f = act_f64(bits, dtype).astype(np.float32) * np.float32(2.0 ** a)
    return wl.f32_to_bf16_bits(f) if dtype == "bf16" else wl.f32_to_f16_bits(f)


def _linear(milo, projs):
    gpu = [milo.QWeight.quantize(f16_dev(p.W), f16_dev(p.U) if p.rank else None,
                                 f16_dev(p.V) if p.rank else None) for p in projs]
    ref = [oracle.quantize_projection(p.W, p.U, p.V) for p in projs]
    return milo.GroupedLinear(gpu), ref


def _linear_ref(ref, X, ids, k, n):
    y = np.zeros((X.shape[0] * k, n))
    flat = ids.reshape(-1)
    for e in range(len(ref)):
        rows = np.flatnonzero(flat == e)
        if rows.size:
            y[rows] = oracle.linear(X[rows // k], ref[e])
    return y


def _run_linear(milo, lin, x_bits, dt, ids, k, E):
    r = milo.milo_route(None, k, False, E=E, ids=to_dev(ids.astype(np.int32)))
    st = milo.new_status()
    y = lin(act_dev(x_bits, dt), r["offsets"], r["perm"], k=k, out_dtype=torch.float32, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return y.cpu().numpy()


@pytest.mark.parametrize("a", [-10, -14, -24, 12, 20])
def test_single_expert_bf16_rows_scaled_by_powers_of_two(milo, gemm_path, a):
    """The single-expert decode shape (1024 x 1024, rank 16) with bf16 rows
    x 2^a: 2^-24 lies wholly below the fp16 range, 2^20 wholly above it."""
    _, P = wl.single(seed_workload="t_scale1")
    x = wl.gen_activations(np.random.default_rng(71), 3, 1024, "bf16")
    lin, ref = _linear(milo, [P])
    ids = np.zeros((3, 1), np.int32)
    y_ref = (2.0 ** a) * _linear_ref(ref, act_f64(x, "bf16"), ids, 1, 1024)
    y = _run_linear(milo, lin, scaled_bits(x, "bf16", a), "bf16", ids, 1, 1)
    err = rel_err(y, y_ref)
    assert err <= REL_TOL, (a, err)


@pytest.mark.parametrize("a", [-10, -14])
def test_single_expert_fp16_small_rows(milo, gemm_path, a):
    """fp16 rows x 2^-10 and x 2^-14: most values are fp16 subnormals, which the
    kernels must take exactly; the oracle runs on the same bits."""
    x0, P = wl.single(seed_workload="t_scale2", T=2)
    x = scaled_bits(x0, "f16", a)
    assert (np.abs(act_f64(x, "f16")) < 2.0 ** -14).mean() > (0.5 if a == -14 else 0.0)
    lin, ref = _linear(milo, [P])
    ids = np.zeros((2, 1), np.int32)
    y_ref = _linear_ref(ref, act_f64(x, "f16"), ids, 1, 1024)
    y = _run_linear(milo, lin, x, "f16", ids, 1, 1)
    err = rel_err(y, y_ref)
    assert err <= REL_TOL, (a, err)


def test_rows_of_different_scales_in_one_tile(milo, gemm_path):
    """Rows of one expert's tile at scales 2^-20 ... 2^16: each row keeps its
    own scale (300 rows over 2 experts, ranks 8 and 40, K = 640)."""
    projs = [wl.make_projection("t_scale3", "w", e, 192, 640, r) for e, r in enumerate((8, 40))]
    lin, ref = _linear(milo, projs)
    T = 300
    x = wl.gen_activations(np.random.default_rng(72), T, 640, "bf16")
    exps = np.random.default_rng(73).integers(-20, 17, T)
    xs = np.stack([scaled_bits(x[i:i + 1], "bf16", int(exps[i]))[0] for i in range(T)])
    ids = np.random.default_rng(74).choice(2, size=(T, 1), p=[0.45, 0.55]).astype(np.int32)
    y_ref = _linear_ref(ref, act_f64(x, "bf16"), ids, 1, 192) * (2.0 ** exps)[:, None]
    y = _run_linear(milo, lin, xs, "bf16", ids, 1, 2)
    # per-row relative error: each row has its own scale
    worst = max(rel_err(y[i], y_ref[i]) for i in range(T))
    assert worst <= REL_TOL, worst


def _layer(milo, wk):
    experts, ref = [], []
    for e in range(wk.n_experts):
        d, r = {}, {}
        for name in ("w1", "w3", "w2"):
            P = wk.experts[e][name]
            d[name] = milo.QWeight.quantize(f16_dev(P.W), f16_dev(P.U) if P.rank else None,
                                            f16_dev(P.V) if P.rank else None)
            r[name] = oracle.quantize_projection(P.W, P.U, P.V)
        experts.append(d)
        ref.append(r)
    return milo.MoELayer(experts, wk.n_routed, wk.n_shared, wk.top_k), ref


def _layer_check(milo, wk):
    layer, ref = _layer(milo, wk)
    st = milo.new_status()
    r = milo.milo_route(f16_dev(wk.logits), wk.top_k, wk.renorm, dev_status=st)
    y = layer(act_dev(wk.x, wk.x_dtype), r, out_dtype=torch.float32, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ids, w, _, _, inv, _ = oracle.route(wk.logits, wk.top_k, wk.renorm)
    y_ref, h_ref, st_ref = oracle.moe_forward(wk.x, wk.x_dtype == "bf16", ids, w, ref, wk.n_routed,
                                              wk.n_shared, wk.hidden, wk.inter, want_h=True)
    assert st_ref == 0
    err = rel_err(y.cpu().numpy(), y_ref)
    assert err <= REL_TOL, err
    h = layer.h_view(wk.T).cpu().numpy().view(np.uint16)
    Tk = wk.T * wk.top_k
    h_gpu = np.concatenate([h[inv], h[Tk:]]).view(np.float16).astype(np.float64)
    h64 = h_ref.view(np.float16).astype(np.float64)
    # h is fp16 on both sides, each rounding its own silu(a) b (the oracle's
    # in fp64): every element within REL_TOL of the layer's scale, or one
    # fp16 ulp apart (for subnormal h one ulp, 2^-24, can exceed REL_TOL)
    rms = float(np.sqrt(np.mean(h64 ** 2)))
    ulp = np.spacing(np.abs(h_ref.view(np.float16))).astype(np.float64)
    bound = np.maximum(REL_TOL * np.maximum(np.abs(h64), rms), ulp)
    worst = float(np.max(np.abs(h_gpu - h64) / bound))
    assert worst <= 1.0, worst
    return h64


@pytest.mark.parametrize("a", [-8, 6])
def test_moe_layer_scaled_inputs(milo, gemm_path, a):
    """A small SwiGLU layer (shared expert, top-2, ranks 0-16) on bf16 inputs
    x 2^-8 and x 2^6 (at 2^8 the fp16 h overflows, by the layer's definition);
    the oracle runs on the scaled inputs."""
    wk = wl.small_moe("t_scale4", T=24, hidden=256, inter=384, n_routed=4, n_shared=1, top_k=2)
    wk.x = scaled_bits(wk.x, "bf16", a)
    _layer_check(milo, wk)


@pytest.mark.parametrize("a", [-8, -12])
def test_moe_layer_small_swiglu_output(milo, gemm_path, a):
    """The w3 projection W3 + U3 V3 scaled by 2^a (W3 and U3 each x 2^a) makes
    h = silu(x W1^T) (x W3^T) small: at 2^-12 nearly all of it is fp16
    subnormal, values whose products with the largest field factor 2^-6 would
    lose their low bits (or vanish) if the activations were scaled down
    instead of up."""
    wk = wl.small_moe("t_scale5", T=24, hidden=256, inter=384, n_routed=4, n_shared=1, top_k=2)
    for e in range(wk.n_experts):
        P = wk.experts[e]["w3"]
        P.W = scaled_bits(P.W, "f16", a)
        P.U = scaled_bits(P.U, "f16", a)
    h = _layer_check(milo, wk)
    med = float(np.median(np.abs(h[h != 0])))
    assert 2.0 ** -18 < med < 2.0 ** -9, med

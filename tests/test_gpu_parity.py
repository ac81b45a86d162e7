"""GPU parity through the C ABI: the sm_100a kernels of libmilo against the CPU
oracle on the same seeded inputs.

Bit-exact: packing (Q, scale, zero), the kernels' field extraction (unpack),
routing ids, offsets, perm and inv_perm.  Within REL_TOL: the routed weights,
the compensated grouped linear, the SwiGLU activations and the layer output.
Sizes here span several tiles with ragged tails; tests/test_gpu_fullsize.py
runs the workload shapes themselves.
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
    """Run a test on the mma.sync grouped GEMM (chosen for few rows per expert)
    and on the tcgen05 one (chosen for many)."""
    milo.milo_set_gemm_path(request.param)
    yield request.param
    milo.milo_set_gemm_path("auto")


def _status(st):
    torch.cuda.synchronize()
    return int(st.item())


# ---------------------------------------------------------------------------
# packing and extraction
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("N,K", [(1, 128), (48, 384), (208, 1024), (1024, 1024), (16, 14336), (130, 1408)])
def test_pack_bit_exact(milo, N, K):
    W = wl.gen_weight(np.random.default_rng(N * 7 + K), N, K)
    st = milo.new_status()
    blob = milo.milo_pack(f16_dev(W), dev_status=st)
    q_ref, s_ref, z_ref, st_ref = oracle.quantize(W)
    assert _status(st) == st_ref == 0
    assert np.array_equal(blob.cpu().numpy(), oracle.tile_pack(oracle.pack(q_ref), s_ref, z_ref, K))


def test_pack_degenerate_and_signed_zero_groups(milo):
    W = np.zeros((4, 128), np.float32)
    W[0] = 0.5                                   # constant group -> s = 1
    W[1, :64] = -0.0                             # all -0
    W[2] = np.linspace(-1e-7, 1e-7, 128)         # subnormal-range values
    W[3, :9] = [0, 7, 0.5, 1.5, 2.5, 3.5, 4.5, 5.5, 6.5]   # ties to even
    Wb = W.astype(np.float16).view(np.uint16)
    blob = milo.milo_pack(f16_dev(Wb))
    q_ref, s_ref, z_ref, _ = oracle.quantize(Wb)
    assert np.array_equal(blob.cpu().numpy(), oracle.tile_pack(oracle.pack(q_ref), s_ref, z_ref, 128))


def test_pack_flags_nonfinite(milo):
    W = wl.gen_weight(np.random.default_rng(3), 2, 128)
    W[1, 3] = 0x7E00   # NaN
    st = milo.new_status()
    milo.milo_pack(f16_dev(W), dev_status=st)
    assert _status(st) & milo.MILO_DEV_NONFINITE


@pytest.mark.parametrize("N,K", [(3, 128), (64, 1408), (5, 4096)])
def test_unpack_bit_exact(milo, N, K):
    q = np.random.default_rng(N + K).integers(0, 8, (N, K), dtype=np.uint8)
    G = K // 64
    blob = oracle.tile_pack(oracle.pack(q), np.zeros((G, N), np.uint16), np.zeros((G, N), np.uint16), K)
    codes = milo.milo_unpack(to_dev(blob), N, K)
    assert np.array_equal(codes.cpu().numpy(), q)


@pytest.mark.parametrize("N,K,mul", [(48, 384, 1.0), (130, 1408, 1.0), (64, 256, 2.0 ** -12), (16, 128, 2.0 ** 8)])
def test_dequantize_bit_exact(milo, N, K, mul):
    """milo_dequantize (the unfused baseline's first pass): fp16((q - z) s) for
    every weight, bit for bit against the oracle's fp64 dequantisation rounded
    by its own fp16 conversion; tiny weights (subnormal s) and large ones too."""
    W = wl.gen_weight(np.random.default_rng(N + K), N, K)
    W = wl.f32_to_f16_bits(wl.f16_bits_to_f32(W) * np.float32(mul))
    blob = milo.milo_pack(f16_dev(W))
    W_hat = milo.milo_dequantize(blob, N, K).cpu().numpy().view(np.uint16)
    q, s, z, _ = oracle.quantize(W)
    ref = oracle.d2h(oracle.dequant(q, s, z)).reshape(N, K)
    assert np.array_equal(W_hat, ref)


# ---------------------------------------------------------------------------
# routing
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("T,E,k,renorm,coarse", [
    (16, 8, 2, True, False), (64, 64, 6, False, False), (8192, 8, 2, True, False),
    (300, 8, 2, True, True), (33, 64, 6, False, True), (1, 4, 4, True, False),
    (2000, 256, 8, False, False)])
def test_route_bit_exact(milo, T, E, k, renorm, coarse):
    rng = np.random.default_rng(T * 31 + E)
    if coarse:   # many exact ties
        L = (rng.integers(-2, 3, (T, E)) * 0.5).astype(np.float16).view(np.uint16)
    else:
        L = wl.gen_normal_f16(rng, (T, E), 1.0)
    st = milo.new_status()
    r = milo.milo_route(f16_dev(L), k, renorm, dev_status=st)
    ids, w, off, perm, inv, st_ref = oracle.route(L, k, renorm)
    assert _status(st) == st_ref == 0
    assert np.array_equal(r["ids"].cpu().numpy(), ids)
    assert np.array_equal(r["offsets"].cpu().numpy(), off)
    assert np.array_equal(r["perm"].cpu().numpy(), perm)
    assert np.array_equal(r["inv_perm"].cpu().numpy(), inv)
    np.testing.assert_allclose(r["w"].cpu().numpy(), w, rtol=2e-6, atol=1e-7)


def test_route_ids_given_zipf_and_bad_ids(milo):
    ids = wl.gen_zipf_ids(np.random.default_rng(5), 1024, 8).reshape(-1, 1)
    r = milo.milo_route(None, 1, False, E=8, ids=to_dev(ids))
    off, perm, inv, _ = oracle.group(ids, 8)
    assert np.array_equal(r["offsets"].cpu().numpy(), off)
    assert np.array_equal(r["perm"].cpu().numpy(), perm)
    assert np.array_equal(r["inv_perm"].cpu().numpy(), inv)
    bad = np.array([[0, 3], [9, 1], [2, -1]], np.int32)
    st = milo.new_status()
    r = milo.milo_route(None, 2, False, E=4, ids=to_dev(bad), dev_status=st)
    off, perm, inv, st_ref = oracle.group(bad, 4)
    assert _status(st) & milo.MILO_DEV_BAD_EXPERT_ID and st_ref & oracle.BAD_EXPERT
    assert np.array_equal(r["offsets"].cpu().numpy(), off)
    assert np.array_equal(r["perm"].cpu().numpy()[:off[-1]], perm[:off[-1]])
    assert np.array_equal(r["inv_perm"].cpu().numpy(), inv)


def test_route_flags_nan_logits(milo):
    L = wl.gen_normal_f16(np.random.default_rng(6), (4, 8), 1.0)
    L[2, 5] = 0x7E00
    st = milo.new_status()
    milo.milo_route(f16_dev(L), 2, True, dev_status=st)
    assert _status(st) & milo.MILO_DEV_NONFINITE


# ---------------------------------------------------------------------------
# grouped linear with the compensator
# ---------------------------------------------------------------------------

def _linear_pair(milo, projs, lorc_int3=False):
    gpu = [milo.QWeight.quantize(f16_dev(p.W), f16_dev(p.U) if p.rank else None,
                                 f16_dev(p.V) if p.rank else None, lorc_int3=lorc_int3) for p in projs]
    ref = [oracle.quantize_projection(p.W, p.U, p.V, lorc_int3=lorc_int3) for p in projs]
    return milo.GroupedLinear(gpu), ref


def _linear_check(milo, projs, x_bits, x_dt, ids, k, out_dtypes=(torch.float32,), lorc_int3=False):
    lin, ref = _linear_pair(milo, projs, lorc_int3)
    E = len(projs)
    T = x_bits.shape[0]
    r = milo.milo_route(None, k, False, E=E, ids=to_dev(ids.astype(np.int32)))
    st = milo.new_status()
    x = act_dev(x_bits, x_dt)
    y = lin(x, r["offsets"], r["perm"], k=k, out_dtype=torch.float32, dev_status=st)
    assert _status(st) == 0
    X = act_f64(x_bits, x_dt)
    y_ref = np.zeros((T * k, projs[0].n))
    flat = ids.reshape(-1)
    for e in range(E):
        rows = np.flatnonzero(flat == e)
        if rows.size:
            y_ref[rows] = oracle.linear(X[rows // k], ref[e])
    err = rel_err(y.cpu().numpy(), y_ref)
    assert err <= REL_TOL, err
    y32 = y
    for dt in out_dtypes[1:]:
        yd = lin(x, r["offsets"], r["perm"], k=k, out_dtype=dt)
        assert torch.equal(yd.view(torch.int16), y32.to(dt).view(torch.int16))
    return err


def test_linear_single_expert_decode_rank16(milo, gemm_path):
    """1 token, W 1024x1024 with outliers, rank-16 compensator."""
    x, P = wl.single(seed_workload="t_single")
    _linear_check(milo, [P], x, "f16", np.zeros((1, 1), np.int32), 1,
                  (torch.float32, torch.float16, torch.bfloat16))


def test_linear_ragged_rows_multi_token_tiles(milo, gemm_path):
    """N = 208 (ragged last row tile), K = 384 (half-empty last K chunk),
    experts of rank 0 / 8 / 24, 53 tokens over 3 experts (one expert > 16 rows)."""
    projs = [wl.make_projection("t_rag", "w", e, 208, 384, r) for e, r in enumerate((0, 8, 24))]
    x = wl.gen_activations(np.random.default_rng(8), 53, 384, "bf16")
    ids = np.random.default_rng(9).choice(3, size=(53, 1), p=[0.1, 0.7, 0.2]).astype(np.int32)
    _linear_check(milo, projs, x, "bf16", ids, 1, (torch.float32, torch.float16))


def test_linear_top2_slots_and_idle_experts(milo, gemm_path):
    projs = [wl.make_projection("t_k2", "w", e, 256, 512, 16 * (e % 3)) for e in range(6)]
    x = wl.gen_activations(np.random.default_rng(10), 3, 512, "f16")
    ids = np.array([[4, 1], [1, 0], [4, 5]], np.int32)   # experts 2, 3 idle
    _linear_check(milo, projs, x, "f16", ids, 2)


def test_linear_all_rows_one_expert(milo, gemm_path):
    projs = [wl.make_projection("t_one", "w", e, 128, 256, 8) for e in range(4)]
    x = wl.gen_activations(np.random.default_rng(11), 70, 256, "bf16")
    _linear_check(milo, projs, x, "bf16", np.full((70, 1), 2, np.int32), 1)


def test_linear_many_rows_per_expert(milo, gemm_path):
    """300 rows over 2 experts (several 128-row tiles and a ragged one), N = 192
    (one and a half 128-row weight tiles), K = 640 (odd number of super-blocks),
    ranks 8 and 40."""
    projs = [wl.make_projection("t_many", "w", e, 192, 640, r) for e, r in enumerate((8, 40))]
    x = wl.gen_activations(np.random.default_rng(13), 300, 640, "bf16")
    ids = np.random.default_rng(14).choice(2, size=(300, 1), p=[0.55, 0.45]).astype(np.int32)
    _linear_check(milo, projs, x, "bf16", ids, 1, (torch.float32, torch.float16))


def test_linear_bad_ids_dropped_and_zero(milo, gemm_path):
    projs = [wl.make_projection("t_bad", "w", e, 128, 256, 0) for e in range(2)]
    lin, ref = _linear_pair(milo, projs)
    x_bits = wl.gen_activations(np.random.default_rng(12), 3, 256, "f16")
    ids = np.array([[0], [7], [1]], np.int32)
    st = milo.new_status()
    r = milo.milo_route(None, 1, False, E=2, ids=to_dev(ids), dev_status=st)
    y = lin(act_dev(x_bits, "f16"), r["offsets"], r["perm"], k=1, dev_status=st)
    assert _status(st) & milo.MILO_DEV_BAD_EXPERT_ID
    y = y.cpu().numpy()
    assert not y[1].any()
    X = act_f64(x_bits, "f16")
    assert rel_err(y[0], oracle.linear(X[:1], ref[0])[0]) <= REL_TOL
    assert rel_err(y[2], oracle.linear(X[2:], ref[1])[0]) <= REL_TOL


def test_linear_large_bf16_rows_and_fp16_output_range(milo):
    """bf16 activations of 1e6 (beyond fp16) are valid input: the f32 result
    matches the oracle; the same result requested as fp16 overflows, which
    sets FP16_RANGE."""
    projs = [wl.make_projection("t_rng", "w", 0, 128, 128, 0)]
    lin, ref = _linear_pair(milo, projs)
    x = wl.f32_to_bf16_bits(np.full((1, 128), 1.0e6, np.float32))
    r = milo.milo_route(None, 1, False, E=1, ids=to_dev(np.zeros((1, 1), np.int32)))
    st = milo.new_status()
    y = lin(act_dev(x, "bf16"), r["offsets"], r["perm"], k=1, dev_status=st)
    assert _status(st) == 0
    y_ref = oracle.linear(act_f64(x, "bf16"), ref[0])
    assert rel_err(y.cpu().numpy(), y_ref) <= REL_TOL
    assert np.abs(y_ref).max() > 65504
    lin(act_dev(x, "bf16"), r["offsets"], r["perm"], k=1, out_dtype=torch.float16, dev_status=st)
    assert _status(st) & milo.MILO_DEV_FP16_RANGE


def test_linear_rejects_bad_shapes(milo):
    W = torch.zeros((16, 100), dtype=torch.float16, device="cuda")
    with pytest.raises(milo.MiloError) as e:
        milo.milo_pack(W)
    assert e.value.status == milo.MILO_ERR_UNSUPPORTED_SHAPE


# ---------------------------------------------------------------------------
# full SwiGLU MoE layer (small shapes)
# ---------------------------------------------------------------------------

def gpu_layer(milo, wk, lorc_int3=False):
    experts = []
    for e in range(wk.n_experts):
        d = {}
        for name in ("w1", "w3", "w2"):
            P = wk.experts[e][name]
            d[name] = milo.QWeight.quantize(f16_dev(P.W), f16_dev(P.U) if P.rank else None,
                                            f16_dev(P.V) if P.rank else None, lorc_int3=lorc_int3)
        experts.append(d)
    return milo.MoELayer(experts, wk.n_routed, wk.n_shared, wk.top_k)


def oracle_layer(wk, lorc_int3=False):
    return [{name: oracle.quantize_projection(wk.experts[e][name].W, wk.experts[e][name].U,
                                              wk.experts[e][name].V, lorc_int3=lorc_int3)
             for name in ("w1", "w3", "w2")} for e in range(wk.n_experts)]


def run_layer_parity(milo, wk, check_h=True, out_dtypes=(torch.float32,), lorc_int3=False):
    layer = gpu_layer(milo, wk, lorc_int3)
    st = milo.new_status()
    r = milo.milo_route(f16_dev(wk.logits), wk.top_k, wk.renorm, dev_status=st)
    x = act_dev(wk.x, wk.x_dtype)
    y = layer(x, r, out_dtype=torch.float32, dev_status=st)
    assert _status(st) == 0
    ids, w, off, perm, inv, _ = oracle.route(wk.logits, wk.top_k, wk.renorm)
    assert np.array_equal(r["ids"].cpu().numpy(), ids)
    ref = oracle_layer(wk, lorc_int3)
    y_ref, h_ref, st_ref = oracle.moe_forward(wk.x, wk.x_dtype == "bf16", ids, w, ref, wk.n_routed,
                                              wk.n_shared, wk.hidden, wk.inter, want_h=True)
    assert st_ref == 0
    err = rel_err(y.cpu().numpy(), y_ref)
    assert err <= REL_TOL, err
    if check_h:
        h = layer.h_view(wk.T).cpu().numpy().view(np.uint16)
        Tk = wk.T * wk.top_k
        h_gpu = np.concatenate([h[inv], h[Tk:]]).view(np.float16).astype(np.float64)
        herr = rel_err(h_gpu, h_ref.view(np.float16).astype(np.float64))
        assert herr <= REL_TOL, herr
    for dt in out_dtypes[1:]:
        yd = layer(x, r, out_dtype=dt)
        assert torch.equal(yd.view(torch.int16), y.to(dt).view(torch.int16))
    return err


def test_moe_small_shared_expert(milo, gemm_path):
    wk = wl.small_moe("t_moe1", T=5, hidden=256, inter=384, n_routed=4, n_shared=1, top_k=2)
    run_layer_parity(milo, wk, out_dtypes=(torch.float32, torch.bfloat16, torch.float16))


def test_moe_small_no_compensator_full_softmax(milo, gemm_path):
    wk = wl.small_moe("t_moe2", T=19, hidden=384, inter=256, n_routed=6, n_shared=0, top_k=3,
                      renorm=False, rank_choices=(0,), x_dtype="f16")
    run_layer_parity(milo, wk)


def test_moe_small_many_tokens_per_expert(milo, gemm_path):
    wk = wl.small_moe("t_moe3", T=90, hidden=256, inter=512, n_routed=3, n_shared=2, top_k=1,
                      rank_choices=(8, 64))
    run_layer_parity(milo, wk)


def test_moe_zero_tokens_is_a_no_op(milo):
    wk = wl.small_moe("t_moe4", T=2, hidden=128, inter=128, n_routed=2, n_shared=0, top_k=1)
    layer = gpu_layer(milo, wk)
    x = torch.zeros((0, 128), dtype=torch.bfloat16, device="cuda")
    r = {"w": None, "offsets": torch.zeros(3, dtype=torch.int32, device="cuda"),
         "perm": None, "inv_perm": None}
    y = layer(x, r)
    assert y.shape == (0, 128)


@pytest.mark.parametrize("T", [6, 600])
def test_moe_forward_cuda_graph_replay_bit_exact(milo, T):
    """Route + layer captured in one CUDA graph (stream capture of every launch,
    the programmatic dependencies included) and replayed on new inputs gives
    the same bits as the eager calls on those inputs.  600 tokens take the
    multi-block top-k and, with 2 experts, the tcgen05 GEMM."""
    wk = wl.small_moe("t_graph", T=T, hidden=256, inter=384, n_routed=2 if T > 100 else 4, n_shared=1,
                      top_k=2, rank_choices=(0, 16))
    layer = gpu_layer(milo, wk)
    E, k = wk.n_routed, wk.top_k
    logits = f16_dev(wk.logits)
    x = act_dev(wk.x, wk.x_dtype)
    st = milo.new_status()
    ws = layer.workspace(T)
    route = {"ids": torch.empty((T, k), dtype=torch.int32, device="cuda"),
             "w": torch.empty((T, k), dtype=torch.float32, device="cuda"),
             "offsets": torch.empty(E + 1, dtype=torch.int32, device="cuda"),
             "perm": torch.empty(T * k, dtype=torch.int32, device="cuda"),
             "inv_perm": torch.empty(T * k, dtype=torch.int32, device="cuda")}
    y = torch.empty((T, wk.hidden), dtype=torch.float32, device="cuda")

    def step():
        milo.milo_route(logits, k, wk.renorm, dev_status=st, out=route)
        layer(x, route, out_dtype=torch.float32, dev_status=st, y=y, ws=ws)

    step()
    torch.cuda.synchronize()
    y_eager = y.clone()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    # new inputs in place, then replay
    rng = np.random.default_rng(5)
    logits.copy_(f16_dev(rng.standard_normal(wk.logits.shape).astype(np.float16).view(np.uint16)))
    x.copy_(act_dev(wl.gen_activations(rng, T, wk.hidden, wk.x_dtype), wk.x_dtype))
    y.zero_()
    g.replay()
    torch.cuda.synchronize()
    y_graph = y.clone()
    step()
    torch.cuda.synchronize()
    assert _status(st) == 0
    assert torch.equal(y_graph.view(torch.int32), y.view(torch.int32))
    assert not torch.equal(y_graph, y_eager)
    del g


# --- int3 compensators: U^T and V packed like weights ---------------------------

def test_linear_int3_compensator_decode_rows(milo, gemm_path):
    """Few rows per expert (K-sliced down-projection), N = 256, K = 640 (odd
    number of super-blocks), ranks 8 and 64."""
    projs = [wl.make_projection("t_l3a", "w", e, 256, 640, r) for e, r in enumerate((8, 64))]
    x = wl.gen_activations(np.random.default_rng(31), 6, 640, "bf16")
    ids = np.array([[0], [1], [1], [0], [1], [1]], np.int32)
    _linear_check(milo, projs, x, "bf16", ids, 1, lorc_int3=True)


def test_linear_int3_compensator_many_rows(milo, gemm_path):
    """300 rows over 2 experts (64-row down-projection tiles; the tcgen05 path
    takes them), N = 384 (three 128-row weight tiles), K = 512, ranks 16 and 40."""
    projs = [wl.make_projection("t_l3b", "w", e, 384, 512, r) for e, r in enumerate((16, 40))]
    x = wl.gen_activations(np.random.default_rng(32), 300, 512, "bf16")
    ids = np.random.default_rng(33).choice(2, size=(300, 1), p=[0.4, 0.6]).astype(np.int32)
    _linear_check(milo, projs, x, "bf16", ids, 1, (torch.float32, torch.float16), lorc_int3=True)


@pytest.mark.parametrize("lorc_int3", [False, True])
def test_linear_compensator_long_k(milo, gemm_path, lorc_int3):
    """K = 4224 (33 super-blocks): the compensator's down-projection runs in
    several K slices, the last one ragged (a half chunk, a partial stage);
    ranks 8, 40 (a partial 32-rank block) and 64; 5 rows over 3 experts."""
    projs = [wl.make_projection("t_longk", "w", e, 256, 4224, r) for e, r in enumerate((8, 40, 64))]
    x = wl.gen_activations(np.random.default_rng(34), 5, 4224, "bf16")
    ids = np.array([[2], [0], [1], [2], [2]], np.int32)
    _linear_check(milo, projs, x, "bf16", ids, 1, lorc_int3=lorc_int3)


def test_moe_int3_compensator(milo, gemm_path):
    wk = wl.small_moe("t_moe_l3", T=24, hidden=256, inter=384, n_routed=4, n_shared=1, top_k=2,
                      rank_choices=(0, 16, 32))
    run_layer_parity(milo, wk, lorc_int3=True)


def test_moe_int3_compensator_many_tokens(milo, gemm_path):
    wk = wl.small_moe("t_moe_l3b", T=200, hidden=256, inter=512, n_routed=2, n_shared=1, top_k=1,
                      rank_choices=(8, 64))
    run_layer_parity(milo, wk, lorc_int3=True)


def test_int3_compensator_needs_n_multiple_of_128(milo):
    P = wl.make_projection("t_l3c", "w", 0, 192, 256, 8)
    w = milo.QWeight.quantize(f16_dev(P.W), f16_dev(P.U), f16_dev(P.V))
    w.lorc_int3 = True     # fp16 factors declared int3 on an N the format cannot take
    with pytest.raises(milo.MiloError) as e:
        milo.GroupedLinear([w])
    assert e.value.status == milo.MILO_ERR_UNSUPPORTED_SHAPE

"""GPU parity of the offline MiLo quantiser (milo_hqq_pack, milo_quantize_lorc)
against the oracle, through the C ABI.

"MiLo: Efficient Quantized MoE Inference with Mixture of Low-Rank
Compensators", section "MiLo Algorithm: Mixture of Low-Rank Compensators".

Bit-exact: HQQ codes, scales and zeros (the blob), and the fp32 residual, for
the same fp32 target (both sides decide the codes in fp32 in the same order).
Within tolerance: the compensator product U V against the oracle's fp64
subspace iteration on the same residual and random test matrix, and the
per-round errors.  Tolerance derivation: the GPU forms the sketch products in
fp32 (relative error about 1e-6 per product over reductions of up to 14336
terms) and the Gram, Cholesky and Jacobi steps in fp64; the basis spans the
same subspace, and the top-r Ritz projector moves by that perturbation over
the relative gap of the Ritz values at r (about 1e-2 for noise-like residuals
with 2r sketch columns), so U V agrees to about 1e-4; the fp16 rounding of U
and V (2^-11 relative per entry) is shared.  U V is compared at 2e-3 of its
norm (the same bar as the forward path), the errors of rounds 0 and 1 at
1e-3, those of later rounds (which quantise slightly different targets on the
two sides) at 5e-3.
"""
import numpy as np
import pytest

import oracle
import workloads as wl
from parity_util import f16_dev, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

UV_TOL = 2e-3
ERR_TOL = 1e-3
LATE_ROUND_TOL = 5e-3


@pytest.fixture(scope="module")
def milo():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import int3_gemm_rank_b200 as m
    m.lib()
    return m


def _status(st):
    torch.cuda.synchronize()
    return int(st.item())


def _blob_ref(q, s, z, K):
    return oracle.tile_pack(oracle.pack(q), s, z, K)


def _f16(bits):
    return np.asarray(bits).view(np.float16).astype(np.float64)


@pytest.mark.parametrize("N,K,iters", [(1, 128, 20), (150, 384, 20), (64, 1408, 5), (200, 256, 0)])
def test_hqq_pack_bit_exact(milo, N, K, iters):
    W = wl.gen_weight(np.random.default_rng(N + K), N, K)
    st = milo.new_status()
    blob, R = milo.milo_hqq_pack(f16_dev(W), iters=iters, residual=True, dev_status=st)
    q, s, z, st_ref = oracle.hqq(oracle._f16(W), iters)
    assert _status(st) == st_ref == 0
    assert np.array_equal(blob.cpu().numpy(), _blob_ref(q, s, z, K))
    assert np.array_equal(R.cpu().numpy().view(np.uint32), oracle.residual(W, q, s, z).view(np.uint32))


def test_hqq_pack_with_compensator_bit_exact(milo):
    rng = np.random.default_rng(51)
    N, K, r = 130, 512, 16
    W = wl.gen_weight(rng, N, K)
    U = wl.gen_normal_f16(rng, (N, r), 0.01)
    V = wl.gen_normal_f16(rng, (r, K), 0.01)
    blob, R = milo.milo_hqq_pack(f16_dev(W), f16_dev(U), f16_dev(V), residual=True)
    q, s, z, _ = oracle.hqq(oracle.lorc_target(W, U, V))
    assert np.array_equal(blob.cpu().numpy(), _blob_ref(q, s, z, K))
    assert np.array_equal(R.cpu().numpy().view(np.uint32), oracle.residual(W, q, s, z).view(np.uint32))


def test_hqq_one_iteration_is_milo_pack(milo):
    W = wl.gen_weight(np.random.default_rng(52), 96, 768)
    blob, _ = milo.milo_hqq_pack(f16_dev(W), iters=1)
    assert torch.equal(blob, milo.milo_pack(f16_dev(W)))


def test_hqq_pack_flags_nonfinite(milo):
    W = wl.gen_weight(np.random.default_rng(53), 3, 128)
    W[2, 70] = 0x7C00   # +inf
    st = milo.new_status()
    milo.milo_hqq_pack(f16_dev(W), dev_status=st)
    assert _status(st) & milo.MILO_DEV_NONFINITE


def _quantize(milo, W, r, rounds, omega, power_iters=2):
    p = milo.lorc_params(r, rounds=rounds, sketch=omega.shape[1] if r else 0, power_iters=power_iters)
    st = milo.new_status()
    qw, err = milo.milo_quantize_lorc(f16_dev(W), p, to_dev(omega.astype(np.float32)) if r else None,
                                      dev_status=st)
    assert _status(st) == 0
    return qw, err.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("N,K,r", [(192, 384, 16), (130, 256, 8), (64, 1024, 32)])
def test_quantize_lorc_first_round(milo, N, K, r):
    """Round 0: HQQ blob bit-exact; U V against the oracle's subspace iteration
    on the same residual and test matrix; the reported error."""
    rng = np.random.default_rng(N * 3 + r)
    W = wl.gen_weight(rng, N, K)
    om = rng.standard_normal((K, 2 * r)).astype(np.float32)
    qw, err = _quantize(milo, W, r, 0, om)
    q, s, z, _ = oracle.hqq(oracle._f16(W))
    assert np.array_equal(qw.packed.cpu().numpy(), _blob_ref(q, s, z, K))
    R = oracle.residual(W, q, s, z)
    U, V = oracle.rsvd(R, r, om, 2)
    uv = _f16(qw.U.cpu().numpy().view(np.uint16)) @ _f16(qw.V.cpu().numpy().view(np.uint16))
    assert np.linalg.norm(uv - U @ V) <= UV_TOL * np.linalg.norm(U @ V)
    E = R.astype(np.float64) - uv
    assert abs(err[0] - np.linalg.norm(E)) <= 1e-5 * err[0]
    _, _, opt = oracle.svd_truncated(R, r)
    assert opt * (1 - 1e-6) <= err[0] <= 1.03 * opt


def test_quantize_lorc_rounds_track_the_oracle(milo):
    rng = np.random.default_rng(54)
    N, K, r, rounds = 128, 256, 16, 3
    W = wl.gen_weight(rng, N, K)
    om = rng.standard_normal((K, 2 * r)).astype(np.float32)
    qw, err = _quantize(milo, W, r, rounds, om)
    ref = oracle.quantize_lorc(W, r, rounds, om)
    assert err.shape == (rounds + 1,)
    # Rounds 0 and 1 quantise the same targets on both sides (W, then W minus a
    # compensator that agrees to fp16 rounding); from refinement round 2 on, a code decided
    # differently near a rounding boundary moves its group's zero-point fit, so
    # the two runs agree only statistically.
    assert np.all(np.abs(err[:2] - ref["err"][:2]) <= ERR_TOL * ref["err"][:2])
    assert np.all(np.abs(err[2:] - ref["err"][2:]) <= LATE_ROUND_TOL * ref["err"][2:])
    assert np.all(np.diff(err) < 0)
    # the kept round is the last (lowest error); its pieces reproduce its error
    uv = _f16(qw.U.cpu().numpy().view(np.uint16)) @ _f16(qw.V.cpu().numpy().view(np.uint16))
    blob = qw.packed.cpu().numpy()
    # scales and zeros straight from the blob: dequantise through the oracle
    qg, sg, zg = _unblob(blob, N, K)
    E = oracle.residual(W, qg, sg, zg).astype(np.float64) - uv
    assert abs(np.linalg.norm(E) - err.min()) <= 1e-5 * err.min()


def _unblob(blob, N, K, rows=None):
    """Codes [len(rows), K] and scales, zeros [K/64, len(rows)] read back from a
    blob (layout of milo.h), for the given rows or all N."""
    rows = np.arange(N) if rows is None else np.asarray(rows)
    SB = K // 128
    q = np.zeros((len(rows), K), np.uint8)
    s = np.zeros((K // 64, len(rows)), np.uint16)
    z = np.zeros((K // 64, len(rows)), np.uint16)
    for i, n in enumerate(rows):
        t, rr = divmod(int(n), 64)
        for b in range(SB):
            base = (t * SB + b) * 3584
            words = blob[base: base + 3072].view(np.uint32).reshape(64, 12)[rr]
            q[i, 128 * b: 128 * b + 128] = oracle.unpack(words.reshape(1, 12), 128)[0]
            groups = blob[base + 3072: base + 3584].view(np.uint16)
            for h in range(2):
                o = h * 128 + ((rr // 16) * 8 + rr % 8) * 4 + ((rr % 16) // 8) * 2
                s[2 * b + h, i] = groups[o]
                z[2 * b + h, i] = groups[o + 1]
    return q, s, z


def test_quantize_lorc_rank_zero(milo):
    W = wl.gen_weight(np.random.default_rng(55), 70, 256)
    qw, err = _quantize(milo, W, 0, 2, np.zeros((256, 0), np.float32))
    q, s, z, _ = oracle.hqq(oracle._f16(W))
    assert np.array_equal(qw.packed.cpu().numpy(), _blob_ref(q, s, z, 256))
    assert qw.U is None and err.shape == (1,)
    assert abs(err[0] - np.linalg.norm(oracle.residual(W, q, s, z).astype(np.float64))) <= 1e-5 * err[0]


def test_quantize_lorc_single_row(milo):
    """N = 1: the residual has rank 1, so 15 of the 16 sketch columns drop out
    of the basis; U V reproduces the residual up to the fp16 rounding of U, V."""
    rng = np.random.default_rng(56)
    W = wl.gen_weight(rng, 1, 128)
    om = rng.standard_normal((128, 16)).astype(np.float32)
    qw, err = _quantize(milo, W, 8, 0, om)
    q, s, z, _ = oracle.hqq(oracle._f16(W))
    R = oracle.residual(W, q, s, z).astype(np.float64)
    U, V = oracle.rsvd(R, 8, om, 2)
    uv = _f16(qw.U.cpu().numpy().view(np.uint16)) @ _f16(qw.V.cpu().numpy().view(np.uint16))
    assert np.linalg.norm(uv - U @ V) <= UV_TOL * np.linalg.norm(R)
    assert err[0] <= 2 ** -10 * np.linalg.norm(R)


def test_quantize_lorc_exact_weight_gives_zero_compensator(milo):
    """Weights on the int3 grid of their group (0..7 sixteenths, each group
    holding 0 and 7/16): the residual is exactly zero, every sketch column
    drops out, and U, V and the error are zero."""
    rng = np.random.default_rng(58)
    N, K = 64, 256
    q = rng.integers(0, 8, (N, K))
    q[:, ::64] = 0
    q[:, 1::64] = 7
    W = (q / 16.0).astype(np.float16).view(np.uint16)
    om = rng.standard_normal((K, 32)).astype(np.float32)
    qw, err = _quantize(milo, W, 16, 2, om)
    assert np.all(qw.U.cpu().numpy() == 0) and np.all(qw.V.cpu().numpy() == 0)
    assert err[0] == 0.0
    qh, sh, zh, _ = oracle.hqq(oracle._f16(W))
    assert np.array_equal(qw.packed.cpu().numpy(), _blob_ref(qh, sh, zh, K))


def test_quantized_weight_runs_in_the_grouped_linear(milo):
    """The quantiser's output is a QWeight the forward path consumes: the
    grouped linear with it matches the oracle's linear on the same pieces."""
    from parity_util import REL_TOL, rel_err
    rng = np.random.default_rng(57)
    N, K, r = 256, 512, 16
    W = wl.gen_weight(rng, N, K)
    om = rng.standard_normal((K, 2 * r)).astype(np.float32)
    qw, _ = _quantize(milo, W, r, 1, om)
    q, s, z = _unblob(qw.packed.cpu().numpy(), N, K)
    P = oracle.PackedProj(oracle.pack(q), s, z, qw.U.cpu().numpy().view(np.uint16),
                          qw.V.cpu().numpy().view(np.uint16))
    X = wl.gen_activations(rng, 5, K, "f16")
    lin = milo.GroupedLinear([qw])
    route = milo.milo_route(None, 1, False, E=1, ids=to_dev(np.zeros((5, 1), np.int32)))
    y = lin(f16_dev(X), route["offsets"], route["perm"], k=1).cpu().numpy()
    y_ref = oracle.linear(wl.f16_bits_to_f32(X).astype(np.float64), P)
    assert rel_err(y, y_ref) <= REL_TOL


def test_quantize_lorc_full_size_mixtral_w1(milo):
    """The Mixtral-shaped w1 (14336 x 4096), rank 32, one round: HQQ codes,
    scales and zeros bit-exact on sampled rows (rows are quantised
    independently), the fp32 residual bit-exact on those rows, and U V
    against the oracle's fp64 subspace iteration on the full residual."""
    rng = np.random.default_rng(59)
    N, K, r = 14336, 4096, 32
    W = wl.gen_weight(rng, N, K)
    om = rng.standard_normal((K, 2 * r)).astype(np.float32)
    qw, err = _quantize(milo, W, r, 0, om)
    _, R_gpu = milo.milo_hqq_pack(f16_dev(W), residual=True)
    R_gpu = R_gpu.cpu().numpy()
    rows = np.sort(rng.choice(N, size=96, replace=False))
    q, s, z, _ = oracle.hqq(oracle._f16(W[rows]))
    qg, sg, zg = _unblob(qw.packed.cpu().numpy(), N, K, rows)
    assert np.array_equal(qg, q) and np.array_equal(sg, s) and np.array_equal(zg, z)
    assert np.array_equal(R_gpu[rows].view(np.uint32), oracle.residual(W[rows], q, s, z).view(np.uint32))
    U, V = oracle.rsvd(R_gpu, r, om, 2)
    Ug = _f16(qw.U.cpu().numpy().view(np.uint16))
    Vg = _f16(qw.V.cpu().numpy().view(np.uint16))
    ref = U[rows] @ V
    assert np.linalg.norm(Ug[rows] @ Vg - ref) <= UV_TOL * np.linalg.norm(ref)
    E = R_gpu.astype(np.float64) - Ug @ Vg
    assert abs(err[0] - np.linalg.norm(E)) <= 1e-5 * err[0]


def test_quantize_experts_pipeline_runs_the_layer(milo):
    """The offline pipeline on a small layer: ranks from the kurtosis split
    (the oracle's kurtosis and split give the same ranks), every projection
    through the quantiser, and the layer forward with the result matches the
    oracle's forward on the same pieces."""
    from parity_util import REL_TOL, act_dev, rel_err
    wk = wl.small_moe(name="t_pipeline")
    names = ("w1", "w3", "w2")
    experts = [{n: f16_dev(e[n].W) for n in names} for e in wk.experts]
    st = milo.new_status()
    qexp, ranks = milo.quantize_experts(experts, avg_rank=16, rounds=1, dev_status=st)
    assert _status(st) == 0
    kr = [oracle.kurtosis(e[n].W) for e in wk.experts for n in names]
    assert ranks == oracle.assign_ranks(kr, 16)
    assert sum(ranks) <= 16 * len(ranks)
    # the oracle's view of the same quantised pieces
    ref = []
    for e in qexp:
        d = {}
        for n in names:
            qw = e[n]
            q, s, z = _unblob(qw.packed.cpu().numpy(), qw.N, qw.K)
            U = qw.U.cpu().numpy().view(np.uint16) if qw.rank else np.zeros((qw.N, 0), np.uint16)
            V = qw.V.cpu().numpy().view(np.uint16) if qw.rank else np.zeros((0, qw.K), np.uint16)
            d[n] = oracle.PackedProj(oracle.pack(q), s, z, U, V)
        ref.append(d)
    layer = milo.MoELayer(qexp, wk.n_routed, wk.n_shared, wk.top_k)
    r = milo.milo_route(f16_dev(wk.logits), wk.top_k, wk.renorm)
    y = layer(act_dev(wk.x, wk.x_dtype), r, out_dtype=torch.float32, dev_status=st)
    assert _status(st) == 0
    ids, w, *_ = oracle.route(wk.logits, wk.top_k, wk.renorm)
    y_ref, _, st_ref = oracle.moe_forward(wk.x, wk.x_dtype == "bf16", ids, w, ref, wk.n_routed, wk.n_shared,
                                          wk.hidden, wk.inter)
    assert st_ref == 0
    assert rel_err(y.cpu().numpy(), y_ref) <= REL_TOL

"""Pins for the offline MiLo quantiser in the oracle (CPU only).

"MiLo: Efficient Quantized MoE Inference with Mixture of Low-Rank
Compensators", section "MiLo Algorithm: Mixture of Low-Rank Compensators":
HQQ initial quantisation, a rank-r compensator from the SVD of the residual
W - W_quant, and rounds that re-quantise with U V taken into account and
recompute U V from the new residual.

Each pin checks the oracle against something other than itself: a hand-worked
HQQ group (tests/golden/hqq_worked_example.txt), the round-to-nearest
quantiser (one HQQ iteration reduces to it), an independent scalar minimiser
(the zero-point update without shrinkage is a least-squares fit), numpy's
exact SVD (Eckart-Young bounds, exact recovery of low-rank matrices) and
exact integer arithmetic for the fp32 target and residual.
"""
import os

import numpy as np
import pytest
from scipy.optimize import minimize_scalar

import oracle
import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _worked_group():
    t = [0.0, 7.0]
    t += [k + 0.25 for k in range(7)] * 2 + [k + 0.25 for k in range(6)]
    t += [k - 0.25 for k in (1, 2, 3, 4)]
    t += [k + 0.0625 for k in range(7)] * 2 + [0.0625, 1.0625]
    t += [3.0] * (64 - len(t))
    return np.array(t, np.float32)


def _golden_hqq():
    vals = {}
    with open(os.path.join(GOLDEN, "hqq_worked_example.txt")) as f:
        for line in f:
            if line.startswith("#") or ":" not in line:
                continue
            k, v = line.split(":", 1)
            vals[k.strip()] = v.split()
    return vals


def test_hqq_worked_example():
    g = _golden_hqq()
    t = _worked_group()
    assert t.size == 64
    q, s, z, zt, et = oracle.hqq_trace(t, int(g["iters"][0]), float(g["beta"][0]), float(g["kappa"][0]))
    assert s == int(g["scale"][0], 16)
    assert z == int(g["zero"][0], 16)
    for got, want, tol in zip(zt, map(float, g["z_trace"]), map(float, g["z_trace_tol"])):
        assert abs(got - want) <= tol, (zt, g["z_trace"])
    for got, want, tol in zip(et, map(float, g["err_trace"]), map(float, g["err_trace_tol"])):
        assert abs(got - want) <= tol, (et, g["err_trace"])
    assert np.array_equal(q, np.rint(t).astype(np.uint8))


@pytest.mark.parametrize("iters", [0, 1])
def test_hqq_without_a_zero_update_is_round_to_nearest(iters):
    """With no completed update HQQ keeps z0 = -min/s: the round-to-nearest
    quantiser's scale, zero and codes, bit for bit."""
    rng = np.random.default_rng(31)
    W = wl.gen_weight(rng, 48, 256)
    q0, s0, z0, _ = oracle.quantize(W)
    q1, s1, z1, _ = oracle.hqq(oracle._f16(W), iters=iters)
    assert np.array_equal(q0, q1) and np.array_equal(s0, s1) and np.array_equal(z0, z1)


def test_hqq_update_without_shrinkage_is_least_squares_zero():
    """beta -> 0 makes every shrinkage threshold infinite (w_e = 0), and the
    update reduces to the zero point minimising sum (t - (q - z) s)^2 for the
    current codes; checked with a scalar minimiser."""
    rng = np.random.default_rng(32)
    for _ in range(20):
        t = (rng.standard_normal(64) * 0.02).astype(np.float32)
        t[rng.integers(64)] *= 20
        _, s_bits, _, zt, _ = oracle.hqq_trace(t, 1, 1e-30, 1.0)
        s = float(np.float16(np.uint16(s_bits).view(np.float16)))
        q0 = np.clip(np.rint(t.astype(np.float64) / s + zt[0]), 0, 7)
        res = minimize_scalar(lambda z: float(np.sum((t - (q0 - z) * s) ** 2)),
                              bracket=(zt[0] - 1, zt[0] + 1), tol=1e-12)
        assert abs(zt[1] - res.x) <= 1e-5 * max(1.0, abs(res.x))


def test_hqq_without_shrinkage_target_is_a_fixed_point():
    """beta -> infinity: w_e = e, so the update returns the same zero point (up
    to fp32 rounding) and the codes never change."""
    rng = np.random.default_rng(33)
    t = (rng.standard_normal(64) * 0.02).astype(np.float32)
    _, _, _, zt, et = oracle.hqq_trace(t, 5, 1e30, 1.0)
    assert np.all(np.abs(np.diff(zt)) <= 1e-5 * max(1.0, abs(zt[0])))
    assert np.ptp(et) <= 1e-6 * et[0]


def test_hqq_keeps_the_zero_point_of_lowest_l1_error():
    rng = np.random.default_rng(34)
    for _ in range(50):
        t = (rng.standard_normal(64) * 0.02).astype(np.float32)
        t[rng.integers(64, size=3)] *= 15
        q, s_bits, z_bits, zt, et = oracle.hqq_trace(t, 20, 10.0, 1.01)
        # each recorded error is the L1 error at the recorded zero point, by brute force
        s = np.float32(np.uint16(s_bits).view(np.float16))
        for i in (0, 7, 19):
            qi = np.clip(np.rint(t / s + zt[i]), 0, 7).astype(np.float32)
            assert abs(np.sum(np.abs(t - (qi - zt[i]) * s)) - et[i]) <= 1e-5 * et[i]
        best = int(np.argmin(et))
        assert z_bits == int(np.float16(zt[best]).view(np.uint16))
        zf = np.float32(np.uint16(z_bits).view(np.float16))
        assert np.array_equal(q, np.clip(np.rint(t / s + zf), 0, 7).astype(np.uint8))


def test_hqq_matrix_is_the_group_fit_at_every_thread_count():
    """The matrix call is the one-group fit applied to each (row, group), its
    scale and zero stored [K/64, N]; rows split over any number of host
    threads give the same bits."""
    rng = np.random.default_rng(36)
    N, K = 13, 256
    T = oracle._f16(wl.gen_weight(rng, N, K))
    ref = None
    for nt in (1, 3, 5, 64):
        out = oracle.hqq(T, nthreads=nt)
        assert out[3] == 0
        if ref is None:
            ref = out
            continue
        for a, b in zip(ref[:3], out[:3]):
            assert np.array_equal(a, b)
    q, sc, ze, _ = ref
    for n in (0, 6, 12):
        for j in range(K // 64):
            qg, s_bits, z_bits, _, _ = oracle.hqq_trace(T[n, 64 * j:64 * (j + 1)], oracle.HQQ_ITERS,
                                                        oracle.HQQ_BETA, oracle.HQQ_KAPPA)
            assert np.array_equal(q[n, 64 * j:64 * (j + 1)], qg)
            assert sc[j, n] == s_bits and ze[j, n] == z_bits


def test_hqq_lowers_the_l1_error_of_outlier_groups():
    """The point of HQQ's sparsity-promoting fit: on weights with outliers its
    L1 reconstruction error is lower than round-to-nearest's."""
    rng = np.random.default_rng(35)
    W = wl.gen_weight(rng, 64, 512)
    q0, s0, z0, _ = oracle.quantize(W)
    q1, s1, z1, _ = oracle.hqq(oracle._f16(W))
    e0 = np.abs(oracle._f16(W) - oracle.dequant(q0, s0, z0)).sum()
    e1 = np.abs(oracle._f16(W) - oracle.dequant(q1, s1, z1)).sum()
    assert e1 < 0.99 * e0


def test_lorc_target_and_residual_are_exact_where_fp32_is():
    """Integers times powers of two: W - U V and W - (q - z) s are exact in
    fp32, so they equal the fp64 values computed independently."""
    rng = np.random.default_rng(36)
    N, K, r = 16, 128, 8
    W = (rng.integers(-64, 64, (N, K)) / 64.0).astype(np.float16).view(np.uint16)
    U = (rng.integers(-8, 8, (N, r)) / 8.0).astype(np.float16).view(np.uint16)
    V = (rng.integers(-8, 8, (r, K)) / 16.0).astype(np.float16).view(np.uint16)
    T = oracle.lorc_target(W, U, V)
    f = lambda b: np.asarray(b).view(np.float16).astype(np.float64)
    assert np.array_equal(T.astype(np.float64), f(W) - f(U) @ f(V))
    q, s, z, _ = oracle.quantize(W)
    R = oracle.residual(W, q, s, z)
    assert np.allclose(R.astype(np.float64), f(W) - oracle.dequant(q, s, z), rtol=0, atol=2 ** -20)


def test_rsvd_recovers_low_rank_matrices():
    rng = np.random.default_rng(37)
    N, K, r = 200, 256, 16
    for rho in (1, 7, 16):
        R = rng.standard_normal((N, rho)) @ rng.standard_normal((rho, K))
        U, V = oracle.rsvd(R, r, rng.standard_normal((K, 2 * r)), 2)
        assert U.shape == (N, r) and V.shape == (r, K)
        assert np.linalg.norm(R - U @ V) <= 1e-10 * np.linalg.norm(R)


def test_rsvd_within_eckart_young_bounds():
    """No rank-r matrix beats the truncated SVD (lower bound, catches a rank
    above r); subspace iteration with two power steps and 2r columns comes
    within 2 % of it on a flat (noise-like) spectrum."""
    rng = np.random.default_rng(38)
    N, K, r = 300, 256, 16
    R = rng.standard_normal((N, K)) * 1e-3
    U, V = oracle.rsvd(R, r, rng.standard_normal((K, 2 * r)), 2)
    _, _, opt = oracle.svd_truncated(R, r)
    err = np.linalg.norm(R - U @ V)
    assert opt * (1 - 1e-12) <= err <= 1.02 * opt


def test_rsvd_matches_the_truncated_svd_with_a_spectral_gap():
    rng = np.random.default_rng(39)
    N, K, r = 256, 384, 8
    L = rng.standard_normal((N, r)) @ np.diag(np.linspace(10, 5, r)) @ rng.standard_normal((r, K)) / 16
    R = L + rng.standard_normal((N, K)) * 1e-4
    U, V = oracle.rsvd(R, r, rng.standard_normal((K, 2 * r)), 2)
    Ue, Ve, _ = oracle.svd_truncated(R, r)
    assert np.linalg.norm(U @ V - Ue @ Ve) <= 1e-8 * np.linalg.norm(Ue @ Ve)
    # balanced split: U^T U = V V^T = diag(sigma)
    sig = np.linalg.svd(R, compute_uv=False)[:r]
    assert np.allclose(U.T @ U, np.diag(sig), rtol=1e-8, atol=1e-8 * sig[0])
    assert np.allclose(V @ V.T, np.diag(sig), rtol=1e-8, atol=1e-8 * sig[0])


def test_rsvd_of_zero_is_zero():
    U, V = oracle.rsvd(np.zeros((64, 128)), 8, np.random.default_rng(40).standard_normal((128, 16)), 2)
    assert np.all(U == 0) and np.all(V == 0)


def test_quantize_lorc_rounds():
    """Round 0 is HQQ + the compensator of its residual; further rounds lower
    the error on the weight recipe, and the kept round has the lowest."""
    rng = np.random.default_rng(41)
    N, K, r = 128, 256, 16
    W = wl.gen_weight(rng, N, K)
    om = rng.standard_normal((K, 2 * r))
    res = oracle.quantize_lorc(W, r, 3, om)
    assert res["status"] == 0
    e = res["err"]
    assert e.shape == (4,) and np.all(np.diff(e) < 0)
    assert res["best"] == 3
    q0, s0, z0, _ = oracle.hqq(oracle._f16(W))
    R0 = oracle.residual(W, q0, s0, z0)
    U0, V0 = oracle.rsvd(R0, r, om, 2)
    E0 = R0.astype(np.float64) - (U0.astype(np.float16).astype(np.float64) @ V0.astype(np.float16).astype(np.float64))
    assert abs(e[0] - np.linalg.norm(E0)) <= 1e-9 * e[0]
    # the returned pieces reproduce the reported error
    R = oracle.residual(W, res["q"], res["scale"], res["zero"]).astype(np.float64)
    E = R - oracle._f16(res["U"]).astype(np.float64) @ oracle._f16(res["V"]).astype(np.float64)
    assert abs(np.linalg.norm(E) - e[3]) <= 1e-9 * e[3]


def test_quantize_lorc_rank_zero_is_hqq():
    rng = np.random.default_rng(42)
    W = wl.gen_weight(rng, 64, 128)
    res = oracle.quantize_lorc(W, 0, 2, np.zeros((128, 0)))
    q, s, z, _ = oracle.hqq(oracle._f16(W))
    assert np.array_equal(res["q"], q) and np.array_equal(res["zero"], z)
    assert res["U"].shape == (64, 0) and res["V"].shape == (0, 128) and res["err"].shape == (1,)
    assert abs(res["err"][0] - np.linalg.norm(oracle.residual(W, q, s, z).astype(np.float64))) <= 1e-12

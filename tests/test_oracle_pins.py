"""Pins for the CPU oracle: each check ties it to something other than itself.

The pins come from the pages of "MiLo: Efficient Quantized MoE Inference with
Mixture of Low-Rank Compensators" (32 int3 codes in three 32-bit words with no
wasted bit; asymmetric dequantisation with a zero point; W_out = W_quant + U V;
top-k expert routing) and from the mathematics: hand-worked examples
(tests/golden/), exhaustive and brute-force checks on tiny inputs, closed forms,
invariants, and special cases that reduce to a library routine (numpy matmul,
numpy float16 rounding, scipy's logistic function).
"""
import itertools
import os

import numpy as np
import pytest

import oracle
import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------------------
# fp16 conversion (numpy's float16 cast is IEEE round-to-nearest-even)
# ---------------------------------------------------------------------------

def test_f2h_matches_numpy_rounding():
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(10.0) ** rng.integers(-9, 5, 20000),
        np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e9, -1e9, 2 ** -24, 2 ** -25, 3 * 2 ** -26,
                  2 ** -14, 2 ** -14 - 2 ** -25, 1.0 + 2 ** -11, 1.0 + 3 * 2 ** -11], np.float32)]
    ).astype(np.float32)
    lib = oracle.lib()
    got = np.array([lib.milo_ref_f2h(float(v)) for v in vals], np.uint16)
    with np.errstate(over="ignore"):
        exp = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, exp)
    # fp64 inputs round once, straight to fp16 (no double rounding through fp32)
    d = np.array([-905.2500128746033, 12596.00043296814, 1.0 + 2.0 ** -11 + 2.0 ** -40])
    got = np.array([lib.milo_ref_d2h(float(v)) for v in d], np.uint16)
    assert np.array_equal(got, d.astype(np.float16).view(np.uint16))


def test_h2d_exact_for_every_pattern():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    finite = (bits & 0x7C00) != 0x7C00
    got = oracle.h2d(bits[finite])
    exp = bits[finite].view(np.float16).astype(np.float64)
    assert np.array_equal(got, exp)


# ---------------------------------------------------------------------------
# packing
# ---------------------------------------------------------------------------

def _golden_units():
    units, rows = [], []
    with open(os.path.join(GOLDEN, "pack_worked_examples.txt")) as f:
        for line in f:
            line = line.strip()
            if line.startswith("unit "):
                codes, words = line[5:].split(":")
                units.append(([int(c) for c in codes.split()], [int(w, 16) for w in words.split()]))
            elif line.startswith("row128 "):
                rows.append([int(w, 16) for w in line.split(":")[1].split()])
    return units, rows


def _unit_to_row(u):
    """Place unit codes u_0..u_31 as unit c=0 of a K=128 row (other codes 0)."""
    q = np.zeros((1, 128), np.uint8)
    q[0, 0:16] = u[:16]
    q[0, 64:80] = u[16:]
    return q


def test_pack_hand_worked_units():
    units, _ = _golden_units()
    assert len(units) == 4
    for codes, words in units:
        Q = oracle.pack(_unit_to_row(codes))
        assert list(Q[0, 0:3]) == words, (codes, [hex(w) for w in Q[0, :3]])
        assert not Q[0, 3:].any()


def test_pack_hand_worked_superblock():
    _, rows = _golden_units()
    q = (np.arange(128) // 16 % 8).astype(np.uint8)[None, :]
    Q = oracle.pack(q)
    assert list(Q[0]) == rows[0]


def test_pack_uses_every_bit_once():
    """No wasted bit: the 3 bits of each of the 128 codes of a super-block land on
    384 distinct bits of its 12 words (exhaustive one-hot)."""
    seen = set()
    for k in range(128):
        for beta in range(3):
            q = np.zeros((1, 128), np.uint8)
            q[0, k] = 1 << beta
            Q = oracle.pack(q)
            nz = np.flatnonzero(Q[0])
            assert len(nz) == 1
            word = int(nz[0])
            assert bin(int(Q[0, word])).count("1") == 1
            bit = int(Q[0, word]).bit_length() - 1
            seen.add((word, bit))
    assert len(seen) == 384


def test_pack_superblocks_are_independent_and_k_major():
    """Super-block b depends only on codes [128b, 128b+128) and sits in words 12b..12b+11."""
    rng = np.random.default_rng(2)
    q = rng.integers(0, 8, (3, 512), dtype=np.uint8)
    Q = oracle.pack(q)
    for b in range(4):
        Qb = oracle.pack(np.ascontiguousarray(q[:, 128 * b:128 * (b + 1)]))
        assert np.array_equal(Q[:, 12 * b:12 * (b + 1)], Qb)


def test_unpack_roundtrip_exhaustive_one_hot_and_random():
    for k in range(128):
        for v in range(1, 8):
            q = np.zeros((1, 128), np.uint8)
            q[0, k] = v
            assert np.array_equal(oracle.unpack(oracle.pack(q), 128), q)
    rng = np.random.default_rng(3)
    q = rng.integers(0, 8, (40, 256 * 4), dtype=np.uint8)   # 10^4 random units
    assert np.array_equal(oracle.unpack(oracle.pack(q), q.shape[1]), q)


def test_device_blob_matches_reshape():
    """The device blob of a packed weight: 64-row tiles (zero rows pad the last),
    one block per (tile, super-block) = the tile's words for the super-block,
    then its two groups' scales and zeros, interleaved as (s, z) of rows j and
    j + 8 of each 16-row block.  Checked against numpy reshapes/transposes of the
    padded arrays, for N that is and is not a multiple of 64 and for even and odd
    K/128."""
    rng = np.random.default_rng(11)
    for N, K in ((64, 256), (100, 384), (16, 128), (130, 640)):
        SB, G, NT = K // 128, K // 64, (N + 63) // 64
        Q = rng.integers(0, 2 ** 32, (N, 3 * K // 32), dtype=np.uint64).astype(np.uint32)
        sc = rng.integers(0, 2 ** 16, (G, N), dtype=np.uint32).astype(np.uint16)
        ze = rng.integers(0, 2 ** 16, (G, N), dtype=np.uint32).astype(np.uint16)
        Qp = np.zeros((NT * 64, 3 * K // 32), np.uint32); Qp[:N] = Q
        sp = np.zeros((G, NT * 64), np.uint16); sp[:, :N] = sc
        zp = np.zeros((G, NT * 64), np.uint16); zp[:, :N] = ze
        words = Qp.reshape(NT, 64, SB, 12).transpose(0, 2, 1, 3)          # [t][b][r][j]
        # [g][t][m][hi][j][s|z] with row r = 16m + 8hi + j, stored as [t][g][m][j][hi][s|z]
        groups = np.stack([sp.reshape(G, NT, 4, 2, 8), zp.reshape(G, NT, 4, 2, 8)], axis=-1)
        groups = groups.transpose(1, 0, 2, 4, 3, 5)
        parts = []
        for t in range(NT):
            for b in range(SB):
                parts.append(words[t, b].reshape(-1).view(np.uint8))
                parts.append(groups[t, 2 * b:2 * b + 2].reshape(-1).view(np.uint8))
        want = np.concatenate(parts)
        assert want.size == NT * SB * 3584
        assert np.array_equal(oracle.tile_pack(Q, sc, ze, K), want)


def test_unit_codes_share_one_group_per_pair():
    """Each 16-bit half-pair (bits [3i,3i+3) and [16+3i,..)) of a word carries two
    codes of the same scale group; the spare bits of a unit belong to one group."""
    for k in range(0, 128, 2):
        w0, b0 = oracle.code_bit(k, 0)
        w1, b1 = oracle.code_bit(k + 1, 0)
        if b0 < 15:   # regular field: partner code sits 16 bits higher in the same word
            assert w0 == w1 and b1 == b0 + 16
            assert (k // 64) == ((k + 1) // 64)


# ---------------------------------------------------------------------------
# quantiser
# ---------------------------------------------------------------------------

def _h(vals):
    return np.array(vals, np.float32).astype(np.float16).view(np.uint16)


def test_quantize_hand_worked_groups():
    # (a) w_i = (i mod 8)/4 - 1/2 -> s = 0.25, z = 2, q_i = i mod 8
    a = ((np.arange(64) % 8) / 4.0 - 0.5)
    q, s, z, st = oracle.quantize(_h(a)[None, :])
    assert st == 0 and s[0, 0] == 0x3400 and z[0, 0] == 0x4000
    assert np.array_equal(q[0], np.arange(64) % 8)
    # (b) ties go to the even code
    b = np.zeros(64); b[:9] = [0, 7, 0.5, 1.5, 2.5, 3.5, 4.5, 5.5, 6.5]
    q, s, z, _ = oracle.quantize(_h(b)[None, :])
    assert s[0, 0] == 0x3C00 and z[0, 0] == 0x8000     # z = -(+0)/1 = -0
    assert list(q[0, :9]) == [0, 7, 0, 2, 2, 4, 4, 6, 6] and not q[0, 9:].any()
    # (c) a constant group is reconstructed exactly
    c = np.full(64, 0.5)
    q, s, z, _ = oracle.quantize(_h(c)[None, :])
    assert s[0, 0] == 0x3C00 and z[0, 0] == 0xB800 and not q.any()
    assert np.all(oracle.dequant(q, s, z) == 0.5)


def test_quantize_brute_force_nearest_level():
    """Every code is the nearest of the 8 levels (q - z) s in the fp32 arithmetic
    of the rule; min maps to 0 and max to 7; codes stay in [0, 7]."""
    W = wl.gen_weight(np.random.default_rng(4), 16, 256)
    q, s, z, st = oracle.quantize(W)
    assert st == 0 and q.max() <= 7
    w = W.view(np.float16).astype(np.float32)
    sf = s.view(np.float16).astype(np.float32)
    zf = z.view(np.float16).astype(np.float32)
    for n in range(16):
        for j in range(4):
            g = w[n, 64 * j:64 * (j + 1)]
            sv, zv = sf[j, n], zf[j, n]
            u = g / sv + zv          # fp32, as in the rule
            levels = np.arange(8, dtype=np.float32)
            d = np.abs(u[:, None] - levels[None, :])
            best = np.argmin(d, axis=1)
            # ties are exactly .5 and go to the even level
            tie = np.isclose(np.sort(d, axis=1)[:, 0], np.sort(d, axis=1)[:, 1], rtol=0, atol=0)
            best[tie] = np.round(u[tie])
            best = np.clip(best, 0, 7)
            assert np.array_equal(q[n, 64 * j:64 * (j + 1)], best)
            assert q[n, 64 * j + int(np.argmin(g))] == 0
            assert q[n, 64 * j + int(np.argmax(g))] == 7


def test_quantize_roundtrip_error_bound():
    """|w - w_hat| <= s/2 + (rounding of z and of w/s) for every weight."""
    W = wl.gen_weight(np.random.default_rng(5), 32, 512)
    q, s, z, _ = oracle.quantize(W)
    w = W.view(np.float16).astype(np.float64)
    wh = oracle.dequant(q, s, z)
    sf = np.repeat(s.view(np.float16).astype(np.float64).T, 64, axis=1)
    zf = np.repeat(z.view(np.float16).astype(np.float64).T, 64, axis=1)
    bound = sf * (0.5 + 2.0 ** -11 * (np.abs(zf) + 8.0) + 2.0 ** -20)
    assert np.all(np.abs(w - wh) <= bound)


def test_quantize_flags_nonfinite():
    W = wl.gen_weight(np.random.default_rng(6), 2, 128)
    W[1, 5] = 0x7C00   # +inf
    _, _, _, st = oracle.quantize(W)
    assert st & oracle.NONFINITE


def test_dequant_closed_form():
    q = np.array([[0, 7, 3, 4] * 32], np.uint8)
    s = np.array([[0x3800], [0x4000]], np.uint16)   # 0.5 then 2.0
    z = np.array([[0x4200], [0x3C00]], np.uint16)   # 3.0 then 1.0
    wh = oracle.dequant(q, s, z)
    exp = np.concatenate([(np.array([0, 7, 3, 4] * 16) - 3.0) * 0.5,
                          (np.array([0, 7, 3, 4] * 16) - 1.0) * 2.0])
    assert np.array_equal(wh[0], exp)


# ---------------------------------------------------------------------------
# linear with compensator: y = x w_hat^T + (x V^T) U^T
# ---------------------------------------------------------------------------

def _proj_from_codes(q, s_val, z_val, U=None, V=None):
    N, K = q.shape
    s = np.full((K // 64, N), s_val, np.uint16)
    z = np.full((K // 64, N), z_val, np.uint16)
    U = np.zeros((N, 0), np.uint16) if U is None else U
    V = np.zeros((0, K), np.uint16) if V is None else V
    return oracle.PackedProj(oracle.pack(q), s, z, U, V)


def test_linear_integer_hand_case_exact():
    """s = 1, z = 4: w_hat = q - 4 is an integer matrix, integer x gives an exact
    integer y equal to numpy's integer matmul."""
    rng = np.random.default_rng(7)
    q = rng.integers(0, 8, (8, 128), dtype=np.uint8)
    X = rng.integers(-3, 4, (8, 128)).astype(np.float64)
    P = _proj_from_codes(q, 0x3C00, 0x4400)
    Y = oracle.linear(X, P)
    exp = X.astype(np.int64) @ (q.astype(np.int64) - 4).T
    assert np.array_equal(Y, exp.astype(np.float64))


def test_linear_rank1_compensator_exact_and_oriented():
    """Rank-1 integer U [N,1], V [1,K] adds (x V^T) U^T exactly; N != K so a
    transposed operand cannot pass."""
    rng = np.random.default_rng(8)
    N, K = 24, 128
    q = rng.integers(0, 8, (N, K), dtype=np.uint8)
    X = rng.integers(-2, 3, (3, K)).astype(np.float64)
    Ui = rng.integers(-3, 4, (N, 1))
    Vi = rng.integers(-3, 4, (1, K))
    P0 = _proj_from_codes(q, 0x3C00, 0x4400)
    P1 = _proj_from_codes(q, 0x3C00, 0x4400, _h(Ui), _h(Vi))
    Y0, Y1 = oracle.linear(X, P0), oracle.linear(X, P1)
    assert np.array_equal(Y1 - Y0, ((X.astype(np.int64) @ Vi.T) @ Ui.T).astype(np.float64))


def test_linear_rank0_equals_plain_quantized_gemm_and_matches_numpy():
    rng = np.random.default_rng(9)
    W = wl.gen_weight(rng, 48, 256)
    U = wl.gen_normal_f16(rng, (48, 16), 0.01)
    V = wl.gen_normal_f16(rng, (16, 256), 0.01)
    X = rng.standard_normal((5, 256))
    q, s, z, _ = oracle.quantize(W)
    wh = oracle.dequant(q, s, z)
    P0 = oracle.PackedProj(oracle.pack(q), s, z, np.zeros((48, 0), np.uint16), np.zeros((0, 256), np.uint16))
    P = oracle.PackedProj(oracle.pack(q), s, z, U, V)
    np.testing.assert_allclose(oracle.linear(X, P0), X @ wh.T, rtol=1e-12, atol=1e-12)
    Uf = U.view(np.float16).astype(np.float64)
    Vf = V.view(np.float16).astype(np.float64)
    np.testing.assert_allclose(oracle.linear(X, P), X @ (wh + Uf @ Vf).T, rtol=1e-12, atol=1e-12)


def _int3_exact_matrix(rng, R, C):
    """fp16 bits of an R x C matrix whose every group of 64 along C holds the
    levels (q - 3) * 2^-6 with q = 0 and q = 7 both present: the quantiser then
    recovers s = 2^-6, z = 3 and the codes exactly."""
    q = rng.integers(0, 8, (R, C))
    for g0 in range(0, C, 64):
        q[:, g0] = 0
        q[:, g0 + 1] = 7
    vals = ((q - 3) * 2.0 ** -6).astype(np.float16)
    return vals.view(np.uint16), q


def test_linear_int3_compensator_exact_levels_equal_fp16():
    """int3 compensator (U^T grouped along N, V along K): with U and V already
    on the int3 levels the quantised compensator equals the fp16 one exactly;
    N != K so a transposed operand changes the result."""
    rng = np.random.default_rng(21)
    N, K, r = 384, 256, 8      # U^T is packed along N: N is a multiple of 128 too
    W = wl.gen_weight(rng, N, K)
    Ut, _ = _int3_exact_matrix(rng, r, N)       # U^T [r, N]
    V, _ = _int3_exact_matrix(rng, r, K)
    U = np.ascontiguousarray(Ut.T)
    X = rng.standard_normal((4, K))
    P16 = oracle.quantize_projection(W, U, V)
    P3 = oracle.quantize_projection(W, U, V, lorc_int3=True)
    assert P3.lorc3 is not None
    assert np.array_equal(oracle.linear(X, P3), oracle.linear(X, P16))


def test_linear_int3_compensator_rounding_bound():
    """Random U, V: each dequantised compensator entry is within half a step
    (s/2 plus the zero point's rounding) of its fp16 value, so the int3 and
    fp16 outputs differ by at most the propagated bound."""
    rng = np.random.default_rng(22)
    N, K, r = 128, 384, 16
    W = wl.gen_weight(rng, N, K)
    U = wl.gen_normal_f16(rng, (N, r), 0.01)
    V = wl.gen_normal_f16(rng, (r, K), 0.01)
    X = rng.standard_normal((3, K))
    qu, su, zu, _ = oracle.quantize(np.ascontiguousarray(U.T))
    qv, sv, zv, _ = oracle.quantize(V)
    Uh = oracle.dequant(qu, su, zu).T
    Vh = oracle.dequant(qv, sv, zv)
    Uf = U.view(np.float16).astype(np.float64)
    Vf = V.view(np.float16).astype(np.float64)
    step_u = np.repeat(su.view(np.float16).astype(np.float64).T, 64, axis=1).T   # [N, r] per entry
    step_v = np.repeat(sv.view(np.float16).astype(np.float64).T, 64, axis=1)     # [r, K]
    assert np.all(np.abs(Uh - Uf) <= 0.5 * step_u * (1 + 2 ** -9) + 1e-12)
    assert np.all(np.abs(Vh - Vf) <= 0.5 * step_v * (1 + 2 ** -9) + 1e-12)
    P16 = oracle.quantize_projection(W, U, V)
    P3 = oracle.quantize_projection(W, U, V, lorc_int3=True)
    d = oracle.linear(X, P3) - oracle.linear(X, P16)
    np.testing.assert_allclose(d, (X @ Vh.T) @ Uh.T - (X @ Vf.T) @ Uf.T, rtol=1e-9, atol=1e-12)


def test_linear_independent_of_thread_count():
    rng = np.random.default_rng(10)
    W = wl.gen_weight(rng, 37, 128)
    X = rng.standard_normal((3, 128))
    q, s, z, _ = oracle.quantize(W)
    P = oracle.PackedProj(oracle.pack(q), s, z, np.zeros((37, 0), np.uint16), np.zeros((0, 128), np.uint16))
    assert np.array_equal(oracle.linear(X, P, nthreads=1), oracle.linear(X, P, nthreads=5))


# ---------------------------------------------------------------------------
# routing
# ---------------------------------------------------------------------------

def test_route_brute_force_over_subsets():
    rng = np.random.default_rng(11)
    for E, k in ((4, 1), (6, 2), (8, 2), (8, 3)):
        # coarse logits make ties frequent
        L = _h(rng.integers(-3, 4, (40, E)) * 0.5)
        ids, w, off, perm, inv, st = oracle.route(L, k, renorm=True)
        assert st == 0
        lf = L.view(np.float16).astype(np.float64)
        for t in range(40):
            # the best subset by (sum of logits, then lexicographically smallest ids)
            best = max(itertools.combinations(range(E), k),
                       key=lambda c: (sorted(lf[t, list(c)], reverse=True), [-i for i in c]))
            assert sorted(ids[t]) == sorted(best)
            # slot order: descending logit, ties by lower id
            order = sorted(ids[t], key=lambda e: (-lf[t, e], e))
            assert list(ids[t]) == order


def test_route_hand_example_with_ties():
    L = np.zeros((4, 8), np.float32)
    L[1] = np.arange(8)[::-1]          # descending -> experts 0, 1
    L[2] = np.arange(8)                # ascending -> experts 7, 6
    L[3] = [1, 5, 5, 0, 0, 0, 0, 0]    # tie at 5 -> 1 then 2
    ids, w, off, perm, inv, _ = oracle.route(_h(L), 2, renorm=True)
    assert ids.tolist() == [[0, 1], [0, 1], [7, 6], [1, 2]]
    np.testing.assert_allclose(w[0], [0.5, 0.5], rtol=0, atol=1e-15)
    np.testing.assert_allclose(w[3], [0.5, 0.5], rtol=0, atol=1e-15)
    np.testing.assert_allclose(w[1], [1 / (1 + np.exp(-1.0)), 1 / (1 + np.exp(1.0))], rtol=1e-14)
    assert off.tolist() == [0, 2, 5, 6, 6, 6, 6, 7, 8]
    # expert 0: flat slots 0 (t0 j0), 2 (t1 j0); expert 1: 1, 3, 6; expert 2: 7; 6: 5; 7: 4
    assert perm.tolist() == [0, 2, 1, 3, 6, 7, 5, 4]
    assert np.array_equal(inv[perm], np.arange(8))


def test_route_weights_match_softmax_library():
    from scipy.special import softmax
    rng = np.random.default_rng(12)
    L = wl.gen_normal_f16(rng, (30, 64), 1.0)
    lf = L.view(np.float16).astype(np.float64)
    ids, w, *_ = oracle.route(L, 6, renorm=False)
    full = softmax(lf, axis=1)
    np.testing.assert_allclose(w, np.take_along_axis(full, ids, 1), rtol=1e-13)
    ids, w, *_ = oracle.route(L, 6, renorm=True)
    part = softmax(np.take_along_axis(lf, ids, 1), axis=1)
    np.testing.assert_allclose(w, part, rtol=1e-13)


def test_group_invariants():
    rng = np.random.default_rng(13)
    for T, k, E in ((1, 1, 1), (0, 2, 4), (17, 2, 8), (300, 6, 64), (64, 1, 8)):
        ids = rng.integers(0, E, (T, k)).astype(np.int32)
        off, perm, inv, st = oracle.group(ids, E)
        assert st == 0
        assert off[0] == 0 and off[-1] == T * k and np.all(np.diff(off) >= 0)
        assert np.array_equal(np.diff(off), np.bincount(ids.ravel(), minlength=E))
        assert np.array_equal(np.sort(perm), np.arange(T * k))
        assert np.array_equal(inv[perm], np.arange(T * k))
        flat = ids.ravel()
        for e in range(E):
            seg = perm[off[e]:off[e + 1]]
            assert np.all(flat[seg] == e) and np.all(np.diff(seg) > 0)


def test_group_flags_bad_ids():
    ids = np.array([[0, 9], [1, -1]], np.int32)
    off, perm, inv, st = oracle.group(ids, 4)
    assert st & oracle.BAD_EXPERT
    assert off[-1] == 2 and inv[1] == -1 and inv[3] == -1


# ---------------------------------------------------------------------------
# SwiGLU and the MoE layer
# ---------------------------------------------------------------------------

def test_silu_closed_forms():
    from scipy.special import expit
    assert oracle.silu(0.0) == 0.0
    assert oracle.silu(50.0) == pytest.approx(50.0, rel=1e-15)
    assert abs(oracle.silu(-50.0)) < 1e-19
    for a in np.linspace(-8, 8, 33):
        assert oracle.silu(a) == pytest.approx(a * expit(a), rel=1e-14, abs=1e-300)


def _small_layer(E=3, S=1, H=128, I=256, ranks=(0, 8, 16, 8), seed=14):
    rng = np.random.default_rng(seed)
    experts = []
    for e in range(E + S):
        d = {}
        for name, (n, kk) in (("w1", (I, H)), ("w3", (I, H)), ("w2", (H, I))):
            W = wl.gen_weight(rng, n, kk)
            U = wl.gen_normal_f16(rng, (n, ranks[e]), 0.01)
            V = wl.gen_normal_f16(rng, (ranks[e], kk), 0.01)
            d[name] = oracle.quantize_projection(W, U, V)
        experts.append(d)
    return experts


def _expert_by_hand(xrow, d):
    a = oracle.linear(xrow, d["w1"])
    b = oracle.linear(xrow, d["w3"])
    h = np.array([oracle.silu(v) for v in a.ravel()]).reshape(a.shape) * b
    hq = h.astype(np.float16).astype(np.float64)      # activations are fp16
    return oracle.linear(hq, d["w2"]), hq


def test_moe_single_expert_reduces_to_chain():
    H, I = 128, 256
    ex = _small_layer(E=1, S=0, H=H, I=I, ranks=(16,))
    x = wl.gen_activations(np.random.default_rng(15), 3, H, "bf16")
    ids = np.zeros((3, 1), np.int32)
    w = np.ones((3, 1))
    y, h, st = oracle.moe_forward(x, True, ids, w, ex, 1, 0, H, I, want_h=True)
    X = wl.bf16_bits_to_f32(x).astype(np.float64)
    y_ref, hq = _expert_by_hand(X, ex[0])
    assert st == 0
    np.testing.assert_allclose(y, y_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(h.view(np.float16).astype(np.float64), hq, rtol=0, atol=0)


def test_moe_combine_weights_slots_and_shared():
    """y[t] = sum_j w[t,j] expert_{ids[t,j]}(x_t) + sum_s shared_s(x_t), checked
    slot by slot against single-expert evaluations."""
    H, I, E, S = 128, 256, 3, 1
    ex = _small_layer(E=E, S=S, H=H, I=I)
    x = wl.gen_activations(np.random.default_rng(16), 4, H, "f16")
    ids = np.array([[0, 2], [1, 0], [2, 1], [2, 0]], np.int32)
    w = np.array([[0.7, 0.3], [0.25, 0.75], [1.0, 0.0], [0.5, 0.5]])
    y, h, st = oracle.moe_forward(x, False, ids, w, ex, E, S, H, I, want_h=True)
    X = x.view(np.float16).astype(np.float64)
    for t in range(4):
        acc = np.zeros(H)
        for j in range(2):
            yy, _ = _expert_by_hand(X[t:t + 1], ex[ids[t, j]])
            acc += w[t, j] * yy[0]
        ys, _ = _expert_by_hand(X[t:t + 1], ex[E])
        acc += ys[0]
        np.testing.assert_allclose(y[t], acc, rtol=1e-11, atol=1e-12)


def test_moe_one_hot_weights_equal_gather_and_relabelling_invariance():
    H, I, E = 128, 256, 3
    ex = _small_layer(E=E, S=0, H=H, I=I)
    x = wl.gen_activations(np.random.default_rng(17), 5, H, "bf16")
    ids = np.array([[0, 1], [1, 2], [2, 0], [0, 2], [1, 0]], np.int32)
    w1h = np.array([[1.0, 0.0]] * 5)
    y, _, _ = oracle.moe_forward(x, True, ids, w1h, ex, E, 0, H, I)
    X = wl.bf16_bits_to_f32(x).astype(np.float64)
    for t in range(5):
        yy, _ = _expert_by_hand(X[t:t + 1], ex[ids[t, 0]])
        np.testing.assert_allclose(y[t], yy[0], rtol=1e-11, atol=1e-12)
    # relabel experts by a permutation: the layer output must not change
    pi = np.array([2, 0, 1])
    ex2 = [None] * E
    for e in range(E):
        ex2[pi[e]] = ex[e]
    w = np.random.default_rng(18).random((5, 2))
    ya, _, _ = oracle.moe_forward(x, True, ids, w, ex, E, 0, H, I)
    yb, _, _ = oracle.moe_forward(x, True, pi[ids].astype(np.int32), w, ex2, E, 0, H, I)
    np.testing.assert_allclose(ya, yb, rtol=1e-12, atol=1e-13)


def test_moe_flags_fp16_range_of_h_not_of_x():
    """Activations are FP16 up to a power-of-two row scale, so a bf16 input
    beyond 65504 is valid (the result stays exact); the SwiGLU output h is an
    fp16 tensor, so a finite silu(a) b that rounds to an fp16 infinity is
    flagged."""
    H, I = 128, 256
    ex = _small_layer(E=1, S=0, H=H, I=I, ranks=(0,))
    ids, w = np.zeros((1, 1), np.int32), np.ones((1, 1))
    big = wl.f32_to_bf16_bits(np.full((1, H), 1.0e6, np.float32))
    y, h, st = oracle.moe_forward(big, True, ids, w, ex, 1, 0, H, I, want_h=True)
    assert st & oracle.FP16_RANGE                       # h overflows
    hf = h.view(np.float16)
    assert np.isinf(hf).any()
    x = wl.f32_to_bf16_bits(np.full((1, H), 70000.0, np.float32))
    rng = np.random.default_rng(19)
    small = {}
    for name, (n, kk), a in (("w1", (I, H), -16), ("w3", (I, H), -16), ("w2", (H, I), 0)):
        W = wl.f32_to_f16_bits(wl.f16_bits_to_f32(wl.gen_weight(rng, n, kk)) * np.float32(2.0 ** a))
        small[name] = oracle.quantize_projection(W, np.zeros((n, 0), np.uint16), np.zeros((0, kk), np.uint16))
    y2, h2, st2 = oracle.moe_forward(x, True, ids, w, [small], 1, 0, H, I, want_h=True)
    assert st2 == 0 and np.isfinite(h2.view(np.float16)).all() and np.isfinite(y2).all()
    assert np.abs(h2.view(np.float16)).max() > 0

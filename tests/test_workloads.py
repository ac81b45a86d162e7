"""The seeded input recipe (workloads.py) checked against its own definition.

The generators hold none of the method's arithmetic, but every parity test and
bench line depends on them drawing what the recipe says: fp16 weights
N(0, 0.02) with round(0.001 n k) distinct entries times 20, compensators
N(0, 0.01), activations N(0, 1) rounded to nearest-even bf16 or fp16,
truncated-Zipf expert ids, and one independent, reproducible stream per
tensor.  CPU only.
"""
import numpy as np

import workloads as wl


def test_bf16_rounding_is_nearest_even():
    """Brute force: the bf16 chosen for an fp32 value is the nearer of its two
    bf16 neighbours, the even one on a tie (exact in fp64)."""
    rng = np.random.default_rng(3)
    f = np.concatenate([
        (rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000)).astype(np.float32),
        # exact ties: bf16 values plus half a bf16 ulp (odd and even low bits)
        (wl.bf16_bits_to_f32(np.arange(0x3F80, 0x3F90, dtype=np.uint16)).view(np.uint32) + 0x8000).view(np.float32),
    ])
    got = wl.f32_to_bf16_bits(f)
    u = f.view(np.uint32)
    lo = (u >> 16).astype(np.uint16)
    hi = lo + np.uint16(1)
    v = f.astype(np.float64)
    dlo = np.abs(v - wl.bf16_bits_to_f32(lo).astype(np.float64))
    dhi = np.abs(wl.bf16_bits_to_f32(hi).astype(np.float64) - v)
    want = np.where(dlo < dhi, lo, np.where(dhi < dlo, hi, np.where(lo & 1, hi, lo)))
    assert np.array_equal(got, want)
    assert np.any(dlo == dhi)                           # the tie cases were exercised


def test_streams_are_reproducible_and_independent():
    a = wl.rng_for("mixtral", "x").standard_normal(8)
    b = wl.rng_for("mixtral", "x").standard_normal(8)
    c = wl.rng_for("mixtral", "logits").standard_normal(8)
    d = wl.rng_for("mixtral", "x", 1).standard_normal(8)
    e = wl.rng_for("deepseek", "x").standard_normal(8)
    assert np.array_equal(a, b)
    for other in (c, d, e):
        assert not np.array_equal(a, other)


def test_weight_recipe_outliers_and_scale():
    """Exactly round(0.001 n k) distinct entries are the base draw times 20
    (each product rounded to fp16 once); the base draw has std 0.02."""
    n, k = 256, 384
    base = wl.f16_bits_to_f32(wl.gen_weight(wl.rng_for("t_wl", "W"), n, k, outlier_frac=0.0)).astype(np.float64)
    full = wl.f16_bits_to_f32(wl.gen_weight(wl.rng_for("t_wl", "W"), n, k)).astype(np.float64)
    moved = np.flatnonzero(base.ravel() != full.ravel())
    assert moved.size == round(0.001 * n * k)
    raw = wl.rng_for("t_wl", "W").standard_normal(n * k, dtype=np.float32) * np.float32(0.02)
    want = wl.f16_bits_to_f32(wl.f32_to_f16_bits(raw[moved] * np.float32(20.0)))
    assert np.array_equal(full.ravel()[moved], want.astype(np.float64))
    assert abs(base.std() / 0.02 - 1.0) < 0.02 and abs(base.mean()) < 0.02 * 0.02


def test_compensator_and_activation_scales():
    U = wl.f16_bits_to_f32(wl.gen_normal_f16(wl.rng_for("t_wl", "U"), (4096, 16), 0.01)).astype(np.float64)
    assert abs(U.std() / 0.01 - 1.0) < 0.02
    x = wl.bf16_bits_to_f32(wl.gen_activations(wl.rng_for("t_wl", "x"), 64, 1024, "bf16")).astype(np.float64)
    assert abs(x.std() - 1.0) < 0.02
    xh = wl.f16_bits_to_f32(wl.gen_activations(wl.rng_for("t_wl", "x"), 64, 1024, "f16")).astype(np.float64)
    # the same draw rounded to fp16 instead of bf16: within half a bf16 ulp
    # plus half an fp16 ulp of each other
    # (relative 2^-8 and 2^-11 of the fp32 draw)
    assert np.all(np.abs(xh - x) <= (2.0 ** -8 + 2.0 ** -11) * 1.01 * np.abs(x) + 2.0 ** -25)
    assert abs(xh.std() - 1.0) < 0.02


def test_zipf_ids_follow_the_truncated_law():
    """P(e) proportional to (e + 1)^-1.1 over 8 experts, expert 0 hottest:
    frequencies of 200,000 draws within 4 standard errors of the law."""
    t, e, s = 200000, 8, 1.1
    ids = wl.gen_zipf_ids(wl.rng_for("t_wl", "ids"), t, e, s)
    assert ids.dtype == np.int32 and ids.min() >= 0 and ids.max() < e
    p = (np.arange(e) + 1.0) ** -s
    p /= p.sum()
    freq = np.bincount(ids, minlength=e) / t
    assert np.all(np.abs(freq - p) < 4 * np.sqrt(p * (1 - p) / t))
    assert np.argmax(freq) == 0


def test_small_layer_shapes_and_ranks():
    wk = wl.small_moe("t_wl_layer", T=7, hidden=256, inter=384, n_routed=4, n_shared=1, top_k=2,
                      rank_choices=(0, 8, 16))
    assert wk.x.shape == (7, 256) and wk.x.dtype == np.uint16
    assert wk.logits.shape == (7, 4) and wk.n_experts == 5 and len(wk.experts) == 5
    for e, d in enumerate(wk.experts):
        assert d["w1"].W.shape == (384, 256) and d["w3"].W.shape == (384, 256) and d["w2"].W.shape == (256, 384)
        for name in ("w1", "w3", "w2"):
            P = d[name]
            assert P.rank == wk.ranks[e] and P.rank in (0, 8, 16)
            assert P.U.shape == (P.n, P.rank) and P.V.shape == (P.rank, P.k)
    # the same name draws the same layer; the projections of one expert differ
    again = wl.small_moe("t_wl_layer", T=7, hidden=256, inter=384, n_routed=4, n_shared=1, top_k=2,
                         rank_choices=(0, 8, 16))
    assert np.array_equal(again.x, wk.x) and np.array_equal(again.experts[3]["w2"].W, wk.experts[3]["w2"].W)
    assert not np.array_equal(wk.experts[0]["w1"].W, wk.experts[0]["w3"].W)

"""GPU parity at the workload sizes, in the launch configuration that bench.py
times (same entry points, same workspace sizing):

* single expert decode (1 x 1024 -> 1024, rank 16): every output;
* Mixtral-8x7B-shaped decode layer (16 tokens, top-2, ranks {0,16,32,64}):
  routing bit-exact, every output of the layer and every SwiGLU activation;
* DeepSeekMoE-16B-shaped decode layer (64 tokens, top-6 of 64 + 2 shared):
  routing bit-exact, every output;
* w1 batch sweep with Zipf routing, T = 1 ... 1024: all rows up to 64 tokens,
  a seeded sample of rows beyond;
* Mixtral-shaped prefill (8192 tokens, rank 64): routing bit-exact for all
  tokens, layer outputs and SwiGLU activations on at least 256 tokens that
  reach every (expert, 128-row tile) of both grouped GEMMs (tokens are
  independent in an MoE layer, so the oracle runs the sampled tokens alone).
"""
from concurrent.futures import ThreadPoolExecutor

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




def _gpu_proj(milo, P, lorc_int3=False):
    return milo.QWeight.quantize(f16_dev(P.W), f16_dev(P.U) if P.rank else None,
                                 f16_dev(P.V) if P.rank else None, lorc_int3=lorc_int3)


def _oracle_projs(projs, lorc_int3=False):
    with ThreadPoolExecutor(8) as ex:
        return list(ex.map(lambda P: oracle.quantize_projection(P.W, P.U, P.V, lorc_int3=lorc_int3), projs))


def _layers(milo, wk, lorc_int3=False):
    names = ("w1", "w3", "w2")
    gpu = [{n: _gpu_proj(milo, wk.experts[e][n], lorc_int3) for n in names} for e in range(wk.n_experts)]
    flat = _oracle_projs([wk.experts[e][n] for e in range(wk.n_experts) for n in names], lorc_int3)
    ref = [{n: flat[3 * e + i] for i, n in enumerate(names)} for e in range(wk.n_experts)]
    return milo.MoELayer(gpu, wk.n_routed, wk.n_shared, wk.top_k), ref


def _route(milo, wk):
    st = milo.new_status()
    r = milo.milo_route(f16_dev(wk.logits), wk.top_k, wk.renorm, dev_status=st)
    ids, w, off, perm, inv, st_ref = oracle.route(wk.logits, wk.top_k, wk.renorm)
    torch.cuda.synchronize()
    assert int(st.item()) == st_ref == 0
    assert np.array_equal(r["ids"].cpu().numpy(), ids)
    assert np.array_equal(r["offsets"].cpu().numpy(), off)
    assert np.array_equal(r["perm"].cpu().numpy(), perm)
    assert np.array_equal(r["inv_perm"].cpu().numpy(), inv)
    np.testing.assert_allclose(r["w"].cpu().numpy(), w, rtol=2e-6, atol=1e-7)
    return r, ids, w, inv


def test_single_expert_decode_full(milo):
    x, P = wl.single()
    lin = milo.GroupedLinear([_gpu_proj(milo, P)])
    r = milo.milo_route(None, 1, False, E=1, ids=to_dev(np.zeros((1, 1), np.int32)))
    st = milo.new_status()
    y = lin(act_dev(x, "f16"), r["offsets"], r["perm"], k=1, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    y_ref = oracle.linear(act_f64(x, "f16"), _oracle_projs([P])[0])
    err = rel_err(y.cpu().numpy(), y_ref)
    assert err <= REL_TOL, err


def _layer_full(milo, wk, lorc_int3=False):
    layer, ref = _layers(milo, wk, lorc_int3)
    r, ids, w, inv = _route(milo, wk)
    st = milo.new_status()
    y = layer(act_dev(wk.x, wk.x_dtype), r, out_dtype=torch.float32, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    y_ref, h_ref, st_ref = oracle.moe_forward(wk.x, wk.x_dtype == "bf16", ids, w, ref, wk.n_routed,
                                              wk.n_shared, wk.hidden, wk.inter, want_h=True)
    assert st_ref == 0
    err = rel_err(y.cpu().numpy(), y_ref)
    assert err <= REL_TOL, err
    h = layer.h_view(wk.T).cpu().numpy().view(np.uint16)
    Tk = wk.T * wk.top_k
    h_gpu = np.concatenate([h[inv], h[Tk:]]).view(np.float16).astype(np.float64)
    herr = rel_err(h_gpu, h_ref.view(np.float16).astype(np.float64))
    assert herr <= REL_TOL, herr


def test_mixtral_decode_layer_full(milo):
    _layer_full(milo, wl.mixtral())


def test_deepseek_decode_layer_full(milo):
    _layer_full(milo, wl.deepseek())


def test_mixtral_decode_layer_full_int3_compensators(milo):
    """The Mixtral-shaped decode layer with U^T and V quantised to int3 too."""
    _layer_full(milo, wl.mixtral(), lorc_int3=True)


def test_w1_sweep_zipf(milo):
    base = wl.sweep(1)
    projs = [base.experts[e]["w1"] for e in range(8)]
    lin = milo.GroupedLinear([_gpu_proj(milo, P) for P in projs])
    ref = _oracle_projs(projs)
    for T in (1, 4, 16, 64, 256, 1024):
        wk = wl.sweep(T) if T > 1 else base
        x = wk.x
        ids = wk.ids
        r = milo.milo_route(None, 1, False, E=8, ids=to_dev(ids))
        st = milo.new_status()
        y = lin(act_dev(x, "bf16"), r["offsets"], r["perm"], k=1, dev_status=st).cpu().numpy()
        assert int(st.item()) == 0
        rows = np.arange(T) if T <= 64 else np.sort(
            np.random.default_rng(T).choice(T, size=48, replace=False))
        X = act_f64(x[rows], "bf16")
        y_ref = np.zeros((rows.size, projs[0].n))
        for e in range(8):
            sel = np.flatnonzero(ids[rows, 0] == e)
            if sel.size:
                y_ref[sel] = oracle.linear(X[sel], ref[e])
        err = rel_err(y[rows], y_ref)
        assert err <= REL_TOL, (T, err)


def prefill_sample(off: np.ndarray, perm: np.ndarray, k: int, T: int, tile: int = 128,
                   at_least: int = 256, seed: int = 55) -> np.ndarray:
    """Tokens whose rows reach every work item of the grouped GEMMs: for each
    expert, the first and the last routed row of each of its `tile`-row
    tiles (the ragged last tile included), the first and the last token, then
    seeded random tokens up to `at_least`."""
    tok = {0, T - 1}
    for e in range(off.size - 1):
        for p0 in range(int(off[e]), int(off[e + 1]), tile):
            p1 = min(p0 + tile, int(off[e + 1])) - 1
            tok.add(int(perm[p0]) // k)
            tok.add(int(perm[p1]) // k)
    rng = np.random.default_rng(seed)
    while len(tok) < at_least:
        tok.add(int(rng.integers(T)))
    return np.array(sorted(tok))


def test_mixtral_prefill_sampled(milo):
    """8192 tokens on the tcgen05 path: every output feature and every SwiGLU
    activation of the sampled tokens, the sample reaching every (expert,
    128-row tile) of both grouped GEMMs at its first and last row."""
    wk = wl.prefill()
    layer, ref = _layers(milo, wk)
    r, ids, w, inv = _route(milo, wk)
    st = milo.new_status()
    y = layer(act_dev(wk.x, wk.x_dtype), r, out_dtype=torch.float32, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    off, perm = r["offsets"].cpu().numpy(), r["perm"].cpu().numpy()
    tok = prefill_sample(off, perm, wk.top_k, wk.T)
    assert tok.size >= 256
    covered = {(e, (int(inv[t * wk.top_k + j]) - int(off[e])) // 128)
               for t in tok for j in range(wk.top_k) for e in [int(ids[t, j])]}
    every = {(e, q) for e in range(wk.n_routed) for q in range((int(off[e + 1] - off[e]) + 127) // 128)}
    assert covered == every
    y_ref, h_ref, st_ref = oracle.moe_forward(wk.x[tok], True, ids[tok], w[tok], ref, wk.n_routed,
                                              wk.n_shared, wk.hidden, wk.inter, want_h=True)
    assert st_ref == 0
    err = rel_err(y.cpu().numpy()[tok], y_ref)
    assert err <= REL_TOL, err
    # h rows of the sampled slots: GPU row inv[t k + j] against the oracle's slot i k + j
    h = layer.h_view(wk.T).cpu().numpy().view(np.uint16)
    rows = np.array([inv[t * wk.top_k + j] for t in tok for j in range(wk.top_k)])
    h_gpu = h[rows].view(np.float16).astype(np.float64)
    herr = rel_err(h_gpu, h_ref.view(np.float16).astype(np.float64))
    assert herr <= REL_TOL, herr

"""Saving and loading packed experts (binding IO; CPU, no kernel runs).

The offline quantiser's output -- each projection's packed blob and its
compensator -- is written to an .npz file and read back bit for bit, with the
sizes checked against the packed layout the library reports.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def milo():
    import int3_gemm_rank_b200 as m
    m.lib()
    return m


def _blob(milo, g, n, k):
    return torch.randint(0, 256, (milo.milo_packed_bytes(n, k),), generator=g, dtype=torch.uint8)


def _experts(milo):
    """Two experts: fp16 compensators of rank 16, an int3 one of rank 8, and a
    projection without compensator."""
    g = torch.Generator().manual_seed(5)
    H, I = 256, 384
    out = []
    for e in range(2):
        d = {}
        for name, (n, k) in (("w1", (I, H)), ("w3", (I, H)), ("w2", (H, I))):
            if name == "w3" and e == 1:
                r = 8
                d[name] = milo.QWeight(_blob(milo, g, n, k), n, k, _blob(milo, g, r, n), _blob(milo, g, r, k),
                                       rank=r, lorc_int3=True)
            elif name == "w2" and e == 0:
                d[name] = milo.QWeight(_blob(milo, g, n, k), n, k)
            else:
                U = torch.randn(n, 16, generator=g).half()
                V = torch.randn(16, k, generator=g).half()
                d[name] = milo.QWeight(_blob(milo, g, n, k), n, k, U, V)
        out.append(d)
    return out


def test_save_load_round_trip(milo, tmp_path):
    ex = _experts(milo)
    path = tmp_path / "layer.npz"
    milo.save_experts(path, ex)
    back = milo.load_experts(path, device="cpu")
    assert len(back) == 2
    for d0, d1 in zip(ex, back):
        assert set(d0) == set(d1) == {"w1", "w3", "w2"}
        for name in d0:
            a, b = d0[name], d1[name]
            assert (a.N, a.K, a.rank, a.lorc_int3) == (b.N, b.K, b.rank, b.lorc_int3)
            assert torch.equal(a.packed, b.packed) and b.packed.dtype == torch.uint8
            if a.rank:
                assert torch.equal(a.U, b.U) and torch.equal(a.V, b.V) and b.U.dtype == a.U.dtype
            else:
                assert b.U is None and b.V is None
    assert back[1]["w3"].lorc_int3 and back[0]["w2"].rank == 0


def test_load_rejects_wrong_sizes(milo, tmp_path):
    ex = _experts(milo)
    path = tmp_path / "layer.npz"
    milo.save_experts(path, ex)
    with np.load(path) as f:
        arrays = {k: f[k] for k in f.files}
    arrays["e0.w1.packed"] = arrays["e0.w1.packed"][:-16]
    bad = tmp_path / "bad.npz"
    np.savez(bad, **arrays)
    with pytest.raises(ValueError, match="e0.w1.packed"):
        milo.load_experts(bad, device="cpu")


def test_save_rejects_a_blob_of_another_shape(milo, tmp_path):
    ex = _experts(milo)
    ex[0]["w1"].packed = ex[0]["w1"].packed[:-1]
    with pytest.raises(ValueError, match="e0.w1.packed"):
        milo.save_experts(tmp_path / "x.npz", ex)

"""The Python binding checks every tensor against the call's shape before its
pointer crosses the C ABI (CPU: every check here fires before a kernel could
launch).

The library reads and writes through raw pointers with the sizes the call
states; a tensor of another dtype, width or length would be read or written
out of bounds on the device, so the binding refuses it on the host.
"""

import pytest

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def milo():
    import int3_gemm_rank_b200 as m
    m.lib()
    return m


@pytest.fixture
def no_device_check(milo, monkeypatch):
    """Lets CPU tensors through the CUDA-device check, so the size checks
    behind it can be exercised without a GPU; nothing here reaches a kernel."""
    monkeypatch.setattr(milo, "_cuda", lambda t, name: None)
    return milo


class _FakeLinear:
    """The fields of a prepared GroupedLinear that the call checks read."""

    def __init__(self, milo, N, K, n_experts):
        self.cs = milo.milo_linear(N, K, n_experts, milo.MILO_GROUP, 0, None)


class _FakeLayer:
    def __init__(self, milo, H, I, n_routed, n_shared, top_k):
        self.cs = milo.milo_moe_layer(H, I, n_routed, n_shared, top_k, milo.MILO_GROUP, 0, None)


def test_arg_checks_dtype_then_shape_then_device(milo):
    t = torch.zeros((4, 8), dtype=torch.float32)
    with pytest.raises(ValueError, match="int32"):
        milo._arg(t, "offsets", (torch.int32,))
    with pytest.raises(ValueError, match=r"shape \(4, 9\)"):
        milo._arg(t, "y", milo._OUT, shape=(4, 9))
    with pytest.raises(ValueError, match="at least 33"):
        milo._arg(t, "perm", None, min_numel=33)
    with pytest.raises(ValueError, match="contiguous CUDA tensor"):
        milo._arg(t, "y", milo._OUT, shape=(4, 8))
    with pytest.raises(ValueError, match="contiguous"):
        milo._arg(t.t(), "y", milo._OUT, shape=(8, 4))
    with pytest.raises(TypeError):
        milo._arg(None, "x")


def test_grouped_linear_refuses_wrong_widths_and_lengths(no_device_check):
    milo = no_device_check
    lin = _FakeLinear(milo, N=256, K=512, n_experts=4)
    off = torch.zeros(5, dtype=torch.int32)
    perm = torch.zeros(6, dtype=torch.int32)
    # x must be [T, K] in fp16 / bf16
    with pytest.raises(ValueError, match=r"x must be \[T, 512\]"):
        milo.milo_grouped_linear(lin, torch.zeros((3, 256), dtype=torch.float16), off, perm, k=2)
    with pytest.raises(ValueError, match=r"x must be \[T, 512\]"):
        milo.milo_grouped_linear(lin, torch.zeros(512, dtype=torch.float16), off, perm, k=2)
    with pytest.raises(ValueError, match="float16 or bfloat16"):
        milo.milo_grouped_linear(lin, torch.zeros((3, 512), dtype=torch.float32), off, perm, k=2)
    x = torch.zeros((3, 512), dtype=torch.bfloat16)
    # offsets: n_experts + 1 int32; perm: T*k int32
    with pytest.raises(ValueError, match="at least 5"):
        milo.milo_grouped_linear(lin, x, torch.zeros(4, dtype=torch.int32), perm, k=2)
    with pytest.raises(ValueError, match="int32"):
        milo.milo_grouped_linear(lin, x, off.long(), perm, k=2)
    with pytest.raises(ValueError, match="at least 6"):
        milo.milo_grouped_linear(lin, x, off, perm[:5], k=2)


def test_grouped_linear_refuses_a_wrong_output(no_device_check):
    milo = no_device_check
    lin = _FakeLinear(milo, N=256, K=512, n_experts=4)
    x = torch.zeros((3, 512), dtype=torch.float16)
    off, perm = torch.zeros(5, dtype=torch.int32), torch.zeros(6, dtype=torch.int32)
    with pytest.raises(ValueError, match=r"shape \(6, 256\)"):
        milo.milo_grouped_linear(lin, x, off, perm, k=2, y=torch.zeros((3, 256)))
    with pytest.raises(ValueError, match="float16 or bfloat16 or float32"):
        milo.milo_grouped_linear(lin, x, off, perm, k=2, y=torch.zeros((6, 256), dtype=torch.float64))
    with pytest.raises(ValueError, match="dev_status"):
        milo.milo_grouped_linear(lin, x, off, perm, k=2, y=torch.zeros((6, 256)),
                                 dev_status=torch.zeros(1, dtype=torch.int64))
    with pytest.raises(ValueError, match=r"shape \(6, 256\)"):
        milo.milo_grouped_linear_noalloc(lin, x, off, perm, k=2, y=torch.zeros((6, 255)))


def test_moe_forward_checks_the_route_and_output(no_device_check):
    milo = no_device_check
    layer = _FakeLayer(milo, H=256, I=384, n_routed=4, n_shared=1, top_k=2)
    T = 5
    x = torch.zeros((T, 256), dtype=torch.bfloat16)
    route = {"w": torch.zeros((T, 2)), "offsets": torch.zeros(5, dtype=torch.int32),
             "perm": torch.zeros(T * 2, dtype=torch.int32), "inv_perm": torch.zeros(T * 2, dtype=torch.int32)}
    with pytest.raises(ValueError, match=r"x must be \[T, 256\]"):
        milo.milo_moe_forward(layer, torch.zeros((T, 384), dtype=torch.bfloat16), route)
    for key, bad in (("w", torch.zeros((T, 1))), ("offsets", torch.zeros(4, dtype=torch.int32)),
                     ("perm", torch.zeros(9, dtype=torch.int32)),
                     ("inv_perm", torch.zeros(T * 2, dtype=torch.int64))):
        r = dict(route, **{key: bad})
        with pytest.raises(ValueError, match=key):
            milo.milo_moe_forward(layer, x, r)
    with pytest.raises(ValueError, match="required"):
        milo.milo_moe_forward(layer, x, dict(route, perm=None))
    with pytest.raises(ValueError, match=r"shape \(5, 256\)"):
        milo.milo_moe_forward(layer, x, route, y=torch.zeros((T * 2, 256)))


def test_workspace_view_never_reports_negative_bytes(no_device_check):
    """A caller's workspace shorter than its alignment slack gives 0 bytes (the
    library then refuses it), never a negative size that ctypes would wrap."""
    milo = no_device_check
    for n in (0, 1, 100, 255, 256, 1000):
        ws = torch.empty(n, dtype=torch.uint8)
        ptr, nb = milo._ws_arg(ws, ws.device)
        assert ptr % 256 == 0 and 0 <= nb <= n
        assert ptr + nb == ws.data_ptr() + n or nb == 0
    ws = torch.empty(300, dtype=torch.float32)        # any dtype: its bytes count
    ptr, nb = milo._ws_arg(ws, ws.device)
    assert ptr + nb == ws.data_ptr() + 1200


def test_route_needs_E_and_matching_ids(milo):
    ids = torch.zeros((4, 2), dtype=torch.int32)
    with pytest.raises(ValueError, match="E"):
        milo.milo_route(None, 2, False, ids=ids)
    with pytest.raises(ValueError, match=r"ids must be \[T, 1\]"):
        milo.milo_route(None, 1, False, E=8, ids=ids)
    with pytest.raises(ValueError, match="int32"):
        milo.milo_route(None, 2, False, E=8, ids=ids.long())
    with pytest.raises(ValueError, match="float16"):
        milo.milo_route(torch.zeros((4, 8)), 2, True)
    with pytest.raises(ValueError, match=r"\[T, E\]"):
        milo.milo_route(torch.zeros(8, dtype=torch.float16), 2, True)


def test_packed_buffers_checked_against_the_shape(no_device_check):
    milo = no_device_check
    need = milo.milo_packed_bytes(128, 256)
    with pytest.raises(ValueError, match=f"at least {need}"):
        milo.milo_dequantize(torch.zeros(need - 1, dtype=torch.uint8), 128, 256)
    with pytest.raises(ValueError, match="uint8"):
        milo.milo_unpack(torch.zeros(need, dtype=torch.int8), 128, 256)
    with pytest.raises(ValueError, match=r"shape \(128, 256\)"):
        milo.milo_dequantize(torch.zeros(need, dtype=torch.uint8), 128, 256,
                             out=torch.zeros((256, 128), dtype=torch.float16))


def test_qweight_pieces_checked_before_the_table_is_written(no_device_check):
    milo = no_device_check
    N, K, r = 128, 256, 16
    blob = torch.zeros(milo.milo_packed_bytes(N, K), dtype=torch.uint8)
    U, V = torch.zeros((N, r), dtype=torch.float16), torch.zeros((r, K), dtype=torch.float16)
    milo.QWeight(blob, N, K, U, V).check()
    with pytest.raises(ValueError, match="at least"):
        milo.QWeight(blob[:-1], N, K, U, V).check()
    with pytest.raises(ValueError, match=r"U must have shape \(128, 16\)"):
        milo.QWeight(blob, N, K, U[:, :8], V, rank=16).check()
    with pytest.raises(ValueError, match=r"V must have shape \(16, 256\)"):
        milo.QWeight(blob, N, K, U, V[:, :128]).check()
    with pytest.raises(ValueError, match="float16"):
        milo.QWeight(blob, N, K, U.float(), V).check()
    # int3 factors: the blobs of U^T [r, N] and V [r, K]
    ub = torch.zeros(milo.milo_packed_bytes(r, N), dtype=torch.uint8)
    vb = torch.zeros(milo.milo_packed_bytes(r, K), dtype=torch.uint8)
    milo.QWeight(blob, N, K, ub, vb, rank=r, lorc_int3=True).check()
    with pytest.raises(ValueError, match="at least"):
        milo.QWeight(blob, N, K, ub[:-16], vb, rank=r, lorc_int3=True).check()
    # an N the int3 format cannot hold (not a multiple of 128): refused by the library's size query
    blob192 = torch.zeros(milo.milo_packed_bytes(192, K), dtype=torch.uint8)
    with pytest.raises(milo.MiloError) as e:
        milo.QWeight(blob192, 192, K, U, V, rank=r, lorc_int3=True).check()
    assert e.value.status == milo.MILO_ERR_UNSUPPORTED_SHAPE


def test_packers_and_quantiser_need_fp16_weights_and_matching_factors(no_device_check):
    milo = no_device_check
    W = torch.zeros((128, 256), dtype=torch.float16)
    for bad in (torch.zeros((128, 256), dtype=torch.uint8), torch.zeros((128, 256), dtype=torch.bfloat16)):
        with pytest.raises(ValueError, match="float16"):
            milo.milo_pack(bad)
        with pytest.raises(ValueError, match="float16"):
            milo.milo_hqq_pack(bad)
        with pytest.raises(ValueError, match="float16"):
            milo.milo_quantize_lorc(bad, milo.lorc_params(0))
    with pytest.raises(ValueError, match=r"\[N, K\]"):
        milo.milo_pack(torch.zeros(256, dtype=torch.float16))
    U, V = torch.zeros((128, 8), dtype=torch.float16), torch.zeros((8, 256), dtype=torch.float16)
    with pytest.raises(ValueError, match="both"):
        milo.milo_hqq_pack(W, U, None)
    with pytest.raises(ValueError, match=r"V must have shape \(8, 256\)"):
        milo.milo_hqq_pack(W, U, V[:, :128])
    with pytest.raises(ValueError, match=r"U must have shape \(128, 8\)"):
        milo.milo_hqq_pack(W, U[:64], V)
    with pytest.raises(ValueError, match="dev_status"):
        milo.milo_pack(W, dev_status=torch.zeros(1, dtype=torch.float32))

"""The C-ABI library builds, loads and exports every entry point that
include/milo.h declares; host-side argument validation (no GPU needed)."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "milo.h")).read()
    return sorted(set(re.findall(r"^MILO_API[^;(]*?\b(milo_\w+)\s*\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def milo():
    from int3_gemm_rank_b200 import build
    build.build()
    import int3_gemm_rank_b200 as m
    return m


def test_header_declares_the_boundary():
    names = _declared()
    for required in ("milo_pack", "milo_route", "milo_moe_forward", "milo_grouped_linear",
                     "milo_layer_prepare", "milo_moe_workspace_bytes"):
        assert required in names


def test_library_exports_every_declared_symbol(milo):
    L = milo.lib()
    for name in _declared():
        assert hasattr(L, name), name
    assert set(milo.EXPORTS) == set(_declared())


def test_checked_build_exports_every_declared_symbol():
    """The checked build (MILO_CHECKED: range checks in the kernels) is the
    same library with the same entry points."""
    from int3_gemm_rank_b200 import build
    path = build.build(checked=True)
    assert path.endswith("libmilo_checked.so")
    L = C.CDLL(path)
    for name in _declared():
        assert hasattr(L, name), name


def test_status_strings_and_version(milo):
    L = milo.lib()
    assert L.milo_version() >= 1
    assert L.milo_status_str(0) == b"ok"
    assert b"shape" in L.milo_status_str(2)


def test_host_validation_rejects_before_launch(milo):
    L = milo.lib()
    fake = C.c_void_p(0x1000)
    # group != 64
    assert L.milo_pack(fake, 16, 128, 32, fake, None, None) == milo.MILO_ERR_UNSUPPORTED_SHAPE
    # K not a multiple of 128
    assert L.milo_pack(fake, 16, 100, 64, fake, None, None) == milo.MILO_ERR_UNSUPPORTED_SHAPE
    assert b"multiple of 128" in L.milo_last_error()
    # NULL pointers
    assert L.milo_pack(None, 16, 128, 64, fake, None, None) == milo.MILO_ERR_INVALID_ARG
    # router limits
    assert L.milo_route(fake, 4, 300, 2, 0, fake, fake, fake, fake, fake, None, None) == \
        milo.MILO_ERR_UNSUPPORTED_SHAPE
    assert L.milo_route(fake, 4, 8, 9, 0, fake, fake, fake, fake, fake, None, None) == \
        milo.MILO_ERR_UNSUPPORTED_SHAPE
    assert L.milo_route(fake, 4, 8, 2, 0x80, fake, fake, fake, fake, fake, None, None) == \
        milo.MILO_ERR_INVALID_ARG


def test_prepare_validates_shapes_and_ranks(milo):
    L = milo.lib()
    nb = C.c_size_t()
    assert L.milo_table_bytes(3, C.byref(nb)) == 0 and nb.value % 64 == 0 and nb.value > 0
    fake = 0x10000
    w = milo.milo_qweight(fake, None, None, 12, 0)   # rank not a multiple of 8
    lin = milo.milo_linear(64, 128, 1, 64, 0, None)
    assert L.milo_linear_prepare(C.byref(lin), C.byref(w), C.c_void_p(fake), 1 << 20) == \
        milo.MILO_ERR_UNSUPPORTED_SHAPE
    lin = milo.milo_linear(64, 200, 1, 64, 0, None)            # K % 128
    w = milo.milo_qweight(fake, None, None, 0, 0)
    assert L.milo_linear_prepare(C.byref(lin), C.byref(w), C.c_void_p(fake), 1 << 20) == \
        milo.MILO_ERR_UNSUPPORTED_SHAPE
    lin = milo.milo_linear(64, 128, 1, 32, 0, None)            # group
    assert L.milo_linear_prepare(C.byref(lin), C.byref(w), C.c_void_p(fake), 1 << 20) == \
        milo.MILO_ERR_UNSUPPORTED_SHAPE
    layer = milo.milo_moe_layer(4096, 14336, 8, 0, 9, 64, 0, None)   # top_k > n_routed
    e = milo.milo_expert(w, w, w)
    assert L.milo_layer_prepare(C.byref(layer), C.byref(e), C.c_void_p(fake), 1 << 20) == \
        milo.MILO_ERR_UNSUPPORTED_SHAPE


def test_workspace_sizes_grow_with_tokens(milo):
    L = milo.lib()
    layer = milo.milo_moe_layer(4096, 14336, 8, 0, 2, 64, 64, None)
    a, b = C.c_size_t(), C.c_size_t()
    assert L.milo_moe_workspace_bytes(C.byref(layer), 16, C.byref(a)) == 0
    assert L.milo_moe_workspace_bytes(C.byref(layer), 8192, C.byref(b)) == 0
    assert 0 < a.value < b.value
    assert L.milo_moe_h_offset(C.byref(layer), 16) % 256 == 0


MAX_ROWS = 0x3FFFFFFF   # MILO_MAX_ROWS


def test_header_states_the_row_limit():
    src = open(os.path.join(ROOT, "include", "milo.h")).read()
    assert re.search(r"#define MILO_MAX_ROWS 0x3FFFFFFF\b", src)


def test_calls_above_the_row_limit_are_refused_before_planning(milo):
    """T*k (grouped linear, router) or T*(top_k + n_shared) (MoE layer) above
    the row limit: the size queries and the calls refuse the shape instead of
    sizing a workspace from a wrapped 32-bit row count.  Every call here
    returns before any CUDA call, so no device is needed."""
    L = milo.lib()
    nb = C.c_size_t(123)
    lin = milo.milo_linear(4096, 4096, 8, 64, 0, None)
    # at the limit the query succeeds; one token more (k = 2) does not
    assert L.milo_linear_workspace_bytes(C.byref(lin), MAX_ROWS // 2, 2, C.byref(nb)) == 0 and nb.value > 0
    assert L.milo_linear_workspace_bytes(C.byref(lin), MAX_ROWS // 2 + 1, 2, C.byref(nb)) == \
        milo.MILO_ERR_UNSUPPORTED_SHAPE
    assert b"MILO_MAX_ROWS" in L.milo_last_error()
    # T * k wraps a signed 32-bit count: 2^31 - 1 tokens, k = 16
    assert L.milo_linear_workspace_bytes(C.byref(lin), 0x7FFFFFFF, 16, C.byref(nb)) == \
        milo.MILO_ERR_UNSUPPORTED_SHAPE
    fake = C.c_void_p(0x10000)
    lin.table = fake
    assert L.milo_grouped_linear(C.byref(lin), fake, milo.MILO_F16, 0x7FFFFFFF, 16, fake, fake, fake,
                                 milo.MILO_F32, fake, 1 << 40, None, None) == milo.MILO_ERR_UNSUPPORTED_SHAPE
    assert L.milo_grouped_linear_noalloc(C.byref(lin), fake, milo.MILO_F16, 0x7FFFFFFF, 16, fake, fake, fake,
                                         milo.MILO_F32, None, None) == milo.MILO_ERR_UNSUPPORTED_SHAPE
    # MoE layer: the shared experts' rows count too
    layer = milo.milo_moe_layer(2048, 1408, 64, 2, 6, 64, 0, None)
    t_max = MAX_ROWS // 8
    assert L.milo_moe_workspace_bytes(C.byref(layer), t_max, C.byref(nb)) == 0 and nb.value > 0
    assert L.milo_moe_h_offset(C.byref(layer), t_max) > 0
    assert L.milo_moe_workspace_bytes(C.byref(layer), t_max + 1, C.byref(nb)) == milo.MILO_ERR_UNSUPPORTED_SHAPE
    assert L.milo_moe_h_offset(C.byref(layer), t_max + 1) == 0
    layer.table = fake
    assert L.milo_moe_forward(C.byref(layer), fake, milo.MILO_BF16, 0x7FFFFFFF, fake, fake, fake, fake, fake,
                              milo.MILO_F32, fake, 1 << 40, None, None) == milo.MILO_ERR_UNSUPPORTED_SHAPE
    # a layer struct whose top_k or n_shared preparation would reject
    bad = milo.milo_moe_layer(2048, 1408, 64, -1, 6, 64, 0, None)
    assert L.milo_moe_workspace_bytes(C.byref(bad), 16, C.byref(nb)) == milo.MILO_ERR_UNSUPPORTED_SHAPE
    bad = milo.milo_moe_layer(2048, 1408, 64, 0, 0, 64, 0, None)
    assert L.milo_moe_workspace_bytes(C.byref(bad), 16, C.byref(nb)) == milo.MILO_ERR_UNSUPPORTED_SHAPE
    # the router keeps the same limit
    assert L.milo_route(fake, 0x7FFFFFFF, 8, 2, 0, fake, fake, fake, fake, fake, None, None) == \
        milo.MILO_ERR_UNSUPPORTED_SHAPE


def test_weight_rows_bounded_so_the_tile_padding_fits_32_bits(milo):
    """A weight of N rows is stored in 64-row tiles; N up to 2^31 - 64 pads to
    a 32-bit count, and above it pack, unpack, dequantise, the size query and
    preparation refuse the shape (no device needed: all return before a
    launch)."""
    L = milo.lib()
    nb = C.c_size_t()
    n_max = 0x7FFFFFFF - 63
    assert L.milo_packed_bytes(n_max, 128, C.byref(nb)) == 0
    assert nb.value == (n_max // 64) * 3584
    for n in (n_max + 1, 0x7FFFFFFF):
        assert L.milo_packed_bytes(n, 128, C.byref(nb)) == milo.MILO_ERR_UNSUPPORTED_SHAPE
        assert b"2^31 - 64" in L.milo_last_error()
    fake = C.c_void_p(0x1000)
    assert L.milo_pack(fake, 0x7FFFFFFF, 128, 64, fake, None, None) == milo.MILO_ERR_UNSUPPORTED_SHAPE
    assert L.milo_unpack(fake, 0x7FFFFFFF, 128, fake, None) == milo.MILO_ERR_UNSUPPORTED_SHAPE
    assert L.milo_dequantize(fake, 0x7FFFFFFF, 128, fake, None) == milo.MILO_ERR_UNSUPPORTED_SHAPE
    w = milo.milo_qweight(0x10000, None, None, 0, 0)
    lin = milo.milo_linear(0x7FFFFFF0, 128, 1, 64, 0, None)   # a multiple of 16 above the bound
    assert L.milo_linear_prepare(C.byref(lin), C.byref(w), C.c_void_p(0x10000), 1 << 20) == \
        milo.MILO_ERR_UNSUPPORTED_SHAPE


def test_size_queries_check_the_struct_fields(milo):
    """The size queries (and the calls) check the shape fields as preparation
    does, and max_rank as preparation sets it: the planning divides by and
    multiplies with them (an expert count of 0 used to divide by zero)."""
    L = milo.lib()
    nb = C.c_size_t()
    U, I = milo.MILO_ERR_UNSUPPORTED_SHAPE, milo.MILO_ERR_INVALID_ARG
    for fields, want in (((256, 512, 0, 64, 0), U),        # no experts
                         ((256, 512, 257, 64, 0), U),      # too many experts
                         ((256, 512, 4, 32, 0), U),        # group
                         ((256, 500, 4, 64, 0), U),        # K % 128
                         ((250, 512, 4, 64, 0), U),        # N % 16
                         ((256, (1 << 24) + 128, 4, 64, 0), U),
                         ((256, 512, 4, 64, 12), I),       # max_rank not a multiple of 8
                         ((256, 512, 4, 64, 72), I),
                         ((256, 512, 4, 64, -8), I),
                         ((256, 512, 4, 64, 64), 0)):
        lin = milo.milo_linear(*fields, None)
        assert L.milo_linear_workspace_bytes(C.byref(lin), 16, 2, C.byref(nb)) == want, fields
    for fields, want in (((2048, 1408, 0, 0, 1, 64, 0), U),      # no routed experts
                         ((2048, 1408, 200, 57, 2, 64, 0), U),   # 257 experts
                         ((2048, 1408, 2**31 - 1, 1, 2, 64, 0), U),
                         ((2048, 1408, 4, 0, 5, 64, 0), U),      # top_k > n_routed
                         ((2048, 1408, 64, 0, 17, 64, 0), U),    # top_k > 16
                         ((2048, 1400, 8, 0, 2, 64, 0), U),      # inter % 128
                         ((2056, 1408, 8, 0, 2, 64, 0), U),      # hidden % 128
                         ((2048, 1408, 8, 0, 2, 64, 65), I),
                         ((2048, 1408, 64, 2, 6, 64, 64), 0)):
        lay = milo.milo_moe_layer(*fields, None)
        assert L.milo_moe_workspace_bytes(C.byref(lay), 16, C.byref(nb)) == want, fields
        assert (L.milo_moe_h_offset(C.byref(lay), 16) > 0) == (want == 0)


def test_size_queries_survive_arbitrary_fields(milo):
    """Seeded fuzz of the size queries over extreme field values: each returns
    a status (or 0 for the h offset), never crashes the process."""
    import random
    L = milo.lib()
    rnd = random.Random(7)
    vals = [-2**31, -129, -1, 0, 1, 7, 8, 16, 64, 100, 128, 1408, 4096, 14336, 2**20, 2**24, 2**30, 2**31 - 1]
    nb = C.c_size_t()
    for _ in range(3000):
        lin = milo.milo_linear(*(rnd.choice(vals) for _ in range(5)), None)
        T, k = rnd.choice(vals), rnd.choice(vals)
        assert L.milo_linear_workspace_bytes(C.byref(lin), T, k, C.byref(nb)) in range(5)
        lay = milo.milo_moe_layer(*(rnd.choice(vals) for _ in range(7)), None)
        assert L.milo_moe_workspace_bytes(C.byref(lay), T, C.byref(nb)) in range(5)
        L.milo_moe_h_offset(C.byref(lay), T)


def test_quantiser_validation_and_workspace(milo):
    L = milo.lib()
    fake = C.c_void_p(0x1000)
    # HQQ pack: K % 128, bad iteration count, non-positive beta, rank > 0 without U
    assert L.milo_hqq_pack(fake, None, None, 0, 16, 100, 20, 10.0, 1.01, fake, None, None, None) == \
        milo.MILO_ERR_UNSUPPORTED_SHAPE
    assert L.milo_hqq_pack(fake, None, None, 0, 16, 128, 1001, 10.0, 1.01, fake, None, None, None) == \
        milo.MILO_ERR_INVALID_ARG
    assert L.milo_hqq_pack(fake, None, None, 0, 16, 128, 20, 0.0, 1.01, fake, None, None, None) == \
        milo.MILO_ERR_INVALID_ARG
    assert L.milo_hqq_pack(fake, None, None, 8, 16, 128, 20, 10.0, 1.01, fake, None, None, None) == \
        milo.MILO_ERR_INVALID_ARG
    nb, nb2 = C.c_size_t(), C.c_size_t()
    p = milo.lorc_params(12)                      # rank not a multiple of 8
    assert L.milo_quantize_lorc_workspace(64, 128, C.byref(p), C.byref(nb)) == milo.MILO_ERR_UNSUPPORTED_SHAPE
    p = milo.lorc_params(16, sketch=24)           # sketch not a multiple of 16
    assert L.milo_quantize_lorc_workspace(64, 128, C.byref(p), C.byref(nb)) == milo.MILO_ERR_INVALID_ARG
    p = milo.lorc_params(16, sketch=8 * 16 + 16)  # sketch above 128
    assert L.milo_quantize_lorc_workspace(64, 128, C.byref(p), C.byref(nb)) == milo.MILO_ERR_INVALID_ARG
    p = milo.lorc_params(16, rounds=17)
    assert L.milo_quantize_lorc_workspace(64, 128, C.byref(p), C.byref(nb)) == milo.MILO_ERR_INVALID_ARG
    p = milo.lorc_params(16)
    assert L.milo_quantize_lorc_workspace(64, 128, C.byref(p), C.byref(nb)) == 0
    assert L.milo_quantize_lorc_workspace(640, 1280, C.byref(p), C.byref(nb2)) == 0
    assert 64 * 128 * 4 < nb.value < nb2.value
    # a workspace one byte short is refused before any launch
    assert L.milo_quantize_lorc(fake, 64, 128, C.byref(p), fake, C.c_void_p(0x10000), C.c_void_p(0x20000),
                                C.c_void_p(0x30000), None, C.c_void_p(0x40000), nb.value - 1, None, None) == \
        milo.MILO_ERR_WORKSPACE

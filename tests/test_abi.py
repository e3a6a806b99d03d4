"""The C-ABI library loads and exports every symbol include/vq.h declares,
and its host-only entry points answer without a GPU."""
import ctypes as C

import pytest

from bit_packed_index_b200 import build, vq


@pytest.fixture(scope="module")
def lib():
    build.build()
    return vq.lib()


def test_every_declared_symbol_is_exported(lib):
    names = vq.exported_names()
    assert set(names) == {"vq_dequant", "vq_repack_tile4", "vq_gemv_workspace_size", "vq_gemv",
                          "vq_gemv_noalloc", "vq_gemm_workspace_size", "vq_gemm",
                          "vq_status_string", "vq_last_cuda_error", "vq_abi_version",
                          "vq_kernel_launches", "vq_encode_workspace_size", "vq_encode",
                          "vq_gemv_multi_workspace_size", "vq_gemv_multi", "vq_rht",
                          "vq_gemv_rht_workspace_size", "vq_gemv_rht", "vq_hessian_workspace_size",
                          "vq_hessian"}
    for n in names:
        assert hasattr(lib, n), n


def test_host_only_calls(lib):
    assert lib.vq_abi_version() == 4
    assert C.sizeof(vq._Desc) == 104      # static_assert'ed in the library
    assert C.sizeof(vq._EncDesc) == 104
    assert vq.kernel_launches() == 0          # nothing launched in this process
    for s in range(7):
        assert lib.vq_status_string(s)
    assert lib.vq_status_string(99) == b"unknown status"


def test_descriptor_validation_needs_no_device(lib):
    """Malformed descriptors are rejected before any CUDA call."""
    d = vq._Desc()
    d.out_features, d.in_features, d.vec_dim, d.n_books = 4, 16, 0, 1   # d = 0
    d.log2k[0] = 8
    d.idx_row_words[0] = 4
    n = C.c_size_t(0)
    assert lib.vq_gemv_workspace_size(C.byref(d), 1, C.byref(n)) == vq.VQ_ERR_INVALID_ARG
    d.vec_dim = 8
    d.log2k[0] = 17                                                        # b > 16
    assert lib.vq_dequant(C.byref(d), None, 16, None) == vq.VQ_ERR_INVALID_ARG
    d.log2k[0] = 8
    d.idx_row_words[0] = 2                                                 # not a multiple of 4
    assert lib.vq_dequant(C.byref(d), None, 16, None) == vq.VQ_ERR_INVALID_ARG
    d.idx_row_words[0] = 4                                                 # but idx is NULL
    assert lib.vq_dequant(C.byref(d), None, 16, None) == vq.VQ_ERR_INVALID_ARG
    assert lib.vq_dequant(None, None, 16, None) == vq.VQ_ERR_INVALID_ARG


def _tiled_desc(n=1000, kin=64, b=16):
    """A well-formed tiled descriptor with fake (aligned, never dereferenced) pointers."""
    d = vq._Desc()
    d.out_features, d.in_features, d.vec_dim, d.n_books = n, kin, 8, 1
    d.log2k[0] = b
    d.idx[0] = 0x10000
    d.codebook[0] = 0x20000
    d.idx_row_words[0] = vq.tile4_words(n, b)
    d.idx_layout = vq.VQ_IDX_TILE4
    return d


def test_layout_field_validation_needs_no_device(lib):
    n = C.c_size_t(0)
    d = _tiled_desc()
    assert lib.vq_gemv_workspace_size(C.byref(d), 1, C.byref(n)) == vq.VQ_OK
    d.idx_layout = 2                                                       # unknown order
    assert lib.vq_gemv_workspace_size(C.byref(d), 1, C.byref(n)) == vq.VQ_ERR_INVALID_ARG
    d.idx_layout = vq.VQ_IDX_TILE4
    d.reserved = 1                                                         # must be zero
    assert lib.vq_gemv_workspace_size(C.byref(d), 1, C.byref(n)) == vq.VQ_ERR_INVALID_ARG
    d.reserved = 0
    d.idx_row_words[0] = vq.tile4_words(1000, 16) - 4                      # tile too short
    assert lib.vq_gemv_workspace_size(C.byref(d), 1, C.byref(n)) == vq.VQ_ERR_INVALID_ARG
    # the tile rule, not the row rule, applies: 64 columns need 4 words per row,
    # but 1000 records of 64 bits need 2000 words per tile
    d.idx_row_words[0] = 4
    assert lib.vq_gemv_workspace_size(C.byref(d), 1, C.byref(n)) == vq.VQ_ERR_INVALID_ARG


def test_output_bias_field_is_checked_on_the_host(lib):
    """The output bias pointer (ABI version 4) is optional, and an fp16 array
    that is not 2-byte aligned is refused before anything runs."""
    n = C.c_size_t(0)
    d = _tiled_desc()
    assert C.sizeof(vq._Desc) - vq._Desc.out_bias.offset == 8      # the last field
    d.out_bias = 0x30000
    assert lib.vq_gemv_workspace_size(C.byref(d), 1, C.byref(n)) == vq.VQ_OK
    d.out_bias = 0x30001
    assert lib.vq_gemv_workspace_size(C.byref(d), 1, C.byref(n)) == vq.VQ_ERR_ALIGNMENT
    assert lib.vq_gemm_workspace_size(C.byref(d), 64, vq.VQ_BF16, C.byref(n)) == vq.VQ_ERR_ALIGNMENT


def test_tiled_workspace_sizes(lib):
    """Batch 1 on a lookup-table-eligible tiled layer needs per-block row sums;
    batch 3 of a 2^16 book takes the tensor-core kernel (status word, the
    scaled fp16 copy of x as 16 rows of whole 64-element steps, the per-row
    scales and sums: 256 + 16 * 64 * 2 + 256 bytes for 8 vectors); layers no
    table kernel takes use the split-K gather kernel, which for this narrow
    layer runs one split (no workspace)."""
    n = C.c_size_t(0)
    d = _tiled_desc(n=1000, kin=64)
    assert lib.vq_gemv_workspace_size(C.byref(d), 1, C.byref(n)) == vq.VQ_OK
    assert n.value > 0 and n.value % (1001 * 4) == 0
    assert lib.vq_gemv_workspace_size(C.byref(d), 3, C.byref(n)) == vq.VQ_OK
    assert n.value == 256 + 16 * 64 * 2 + 256
    d.log2k[0] = 12                                    # a 2^12 book: the small-book table plan
    d.idx_row_words[0] = vq.tile4_words(1000, 12)
    assert lib.vq_gemv_workspace_size(C.byref(d), 1, C.byref(n)) == vq.VQ_OK
    assert n.value > 0 and n.value % (1001 * 4) == 0
    d.vec_dim, d.in_features = 16, 128                 # no table kernel for d = 16: split-K
    assert lib.vq_gemv_workspace_size(C.byref(d), 1, C.byref(n)) == vq.VQ_OK
    assert n.value == 0


def test_repack_argument_checks_need_no_device(lib):
    src = _tiled_desc()
    dst = (C.c_void_p * 2)(0x30000, 0)
    tw = (C.c_int64 * 2)(vq.tile4_words(1000, 16), 0)
    assert lib.vq_repack_tile4(C.byref(src), dst, tw, None) == vq.VQ_ERR_INVALID_ARG  # src tiled
    src.idx_layout = vq.VQ_IDX_ROWS
    src.idx_row_words[0] = 32
    tw[0] = vq.tile4_words(1000, 16) - 4
    assert lib.vq_repack_tile4(C.byref(src), dst, tw, None) == vq.VQ_ERR_INVALID_ARG  # short tile
    tw[0] = vq.tile4_words(1000, 16)
    dst[0] = None
    assert lib.vq_repack_tile4(C.byref(src), dst, tw, None) == vq.VQ_ERR_INVALID_ARG  # no dst
    dst[0] = 0x30008
    assert lib.vq_repack_tile4(C.byref(src), dst, tw, None) == vq.VQ_ERR_ALIGNMENT


def test_table_batch_limit_needs_no_device(lib, monkeypatch):
    """Small batches of a 2^16-book tiled layer plan the per-row table passes
    (per-block row sums) up to batch 2, then the split-K kernel; the
    VQ_LUT_MAX_BATCH override moves that limit."""
    n = C.c_size_t(0)
    d = _tiled_desc(n=1000, kin=64 * 8)
    table = lambda v: v > 0 and v % (1001 * 4) == 0
    for batch, want in ((1, True), (2, True), (3, False)):
        assert lib.vq_gemv_workspace_size(C.byref(d), batch, C.byref(n)) == vq.VQ_OK
        assert table(n.value) == want, (batch, n.value)
    monkeypatch.setenv("VQ_LUT_MAX_BATCH", "0")
    assert lib.vq_gemv_workspace_size(C.byref(d), 1, C.byref(n)) == vq.VQ_OK
    assert not table(n.value)


def test_small_book_table_limit_needs_no_device(lib):
    """Tiled layers with a 2^12 book take the per-row table passes up to
    batch 3 when rows hold at most 1024 vectors and up to batch 5 when they
    hold more; larger batches plan the small-book tensor-core kernel (status
    word, scaled x, per-row scales; no per-block row sums)."""
    n = C.c_size_t(0)
    table = lambda v: v > 0 and v % (1001 * 4) == 0
    for kin, last in ((8 * 1024, 3), (8 * 1025, 5)):
        d = _tiled_desc(n=1000, kin=kin, b=12)
        for batch in range(1, 9):
            assert lib.vq_gemv_workspace_size(C.byref(d), batch, C.byref(n)) == vq.VQ_OK
            assert table(n.value) == (batch <= last), (kin, batch, n.value)


def test_encode_workspace_and_validation_need_no_device(lib):
    """vq_encode_workspace_size: control words + per book the prepared operand
    (K padded to 1024, 32 bytes per centroid) and the fp64 copy (8 bytes per
    component) + unpacked indices per book + the exact-pass list, each rounded
    up to 256 bytes; malformed descriptions are rejected before any CUDA
    call."""
    r256 = lambda x: -(-x // 256) * 256
    n, kin, d = 300, 8 * 100 + 5, 8
    nvec = -(-kin // d)
    got = vq.encode_workspace_size(n, kin, [16, 4], d)
    want = (256 + r256(65536 * 32) + r256(65536 * d * 8) + r256(1024 * 32) + r256(16 * d * 8)
            + 3 * r256(n * nvec * 4))
    assert got == want
    assert vq.encode_workspace_size(0, kin, [16], d) == 0
    assert vq.encode_workspace_size(n, 0, [16], d) == 0
    e = vq._EncDesc()
    e.out_features, e.in_features, e.vec_dim, e.n_books = 4, 16, 8, 1
    e.log2k[0] = 8
    e.ldw = 16
    e.idx_row_words[0] = 4
    n_ = C.c_size_t(0)
    assert lib.vq_encode_workspace_size(C.byref(e), C.byref(n_)) == vq.VQ_OK
    for field, bad in (("vec_dim", 15), ("vec_dim", 0), ("n_books", 3), ("ldw", 15)):
        old = getattr(e, field)
        setattr(e, field, bad)
        assert lib.vq_encode_workspace_size(C.byref(e), C.byref(n_)) == vq.VQ_ERR_INVALID_ARG, field
        setattr(e, field, old)
    e.log2k[0] = 17
    assert lib.vq_encode_workspace_size(C.byref(e), C.byref(n_)) == vq.VQ_ERR_INVALID_ARG
    e.log2k[0] = 8
    e.idx_row_words[0] = 2                       # short and not a multiple of 4
    assert lib.vq_encode_workspace_size(C.byref(e), C.byref(n_)) == vq.VQ_ERR_INVALID_ARG
    e.idx_row_words[0] = 4
    # vq_encode itself: NULL buffers with data are rejected before any launch
    assert lib.vq_encode(C.byref(e), None, 0, None) == vq.VQ_ERR_INVALID_ARG


def test_weighted_encode_workspace_and_validation(lib):
    """With a Hessian the workspace adds, per book, one fp32 c^T H_j c value
    per (whole block of channels j, padded centroid); vec_dim > 8, a short
    ldh or a misaligned H is refused on the host."""
    r256 = lambda x: -(-x // 256) * 256
    n, kin, d = 300, 8 * 100 + 5, 8
    plain = vq.encode_workspace_size(n, kin, [16, 4], d)
    got = vq.encode_workspace_size(n, kin, [16, 4], d, hessian=True)
    assert got == plain + r256(100 * 65536 * 4) + r256(100 * 4) + r256(100 * 1024 * 4) + r256(100 * 4)
    e = vq._EncDesc()
    e.out_features, e.in_features, e.vec_dim, e.n_books = 4, 16, 8, 1
    e.log2k[0] = 8
    e.ldw = 16
    e.idx_row_words[0] = 4
    e.h, e.ldh = 0x40000, 16
    n_ = C.c_size_t(0)
    assert lib.vq_encode_workspace_size(C.byref(e), C.byref(n_)) == vq.VQ_OK
    e.ldh = 15
    assert lib.vq_encode_workspace_size(C.byref(e), C.byref(n_)) == vq.VQ_ERR_INVALID_ARG
    e.ldh = 16
    e.h = 0x40002
    assert lib.vq_encode_workspace_size(C.byref(e), C.byref(n_)) == vq.VQ_ERR_ALIGNMENT
    e.h = 0x40000
    e.vec_dim, e.in_features, e.ldw, e.ldh = 9, 18, 18, 18
    e.idx_row_words[0] = 4
    assert lib.vq_encode_workspace_size(C.byref(e), C.byref(n_)) == vq.VQ_ERR_UNSUPPORTED


def test_new_entry_points_validate_before_any_device_call(lib):
    """Host-side checks of vq_rht, vq_hessian(_workspace_size), vq_gemv_rht
    and vq_gemv_multi: malformed arguments return a status and launch nothing."""
    P = C.c_void_p
    # vq_rht: negative sizes, short strides, bad dtype, NULL buffers with data
    assert lib.vq_rht(None, vq.VQ_FP32, -1, 8, 8, None, 0, None, vq.VQ_FP32, 8, None) == vq.VQ_ERR_INVALID_ARG
    assert lib.vq_rht(None, vq.VQ_FP32, 2, 8, 4, None, 0, None, vq.VQ_FP32, 8, None) == vq.VQ_ERR_INVALID_ARG
    assert lib.vq_rht(None, 7, 2, 8, 8, None, 0, None, vq.VQ_FP32, 8, None) == vq.VQ_ERR_INVALID_ARG
    assert lib.vq_rht(None, vq.VQ_FP32, 2, 8, 8, None, 0, None, vq.VQ_FP32, 8, None) == vq.VQ_ERR_INVALID_ARG
    assert lib.vq_rht(None, vq.VQ_FP32, 0, 8, 8, None, 0, None, vq.VQ_FP32, 8, None) == vq.VQ_OK
    assert lib.vq_rht(P(16), vq.VQ_FP32, 70000, 8, 8, P(16), 0, P(16), vq.VQ_FP32, 8, None) == \
        vq.VQ_ERR_UNSUPPORTED
    assert lib.vq_rht(P(18), vq.VQ_FP32, 2, 8, 8, P(16), 0, P(16), vq.VQ_FP32, 8, None) == vq.VQ_ERR_ALIGNMENT
    # vq_hessian: workspace arithmetic (X^T copy rows padded to 8 tokens) and checks
    n = C.c_size_t(0)
    assert lib.vq_hessian_workspace_size(100, 64, C.byref(n)) == vq.VQ_OK
    assert n.value == 256 + (-(-(64 * 104 * 2) // 256) * 256) + 256
    assert lib.vq_hessian_workspace_size(-1, 64, C.byref(n)) == vq.VQ_ERR_INVALID_ARG
    assert lib.vq_hessian(None, vq.VQ_BF16, 0, 64, 64, None, 64, None, 0, None) == vq.VQ_ERR_INVALID_ARG
    assert lib.vq_hessian(None, vq.VQ_BF16, 10, 64, 32, None, 64, None, 0, None) == vq.VQ_ERR_INVALID_ARG
    assert lib.vq_hessian(None, vq.VQ_FP32, 10, 64, 64, None, 64, None, 0, None) == vq.VQ_ERR_INVALID_ARG
    assert lib.vq_hessian(P(16), vq.VQ_BF16, 10, 64, 64, P(16), 64, None, 0, None) == vq.VQ_ERR_WORKSPACE
    # vq_gemv_multi / vq_gemv_rht: empty or malformed descriptions
    arr = (C.c_void_p * 1)()
    assert lib.vq_gemv_multi(arr, 0, None, vq.VQ_BF16, 1, 8, None, vq.VQ_BF16, None, None, 0, None) == \
        vq.VQ_ERR_INVALID_ARG
    assert lib.vq_gemv_multi(None, 2, None, vq.VQ_BF16, 1, 8, None, vq.VQ_BF16, None, None, 0, None) == \
        vq.VQ_ERR_INVALID_ARG
    d = vq._Desc()
    d.out_features, d.in_features, d.vec_dim, d.n_books = 4, 16, 0, 1   # d = 0
    assert lib.vq_gemv_rht(C.byref(d), None, None, None, vq.VQ_BF16, 1, 16, None, vq.VQ_BF16, 4, None, 0,
                           None) == vq.VQ_ERR_INVALID_ARG


def test_noalloc_scratch_size_matches_the_header():
    """The binding's NOALLOC_SCRATCH_BYTES is the header's
    VQ_NOALLOC_SCRATCH_BYTES (the tests size their layers against it)."""
    import re
    with open(vq.HEADER) as fh:
        m = re.search(r"#define\s+VQ_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", fh.read())
    assert m, "macro not found"
    assert vq.NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))

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
                          "vq_kernel_launches"}
    for n in names:
        assert hasattr(lib, n), n


def test_host_only_calls(lib):
    assert lib.vq_abi_version() == 2
    assert C.sizeof(vq._Desc) == 96       # static_assert'ed in the library
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


def test_tiled_workspace_sizes(lib):
    """Batch 1 on a lookup-table-eligible tiled layer needs per-block row sums;
    batch 3 of a 2^16 book and layers no table kernel takes use the split-K
    gather kernel, which for this narrow layer runs one split (no workspace)."""
    n = C.c_size_t(0)
    d = _tiled_desc(n=1000, kin=64)
    assert lib.vq_gemv_workspace_size(C.byref(d), 1, C.byref(n)) == vq.VQ_OK
    assert n.value > 0 and n.value % (1001 * 4) == 0
    assert lib.vq_gemv_workspace_size(C.byref(d), 3, C.byref(n)) == vq.VQ_OK
    assert n.value == 0
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

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
    assert set(names) == {"vq_dequant", "vq_gemv_workspace_size", "vq_gemv", "vq_gemv_noalloc",
                          "vq_gemm_workspace_size", "vq_gemm", "vq_status_string",
                          "vq_last_cuda_error", "vq_abi_version", "vq_kernel_launches"}
    for n in names:
        assert hasattr(lib, n), n


def test_host_only_calls(lib):
    assert lib.vq_abi_version() == 1
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

"""CPU oracle for the bit-packed VQ/RVQ linear layer -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product (``bit_packed_index_b200``) never
does, and nothing here imports the product: the two share only the seeded
input generators in ``synth``.

The arithmetic lives in ``vq_oracle.c`` (plain C, built here with gcc into
``liboracle.so``); this module marshals numpy arrays for it.  What each
routine computes, and the page passage it follows, is documented in the C
file.  Functions pinned by the not-gpu tests: the conversions, unpack/pack
(row order and tiled order), dequant, matmul/linear, the encoders, the
randomized Hadamard transform and the Hessian.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "vq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

GCC_FLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
             "-shared", "-fPIC", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source (skipped when up to date)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *GCC_FLAGS, "-o", tmp, _SRC, "-lm"], check=True)
    os.replace(tmp, _LIB)
    return _LIB


class _Layer(C.Structure):
    _fields_ = [
        ("out_features", C.c_int64), ("in_features", C.c_int64),
        ("d", C.c_int32), ("n_books", C.c_int32), ("log2k", C.c_int32 * 2),
        ("idx", C.c_void_p * 2), ("row_words", C.c_int64 * 2),
        ("codebook", C.c_void_p * 2), ("scale", C.c_void_p), ("bias", C.c_void_p),
        ("out_bias", C.c_void_p),
    ]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = C.CDLL(build())
            P, I64, I32 = C.c_void_p, C.c_int64, C.c_int
            sig = {
                "vqo_f32_to_f16_array": [P, P, I64], "vqo_f16_to_f32_array": [P, P, I64],
                "vqo_f32_to_bf16_array": [P, P, I64], "vqo_bf16_to_f32_array": [P, P, I64],
                "vqo_unpack": [P, I64, I64, I32, I64, P],
                "vqo_pack": [P, I64, I64, I32, I64, P],
                "vqo_unpack_tile4": [P, I64, I64, I32, I64, P],
                "vqo_pack_tile4": [P, I64, I64, I32, I64, P],
                "vqo_dequant": [P, P, I64],
                "vqo_dequant_rows": [P, P, I64, P, I64],
                "vqo_matmul": [I64, I64, I64, P, I32, I64, P, I64, P, I64],
                "vqo_linear": [P, P, I32, I64, I64, P, I64, P, I64],
                "vqo_encode": [P, I64, I32, P, I64, P],
                "vqo_encode_residual": [P, I64, I32, P, I64, P, I64, P, P],
                "vqo_encode_joint": [P, I64, I32, P, I64, P, I64, P, P],
                "vqo_encode_h": [P, I64, I32, P, P, I64, P],
                "vqo_encode_h_residual": [P, I64, I32, P, P, I64, P, I64, P, P],
                "vqo_rht": [P, I64, I64, P, I32, P],
                "vqo_hessian": [P, I32, I64, I64, I64, P],
                "vqo_rht_block": [I64],
                "vqo_num_threads": [],
            }
            for name, args in sig.items():
                fn = getattr(lib, name)
                fn.argtypes = args
                fn.restype = None if name.endswith("_array") else C.c_int
            lib.vqo_rht_block.restype = C.c_int64
            _lib = lib
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _check(rc: int, what: str):
    if rc:
        raise ValueError(f"oracle {what} rejected its arguments (code {rc})")


# -- conversions ------------------------------------------------------------

def f32_to_f16(a) -> np.ndarray:
    a = np.ascontiguousarray(a, np.float32)
    out = np.empty(a.shape, np.uint16)
    _load().vqo_f32_to_f16_array(_p(a), _p(out), a.size)
    return out


def f16_to_f32(h) -> np.ndarray:
    h = np.ascontiguousarray(h, np.uint16)
    out = np.empty(h.shape, np.float32)
    _load().vqo_f16_to_f32_array(_p(h), _p(out), h.size)
    return out


def f32_to_bf16(a) -> np.ndarray:
    a = np.ascontiguousarray(a, np.float32)
    out = np.empty(a.shape, np.uint16)
    _load().vqo_f32_to_bf16_array(_p(a), _p(out), a.size)
    return out


def bf16_to_f32(h) -> np.ndarray:
    h = np.ascontiguousarray(h, np.uint16)
    out = np.empty(h.shape, np.float32)
    _load().vqo_bf16_to_f32_array(_p(h), _p(out), h.size)
    return out


# -- index streams ----------------------------------------------------------

def unpack(words: np.ndarray, b: int, nvec: int) -> np.ndarray:
    words = np.ascontiguousarray(words, np.uint32)
    n, rw = words.shape
    out = np.empty((n, nvec), np.uint32)
    _check(_load().vqo_unpack(_p(words), n, rw, b, nvec, _p(out)), "unpack")
    return out


def pack(idx: np.ndarray, b: int, row_words: Optional[int] = None) -> np.ndarray:
    idx = np.ascontiguousarray(idx, np.uint32)
    n, nvec = idx.shape
    if row_words is None:
        row_words = -(-(nvec * b) // 128) * 4
    out = np.empty((n, row_words), np.uint32)
    _check(_load().vqo_pack(_p(idx), n, nvec, b, row_words, _p(out)), "pack")
    return out


def tile4_words(n_rows: int, b: int) -> int:
    """Smallest 16-byte-padded tile of the tiled order: n_rows records of 4 fields."""
    return -(-(n_rows * 4 * b) // 128) * 4


def unpack_tile4(words: np.ndarray, b: int, n_rows: int, nvec: int) -> np.ndarray:
    """Indices [n_rows][nvec] from a tiled stream [ceil(nvec/4)][tile_words]."""
    words = np.ascontiguousarray(words, np.uint32)
    tile_words = words.shape[1]
    out = np.empty((n_rows, nvec), np.uint32)
    _check(_load().vqo_unpack_tile4(_p(words), n_rows, tile_words, b, nvec, _p(out)),
           "unpack_tile4")
    return out


def pack_tile4(idx: np.ndarray, b: int, tile_words: Optional[int] = None) -> np.ndarray:
    """The tiled stream [ceil(nvec/4)][tile_words] of idx [N][nvec] (zero padding)."""
    idx = np.ascontiguousarray(idx, np.uint32)
    n, nvec = idx.shape
    if tile_words is None:
        tile_words = tile4_words(n, b)
    out = np.empty((-(-nvec // 4), tile_words), np.uint32)
    _check(_load().vqo_pack_tile4(_p(idx), n, nvec, b, tile_words, _p(out)), "pack_tile4")
    return out


# -- the layer --------------------------------------------------------------

def _layer_struct(layer):
    s = layer.spec
    keep = []
    L = _Layer()
    L.out_features, L.in_features, L.d, L.n_books = s.out_features, s.in_features, s.d, s.n_books
    for m in range(s.n_books):
        w = np.ascontiguousarray(layer.idx_words[m], np.uint32)
        c = np.ascontiguousarray(layer.codebooks[m], np.uint16)
        keep += [w, c]
        L.log2k[m] = s.log2k[m]
        L.idx[m] = w.ctypes.data
        L.row_words[m] = layer.row_words[m]
        L.codebook[m] = c.ctypes.data
    for name in ("scale", "bias", "out_bias"):
        a = getattr(layer, name, None)
        if a is not None:
            a = np.ascontiguousarray(a, np.uint16)
            keep.append(a)
            setattr(L, name, a.ctypes.data)
    return L, keep


def dequant(layer, rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """W_hat as fp16 bits [N][Kin] (or [len(rows)][Kin])."""
    L, keep = _layer_struct(layer)
    kin = layer.spec.in_features
    if rows is None:
        w = np.zeros((layer.spec.out_features, kin), np.uint16)
        _check(_load().vqo_dequant(C.byref(L), _p(w), kin), "dequant")
    else:
        r = np.ascontiguousarray(rows, np.int64)
        w = np.zeros((r.size, kin), np.uint16)
        _check(_load().vqo_dequant_rows(C.byref(L), _p(r), r.size, _p(w), kin), "dequant_rows")
    del keep
    return w


def matmul(x: np.ndarray, w: np.ndarray, kin: Optional[int] = None, x_is_fp16: bool = False) -> np.ndarray:
    """fp64 y[M][N] = x[M][:kin] . w[N][:kin]^T (x bf16 or fp16 bits, w fp16 bits)."""
    x = np.ascontiguousarray(x, np.uint16)
    w = np.ascontiguousarray(w, np.uint16)
    kin = w.shape[1] if kin is None else kin
    M, N = x.shape[0], w.shape[0]
    y = np.empty((M, N), np.float64)
    _check(_load().vqo_matmul(M, N, kin, _p(x), int(x_is_fp16), x.shape[1], _p(w), w.shape[1],
                              _p(y), N), "matmul")
    return y


def linear(layer, x: np.ndarray, rows: Optional[Sequence[int]] = None,
           x_is_fp16: bool = False, out_bias: Optional[np.ndarray] = None) -> np.ndarray:
    """Forward pass in fp64: y[M][n] for all output rows, or for ``rows``.
    The output bias (fp16 bits [N]) is ``out_bias`` when given, else the
    layer's ``out_bias`` attribute (if any)."""
    L, keep = _layer_struct(layer)
    if out_bias is not None:
        ob = np.ascontiguousarray(out_bias, np.uint16)
        if ob.shape != (layer.spec.out_features,):
            raise ValueError("out_bias must hold out_features fp16 values")
        keep.append(ob)
        L.out_bias = ob.ctypes.data
    x = np.ascontiguousarray(x, np.uint16)
    M = x.shape[0]
    if rows is None:
        n_out, rp = layer.spec.out_features, None
    else:
        r = np.ascontiguousarray(rows, np.int64)
        keep.append(r)
        n_out, rp = r.size, _p(r)
    y = np.empty((M, n_out), np.float64)
    _check(_load().vqo_linear(C.byref(L), _p(x), int(x_is_fp16), M, x.shape[1], rp, n_out,
                              _p(y), n_out), "linear")
    del keep
    return y


# -- encoders (tests only) --------------------------------------------------

def encode(v: np.ndarray, book: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, np.float64)
    book = np.ascontiguousarray(book, np.uint16)
    nv, d = v.shape
    idx = np.empty(nv, np.uint32)
    _check(_load().vqo_encode(_p(v), nv, d, _p(book), book.shape[0], _p(idx)), "encode")
    return idx


def encode_residual(v: np.ndarray, book1: np.ndarray, book2: np.ndarray):
    v = np.ascontiguousarray(v, np.float64)
    b1 = np.ascontiguousarray(book1, np.uint16)
    b2 = np.ascontiguousarray(book2, np.uint16)
    nv, d = v.shape
    i1 = np.empty(nv, np.uint32)
    i2 = np.empty(nv, np.uint32)
    _check(_load().vqo_encode_residual(_p(v), nv, d, _p(b1), b1.shape[0], _p(b2), b2.shape[0],
                                       _p(i1), _p(i2)), "encode_residual")
    return i1, i2


def encode_h(v: np.ndarray, hb: np.ndarray, book: np.ndarray) -> np.ndarray:
    """Hessian-weighted nearest centroid: v [nv][d], hb [nv][d][d] (each
    vector's sub-matrix of H), book fp16 bits [K][d]."""
    v = np.ascontiguousarray(v, np.float64)
    hb = np.ascontiguousarray(hb, np.float64)
    book = np.ascontiguousarray(book, np.uint16)
    nv, d = v.shape
    if hb.shape != (nv, d, d):
        raise ValueError("hb must be [nv][d][d]")
    idx = np.empty(nv, np.uint32)
    _check(_load().vqo_encode_h(_p(v), nv, d, _p(hb), _p(book), book.shape[0], _p(idx)), "encode_h")
    return idx


def encode_h_residual(v: np.ndarray, hb: np.ndarray, book1: np.ndarray, book2: np.ndarray):
    v = np.ascontiguousarray(v, np.float64)
    hb = np.ascontiguousarray(hb, np.float64)
    b1 = np.ascontiguousarray(book1, np.uint16)
    b2 = np.ascontiguousarray(book2, np.uint16)
    nv, d = v.shape
    if hb.shape != (nv, d, d):
        raise ValueError("hb must be [nv][d][d]")
    i1 = np.empty(nv, np.uint32)
    i2 = np.empty(nv, np.uint32)
    _check(_load().vqo_encode_h_residual(_p(v), nv, d, _p(hb), _p(b1), b1.shape[0], _p(b2), b2.shape[0],
                                         _p(i1), _p(i2)), "encode_h_residual")
    return i1, i2


def hessian_blocks(h: np.ndarray, kin: int, d: int, rows: int) -> tuple:
    """The sub-matrices H_v of a layer's vectors, in the encoder's vector
    order (row o, vector j): for whole vectors the d x d block of h on
    channels j*d .. j*d+d-1, and for a partial last vector (kin % d != 0)
    the rem x rem block on its valid channels.  Returns (full, last): full
    [rows * (kin // d)][d][d] and last [rows][rem][rem] (None if rem == 0)."""
    h = np.asarray(h, np.float64)
    nfull, rem = kin // d, kin % d
    blocks = np.stack([h[j * d:(j + 1) * d, j * d:(j + 1) * d] for j in range(nfull)]) if nfull else \
        np.zeros((0, d, d))
    full = np.ascontiguousarray(np.broadcast_to(blocks[None], (rows, nfull, d, d)).reshape(rows * nfull, d, d))
    last = None
    if rem:
        b = h[nfull * d:kin, nfull * d:kin]
        last = np.ascontiguousarray(np.broadcast_to(b[None], (rows, rem, rem)))
    return full, last


def encode_joint(v: np.ndarray, book1: np.ndarray, book2: np.ndarray):
    v = np.ascontiguousarray(v, np.float64)
    b1 = np.ascontiguousarray(book1, np.uint16)
    b2 = np.ascontiguousarray(book2, np.uint16)
    nv, d = v.shape
    i1 = np.empty(nv, np.uint32)
    i2 = np.empty(nv, np.uint32)
    _check(_load().vqo_encode_joint(_p(v), nv, d, _p(b1), b1.shape[0], _p(b2), b2.shape[0],
                                    _p(i1), _p(i2)), "encode_joint")
    return i1, i2


# -- randomized Hadamard transform (tests only) ----------------------------

def rht_block(n: int) -> int:
    return int(_load().vqo_rht_block(n))


def rht(x: np.ndarray, signs: np.ndarray, inverse: bool = False) -> np.ndarray:
    """Rows of x (fp64 [rows][n]) through the randomized Hadamard transform with
    the sign bits `signs` (uint32 words, bit t set -> -1)."""
    x = np.ascontiguousarray(np.atleast_2d(x), np.float64)
    signs = np.ascontiguousarray(signs, np.uint32)
    out = np.empty_like(x)
    _check(_load().vqo_rht(_p(x), x.shape[0], x.shape[1], _p(signs), int(inverse), _p(out)), "rht")
    return out


# -- Hessian collection (tests only) -----------------------------------------

def hessian(x: np.ndarray, x_is_fp16: bool = False) -> np.ndarray:
    """Normalised, damped Hessian (fp64 [d][d]) of activations x: bf16 (or fp16)
    bits [n_tokens][d]."""
    x = np.ascontiguousarray(x, np.uint16)
    n, d = x.shape
    out = np.empty((d, d), np.float64)
    _check(_load().vqo_hessian(_p(x), int(x_is_fp16), n, d, d, _p(out)), "hessian")
    return out


def num_threads() -> int:
    return int(_load().vqo_num_threads())

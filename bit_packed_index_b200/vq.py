"""Python binding of libvq (include/vq.h): argument marshalling only.

Every computation runs in the CUDA kernels behind the C ABI; this module only
turns torch tensors into pointers, sizes and the current CUDA stream.  There
is no fallback: if ``libvq.so`` is missing or fails to load, every call raises.

Names follow the C ABI: ``dequant``, ``gemv``, ``gemv_multi``, ``gemv_rht``,
``rht``, ``gemm``, ``repack_tile4``, ``encode``, ``hessian``, plus the
workspace size queries.  A ``Layer`` holds the device tensors of one
quantised layer (packed index streams in row order or in the tiled order,
fp16 codebooks, optional fp16 scale and bias, optional fp16 output bias).
"""
from __future__ import annotations

import ctypes as C
import os
import re
import threading
from dataclasses import dataclass, field
from typing import List, Optional, Sequence

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libvq.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "vq.h")

VQ_OK, VQ_ERR_INVALID_ARG, VQ_ERR_UNSUPPORTED, VQ_ERR_ALIGNMENT = 0, 1, 2, 3
VQ_ERR_WORKSPACE, VQ_ERR_CUDA, VQ_ERR_TIMEOUT = 4, 5, 6
VQ_BF16, VQ_FP16, VQ_FP32 = 0, 1, 2
VQ_IDX_ROWS, VQ_IDX_TILE4 = 0, 1
_LAYOUT = {"rows": VQ_IDX_ROWS, "tile4": VQ_IDX_TILE4}

_DTYPE = {torch.bfloat16: VQ_BF16, torch.float16: VQ_FP16, torch.float32: VQ_FP32}


class VQError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str, cuda_error: int = 0):
        super().__init__(f"{fn}: {msg} (status {status}"
                         + (f", cudaError {cuda_error})" if status == VQ_ERR_CUDA else ")"))
        self.status = status
        self.cuda_error = cuda_error


class _Desc(C.Structure):
    _fields_ = [
        ("out_features", C.c_int32), ("in_features", C.c_int32),
        ("vec_dim", C.c_int32), ("n_books", C.c_int32), ("log2k", C.c_int32 * 2),
        ("idx", C.c_void_p * 2), ("idx_row_words", C.c_int64 * 2),
        ("codebook", C.c_void_p * 2), ("scale", C.c_void_p), ("bias", C.c_void_p),
        ("idx_layout", C.c_int32), ("reserved", C.c_int32), ("out_bias", C.c_void_p),
    ]


class _EncDesc(C.Structure):
    _fields_ = [
        ("out_features", C.c_int32), ("in_features", C.c_int32),
        ("vec_dim", C.c_int32), ("n_books", C.c_int32), ("log2k", C.c_int32 * 2),
        ("w", C.c_void_p), ("ldw", C.c_int64),
        ("codebook", C.c_void_p * 2),
        ("idx", C.c_void_p * 2), ("idx_row_words", C.c_int64 * 2),
        ("h", C.c_void_p), ("ldh", C.c_int64),
    ]


_lock = threading.Lock()
_lib = None


def exported_names() -> List[str]:
    """Function names the header declares (VQ_API ...)."""
    with open(HEADER) as fh:
        text = fh.read()
    return re.findall(r"VQ_API\s+[\w\s\*]+?\b(vq_\w+)\s*\(", text)


def lib():
    """Load libvq.so (raises if it is missing: there is no other code path)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"libvq.so not found at {LIB_PATH}; build it with "
                                   "`python bit_packed_index_b200/build.py`")
            L = C.CDLL(LIB_PATH)
            P, I32, I64, SZ = C.c_void_p, C.c_int32, C.c_int64, C.c_size_t
            L.vq_dequant.argtypes = [P, P, I64, P]
            L.vq_gemv_workspace_size.argtypes = [P, I32, C.POINTER(SZ)]
            L.vq_gemv.argtypes = [P, P, C.c_int, I32, I64, P, C.c_int, I64, P, SZ, P]
            L.vq_gemv_noalloc.argtypes = [P, P, C.c_int, I32, I64, P, C.c_int, I64, P]
            L.vq_gemm_workspace_size.argtypes = [P, I32, C.c_int, C.POINTER(SZ)]
            L.vq_gemm.argtypes = [P, P, C.c_int, I32, I64, P, C.c_int, I64, P, SZ, P]
            L.vq_repack_tile4.argtypes = [P, C.POINTER(P), C.POINTER(I64), P]
            L.vq_gemv_multi_workspace_size.argtypes = [P, I32, I32, C.POINTER(SZ)]
            L.vq_gemv_multi.argtypes = [P, I32, P, C.c_int, I32, I64, P, C.c_int, P, P, SZ, P]
            L.vq_rht.argtypes = [P, C.c_int, I32, I32, I64, P, I32, P, C.c_int, I64, P]
            L.vq_gemv_rht_workspace_size.argtypes = [P, I32, C.POINTER(SZ)]
            L.vq_gemv_rht.argtypes = [P, P, P, P, C.c_int, I32, I64, P, C.c_int, I64, P, SZ, P]
            L.vq_hessian_workspace_size.argtypes = [I32, I32, C.POINTER(SZ)]
            L.vq_hessian.argtypes = [P, C.c_int, I32, I32, I64, P, I64, P, SZ, P]
            L.vq_encode_workspace_size.argtypes = [P, C.POINTER(SZ)]
            L.vq_encode.argtypes = [P, P, SZ, P]
            for fn in ("vq_dequant", "vq_gemv_workspace_size", "vq_gemv", "vq_gemv_noalloc",
                       "vq_gemm_workspace_size", "vq_gemm", "vq_repack_tile4",
                       "vq_encode_workspace_size", "vq_encode", "vq_gemv_multi_workspace_size",
                       "vq_gemv_multi", "vq_rht", "vq_gemv_rht_workspace_size", "vq_gemv_rht",
                       "vq_hessian_workspace_size", "vq_hessian"):
                getattr(L, fn).restype = C.c_int
            L.vq_status_string.argtypes = [C.c_int]
            L.vq_status_string.restype = C.c_char_p
            L.vq_last_cuda_error.restype = C.c_int
            L.vq_abi_version.restype = C.c_int
            L.vq_kernel_launches.restype = C.c_uint64
            _lib = L
    return _lib


def _check(fn: str, status: int):
    if status != VQ_OK:
        L = lib()
        raise VQError(fn, status, L.vq_status_string(status).decode(),
                      L.vq_last_cuda_error() if status == VQ_ERR_CUDA else 0)


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else C.c_void_p(t.data_ptr())


@dataclass
class Layer:
    """Device tensors of one quantised layer (see include/vq.h)."""
    out_features: int
    in_features: int
    vec_dim: int
    log2k: List[int]
    idx: List[torch.Tensor]            # int32 views of uint32 words: [N][row_words] in row
                                       # order, [ceil(nvec/4)][tile_words] tiled
    codebooks: List[torch.Tensor]      # float16 [K][d]
    scale: Optional[torch.Tensor] = None   # float16 [N]
    bias: Optional[torch.Tensor] = None    # float16 [N]
    layout: str = "rows"               # "rows" or "tile4"
    out_bias: Optional[torch.Tensor] = None   # float16 [N], added to y after the product
    _desc: Optional[_Desc] = field(default=None, repr=False)

    @property
    def n_books(self) -> int:
        return len(self.log2k)

    @property
    def device(self) -> torch.device:
        return self.idx[0].device

    def desc(self) -> _Desc:
        if self._desc is None:
            d = _Desc()
            d.out_features, d.in_features = self.out_features, self.in_features
            d.vec_dim, d.n_books = self.vec_dim, self.n_books
            for m in range(self.n_books):
                d.log2k[m] = self.log2k[m]
                d.idx[m] = self.idx[m].data_ptr()
                d.idx_row_words[m] = self.idx[m].stride(0) if self.idx[m].shape[1] > 0 else 0
                d.codebook[m] = self.codebooks[m].data_ptr()
            d.scale = None if self.scale is None else self.scale.data_ptr()
            d.bias = None if self.bias is None else self.bias.data_ptr()
            d.idx_layout = _LAYOUT[self.layout]
            d.out_bias = None if self.out_bias is None else self.out_bias.data_ptr()
            self._desc = d
        return self._desc

    @classmethod
    def from_host(cls, out_features: int, in_features: int, vec_dim: int, log2k: Sequence[int],
                  idx_words: Sequence, codebooks: Sequence, scale=None, bias=None,
                  device="cuda", out_bias=None) -> "Layer":
        """From numpy arrays: uint32 streams, fp16-bit (uint16) codebooks, scale,
        bias and output bias."""
        import numpy as np

        def words(a):
            a = np.ascontiguousarray(a, np.uint32).view(np.int32)
            return torch.from_numpy(a).to(device)

        def halves(a):
            if a is None:
                return None
            a = np.ascontiguousarray(a, np.uint16).view(np.int16)
            return torch.from_numpy(a).to(device).view(torch.float16)

        return cls(out_features, in_features, vec_dim, list(log2k),
                   [words(w) for w in idx_words], [halves(c) for c in codebooks],
                   halves(scale), halves(bias), out_bias=halves(out_bias))

    @classmethod
    def from_synth(cls, data, device="cuda", layout: str = "rows") -> "Layer":
        """From generated host data (row-order streams); layout="tile4" converts
        them on the device with vq_repack_tile4."""
        s = data.spec
        layer = cls.from_host(s.out_features, s.in_features, s.d, s.log2k, data.idx_words,
                              data.codebooks, data.scale, data.bias, device,
                              getattr(data, "out_bias", None))
        if layout == "tile4":
            layer = repack_tile4(layer)
        elif layout != "rows":
            raise ValueError(f"unknown index layout {layout!r}")
        return layer

    def nbytes(self) -> int:
        n = sum(t.numel() * t.element_size() for t in self.idx + self.codebooks)
        for t in (self.scale, self.bias, self.out_bias):
            n += 0 if t is None else t.numel() * 2
        return n


def tile4_words(out_features: int, log2k: int) -> int:
    """Smallest tile stride (32-bit words) of the tiled order: N records of 4 fields."""
    return -(-(out_features * 4 * log2k) // 128) * 4


def repack_tile4(layer: Layer, tile_words: Optional[Sequence[int]] = None) -> Layer:
    """The same layer with its index streams in the tiled order (vq_repack_tile4);
    codebooks, scale and bias are shared with ``layer``."""
    if layer.layout != "rows":
        raise ValueError("repack_tile4 needs a row-order layer")
    nvec = -(-layer.in_features // layer.vec_dim)
    ntile = -(-nvec // 4)
    tw = [tile4_words(layer.out_features, b) if tile_words is None else int(tile_words[m])
          for m, b in enumerate(layer.log2k)]
    dst = [torch.empty((ntile, w), dtype=torch.int32, device=layer.device) for w in tw]
    ptrs = (C.c_void_p * 2)(*([t.data_ptr() for t in dst] + [0] * (2 - len(dst))))
    words = (C.c_int64 * 2)(*(tw + [0] * (2 - len(tw))))
    _check("vq_repack_tile4", lib().vq_repack_tile4(C.byref(layer.desc()), ptrs, words,
                                                    C.c_void_p(_stream(layer.device))))
    return Layer(layer.out_features, layer.in_features, layer.vec_dim, list(layer.log2k), dst,
                 layer.codebooks, layer.scale, layer.bias, layout="tile4", out_bias=layer.out_bias)


def dequant(layer: Layer, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """W_hat, float16 [N][Kin] (or into ``out``, whose row stride is honoured)."""
    if out is None:
        out = torch.empty((layer.out_features, layer.in_features), dtype=torch.float16,
                          device=layer.device)
    ldw = out.stride(0) if out.dim() == 2 and out.shape[0] > 0 else layer.in_features
    _check("vq_dequant", lib().vq_dequant(C.byref(layer.desc()), _ptr(out), ldw,
                                          C.c_void_p(_stream(layer.device))))
    return out


def gemv_workspace_size(layer: Layer, batch: int) -> int:
    n = C.c_size_t(0)
    _check("vq_gemv_workspace_size", lib().vq_gemv_workspace_size(C.byref(layer.desc()), batch,
                                                                  C.byref(n)))
    return n.value


def gemm_workspace_size(layer: Layer, m: int, x_dtype=torch.bfloat16) -> int:
    n = C.c_size_t(0)
    _check("vq_gemm_workspace_size", lib().vq_gemm_workspace_size(
        C.byref(layer.desc()), m, _DTYPE[x_dtype], C.byref(n)))
    return n.value


def _workspace(nbytes: int, device, given: Optional[torch.Tensor]):
    if nbytes == 0:
        return None, 0
    if given is not None:
        return given, given.numel() * given.element_size()
    t = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return t, nbytes


def gemv(layer: Layer, x: torch.Tensor, out_dtype=torch.bfloat16,
         out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """y [B][N] = x [B][Kin] . W_hat^T for B <= 16 (x bf16 or fp16 on the device)."""
    if x.dim() == 1:
        x = x.unsqueeze(0)
    batch = x.shape[0]
    if out is None:
        out = torch.empty((batch, layer.out_features), dtype=out_dtype, device=layer.device)
    ws, ws_bytes = _workspace(gemv_workspace_size(layer, batch), layer.device, workspace)
    ldx = x.stride(0) if batch > 1 else max(x.shape[1], layer.in_features)
    ldy = out.stride(0) if batch > 1 else max(out.shape[1], layer.out_features)
    _check("vq_gemv", lib().vq_gemv(C.byref(layer.desc()), _ptr(x), _DTYPE[x.dtype], batch, ldx,
                                    _ptr(out), _DTYPE[out.dtype], ldy, _ptr(ws), ws_bytes,
                                    C.c_void_p(_stream(layer.device))))
    return out


NOALLOC_SCRATCH_BYTES = 8 << 20


def gemv_noalloc(layer: Layer, x: torch.Tensor, out_dtype=torch.bfloat16,
                 out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """vq_gemv without a workspace, for callers that cannot allocate device
    memory where they run the layer: the split-K scratch is a fixed
    NOALLOC_SCRATCH_BYTES array inside the library (see vq_gemv_noalloc in
    include/vq.h).  Pass ``out`` to keep the call free of allocations."""
    if x.dim() == 1:
        x = x.unsqueeze(0)
    batch = x.shape[0]
    if out is None:
        out = torch.empty((batch, layer.out_features), dtype=out_dtype, device=layer.device)
    ldx = x.stride(0) if batch > 1 else max(x.shape[1], layer.in_features)
    ldy = out.stride(0) if batch > 1 else max(out.shape[1], layer.out_features)
    _check("vq_gemv_noalloc", lib().vq_gemv_noalloc(
        C.byref(layer.desc()), _ptr(x), _DTYPE[x.dtype], batch, ldx, _ptr(out),
        _DTYPE[out.dtype], ldy, C.c_void_p(_stream(layer.device))))
    return out


def gemm(layer: Layer, x: torch.Tensor, out_dtype=torch.bfloat16,
         out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """y [M][N] = x [M][Kin] . W_hat^T on the tensor cores (x bf16 or fp16)."""
    m = x.shape[0]
    if out is None:
        out = torch.empty((m, layer.out_features), dtype=out_dtype, device=layer.device)
    ws, ws_bytes = _workspace(gemm_workspace_size(layer, m, x.dtype), layer.device, workspace)
    ldx = x.stride(0) if m > 1 else max(x.shape[1], layer.in_features)
    ldy = out.stride(0) if m > 1 else max(out.shape[1], layer.out_features)
    _check("vq_gemm", lib().vq_gemm(C.byref(layer.desc()), _ptr(x), _DTYPE[x.dtype], m, ldx,
                                    _ptr(out), _DTYPE[out.dtype], ldy, _ptr(ws), ws_bytes,
                                    C.c_void_p(_stream(layer.device))))
    return out


def _desc_array(layers: Sequence[Layer]):
    arr = (C.c_void_p * len(layers))(*[C.addressof(l.desc()) for l in layers])
    return arr


def gemv_multi_workspace_size(layers: Sequence[Layer], batch: int) -> int:
    n = C.c_size_t(0)
    _check("vq_gemv_multi_workspace_size",
           lib().vq_gemv_multi_workspace_size(_desc_array(layers), len(layers), batch, C.byref(n)))
    return n.value


def gemv_multi(layers: Sequence[Layer], x: torch.Tensor, out_dtype=torch.bfloat16,
               outs: Optional[Sequence[torch.Tensor]] = None,
               workspace: Optional[torch.Tensor] = None) -> List[torch.Tensor]:
    """y_l [B][N_l] = x [B][Kin] . W_hat_l^T for layers sharing x (vq_gemv_multi);
    tiled 2^16-book layers at batch 1 run as one table launch."""
    if x.dim() == 1:
        x = x.unsqueeze(0)
    batch = x.shape[0]
    dev = layers[0].device
    if outs is None:
        outs = [torch.empty((batch, l.out_features), dtype=out_dtype, device=dev) for l in layers]
    ws, ws_bytes = _workspace(gemv_multi_workspace_size(layers, batch), dev, workspace)
    ldx = x.stride(0) if batch > 1 else max(x.shape[1], layers[0].in_features)
    ys = (C.c_void_p * len(layers))(*[o.data_ptr() for o in outs])
    ldy = (C.c_int64 * len(layers))(*[o.stride(0) if batch > 1 else max(o.shape[1], l.out_features)
                                      for o, l in zip(outs, layers)])
    _check("vq_gemv_multi", lib().vq_gemv_multi(_desc_array(layers), len(layers), _ptr(x), _DTYPE[x.dtype],
                                                batch, ldx, ys, _DTYPE[outs[0].dtype], ldy, _ptr(ws),
                                                ws_bytes, C.c_void_p(_stream(dev))))
    return list(outs)


def rht(x: torch.Tensor, signs: torch.Tensor, inverse: bool = False, out_dtype=None,
        out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Randomized Hadamard transform of the rows of x (vq_rht); `signs` holds
    the sign bits as int32 words (bit t set -> -1)."""
    if x.dim() == 1:
        x = x.unsqueeze(0)
    rows, n = x.shape
    if out is None:
        out = torch.empty((rows, n), dtype=out_dtype or x.dtype, device=x.device)
    ld_in = x.stride(0) if rows > 1 else max(n, 1)
    ld_out = out.stride(0) if rows > 1 else max(n, 1)
    _check("vq_rht", lib().vq_rht(_ptr(x), _DTYPE[x.dtype], rows, n, ld_in, _ptr(signs), int(inverse),
                                  _ptr(out), _DTYPE[out.dtype], ld_out, C.c_void_p(_stream(x.device))))
    return out


def gemv_rht_workspace_size(layer: Layer, batch: int) -> int:
    n = C.c_size_t(0)
    _check("vq_gemv_rht_workspace_size",
           lib().vq_gemv_rht_workspace_size(C.byref(layer.desc()), batch, C.byref(n)))
    return n.value


def gemv_rht(layer: Layer, signs_in: torch.Tensor, signs_out: torch.Tensor, x: torch.Tensor,
             out_dtype=torch.bfloat16, out: Optional[torch.Tensor] = None,
             workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """y = U^T (W~ (V x)) for a layer whose streams encode the rotated W~ (vq_gemv_rht)."""
    if x.dim() == 1:
        x = x.unsqueeze(0)
    batch = x.shape[0]
    if out is None:
        out = torch.empty((batch, layer.out_features), dtype=out_dtype, device=layer.device)
    ws, ws_bytes = _workspace(gemv_rht_workspace_size(layer, batch), layer.device, workspace)
    ldx = x.stride(0) if batch > 1 else max(x.shape[1], layer.in_features)
    ldy = out.stride(0) if batch > 1 else max(out.shape[1], layer.out_features)
    _check("vq_gemv_rht", lib().vq_gemv_rht(C.byref(layer.desc()), _ptr(signs_in), _ptr(signs_out), _ptr(x),
                                            _DTYPE[x.dtype], batch, ldx, _ptr(out), _DTYPE[out.dtype], ldy,
                                            _ptr(ws), ws_bytes, C.c_void_p(_stream(layer.device))))
    return out


def hessian_workspace_size(n_tokens: int, d: int) -> int:
    nb = C.c_size_t(0)
    _check("vq_hessian_workspace_size", lib().vq_hessian_workspace_size(n_tokens, d, C.byref(nb)))
    return nb.value


def hessian(x: torch.Tensor, out: Optional[torch.Tensor] = None,
            workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """h = 2 X^T X / n + 0.01 mean(diag) I (float32 [d][d]) of activations x
    (bf16 or fp16 [n_tokens][d] on the device), through vq_hessian."""
    n, d = x.shape
    if out is None:
        out = torch.empty((d, d), dtype=torch.float32, device=x.device)
    ws, ws_bytes = _workspace(hessian_workspace_size(n, d), x.device, workspace)
    ldx = x.stride(0) if n > 1 else max(d, 1)
    _check("vq_hessian", lib().vq_hessian(_ptr(x), _DTYPE[x.dtype], n, d, ldx, _ptr(out), out.stride(0),
                                          _ptr(ws), ws_bytes, C.c_void_p(_stream(x.device))))
    return out


def row_words(in_features: int, vec_dim: int, log2k: int) -> int:
    """Smallest row stride (32-bit words) of a row-order stream."""
    nvec = -(-in_features // vec_dim)
    return -(-(nvec * log2k) // 128) * 4


def _encode_desc(w: torch.Tensor, codebooks, log2k, vec_dim: int, idx,
                 hessian: Optional[torch.Tensor] = None) -> _EncDesc:
    d = _EncDesc()
    d.out_features, d.in_features = w.shape[0], w.shape[1]
    d.vec_dim, d.n_books = vec_dim, len(log2k)
    d.w = w.data_ptr() if w.numel() else None
    d.ldw = w.stride(0) if w.shape[0] > 1 else max(w.shape[1], 1)   # ldw >= Kin
    for m, b in enumerate(log2k):
        d.log2k[m] = b
        d.codebook[m] = codebooks[m].data_ptr()
        d.idx[m] = idx[m].data_ptr() if idx[m].numel() else None
        d.idx_row_words[m] = idx[m].shape[1]
    if hessian is not None:
        if hessian.dtype != torch.float32 or hessian.dim() != 2 or hessian.stride(1) != 1:
            raise ValueError("the Hessian must be a row-major float32 matrix")
        d.h = hessian.data_ptr()
        d.ldh = hessian.stride(0)
    return d


def encode_workspace_size(out_features: int, in_features: int, log2k: Sequence[int],
                          vec_dim: int, hessian: bool = False) -> int:
    d = _EncDesc()
    d.out_features, d.in_features, d.vec_dim, d.n_books = out_features, in_features, vec_dim, len(log2k)
    d.ldw = max(in_features, 1)
    if hessian:                        # any aligned non-null pointer: only sizes are read
        d.h = 256
        d.ldh = max(in_features, 1)
    for m, b in enumerate(log2k):
        d.log2k[m] = int(b)
        d.idx_row_words[m] = row_words(in_features, vec_dim, int(b))
    n = C.c_size_t(0)
    _check("vq_encode_workspace_size", lib().vq_encode_workspace_size(C.byref(d), C.byref(n)))
    return n.value


def encode(w: torch.Tensor, codebooks: Sequence[torch.Tensor], log2k: Sequence[int], vec_dim: int,
           workspace: Optional[torch.Tensor] = None, hessian: Optional[torch.Tensor] = None) -> Layer:
    """Nearest-centroid encoding of W (float16 [N][Kin] on the device) against
    one book, or two as a greedy residual cascade (vq_encode): a row-order
    Layer holding the packed streams and the given codebooks (no scale or
    bias).  With ``hessian`` (float32 [Kin][Kin] on the device, e.g. from
    ``hessian()``) the distance is the Hessian-weighted (v-c)^T H_v (v-c)."""
    if w.dtype != torch.float16 or w.dim() != 2 or (w.shape[0] > 1 and w.stride(1) != 1):
        raise ValueError("w must be a row-major float16 matrix")
    log2k = [int(b) for b in log2k]
    books = [c.contiguous() for c in codebooks[:len(log2k)]]
    idx = [torch.empty((w.shape[0], row_words(w.shape[1], vec_dim, b)), dtype=torch.int32,
                       device=w.device) for b in log2k]
    d = _encode_desc(w, books, log2k, vec_dim, idx, hessian)
    n = C.c_size_t(0)
    _check("vq_encode_workspace_size", lib().vq_encode_workspace_size(C.byref(d), C.byref(n)))
    ws, ws_bytes = _workspace(n.value, w.device, workspace)
    _check("vq_encode", lib().vq_encode(C.byref(d), _ptr(ws), ws_bytes, C.c_void_p(_stream(w.device))))
    return Layer(w.shape[0], w.shape[1], vec_dim, log2k, idx, books)


def kernel_launches() -> int:
    """Kernels this library has launched in this process (host counter)."""
    return int(lib().vq_kernel_launches())


def abi_version() -> int:
    return lib().vq_abi_version()


def status_string(status: int) -> str:
    return lib().vq_status_string(status).decode()

"""Seeded synthetic inputs for the bit-packed VQ/RVQ linear layer.

This module is the only code that both the CPU oracle (``oracle/``) and the
CUDA library (``bit_packed_index_b200``) consume.  It draws random numbers and
lays them out in the storage format; it holds none of the method's arithmetic
(no unpacking, no centroid sums, no scale/bias, no products).

Storage format produced here (the library's index format):

* one packed index stream per codebook, one stream row per output row;
* a row holds ``nvec = ceil(in_features / d)`` fields of ``b = log2 K`` bits,
  field ``j`` occupying bits ``[j*b, j*b + b)`` of the row, numbered
  LSB-first inside little-endian 32-bit words;
* each row starts on a 16-byte boundary: ``row_words`` is a multiple of 4 and
  at least ``ceil(nvec*b / 128) * 4``; bits past ``nvec*b`` are zero here
  (readers must ignore them);
* codebooks are fp16 ``[K][d]`` row-major; scale and bias are fp16 ``[N]``;
  activations are bf16 ``[B][in_features]``.

Uniformly random index words give uniformly distributed indices, so the
streams are drawn as random words directly, with the pad bits cleared.

Value recipes follow the workloads the pages discuss ("VPTQ Guide: Extreme
2-Bit Vector Quantization", sections "Step 2: Multi-Stage Residual Vector
Quantizer" and "Step 4: Verification and Parity Test Harness": randn * 0.02
weights, fp16 codebooks; "Vector Quantization for LLM Weights in Production",
section "Why Scalar Quantization Breaks Below 4 Bits": under 0.1 % outlier
channels).  Draw order inside one layer: codebook 1, codebook 2, index stream
1, index stream 2, scale, bias.  Activations come from their own seed.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "LayerSpec", "LayerData", "make_layer", "make_x", "row_words_for",
    "nvec_for", "WORKLOADS", "Workload", "to_bf16_bits", "to_f16_bits",
]


def nvec_for(in_features: int, d: int) -> int:
    """Number of d-vectors covering one row (the last one may be partial)."""
    return -(-in_features // d)


def row_words_for(nvec: int, b: int) -> int:
    """Minimal 16-byte-padded stream row length, in 32-bit words."""
    return -(-(nvec * b) // 128) * 4


def to_f16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 values -> fp16 bit patterns (numpy's round-to-nearest-even)."""
    return np.ascontiguousarray(np.asarray(a, np.float32).astype(np.float16)).view(np.uint16)


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 values -> bf16 bit patterns (torch's round-to-nearest-even)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


@dataclasses.dataclass(frozen=True)
class LayerSpec:
    out_features: int
    in_features: int
    d: int
    log2k: Tuple[int, ...]                 # one entry per codebook (1 or 2)
    book_std: Tuple[float, ...]            # N(0, std) per codebook
    scale_range: Optional[Tuple[float, float]] = (0.5, 1.5)   # None: no scale
    bias_std: Optional[float] = 1e-3                          # None: no bias
    name: str = ""
    out_bias_std: Optional[float] = None                      # None: no output bias

    @property
    def n_books(self) -> int:
        return len(self.log2k)

    @property
    def nvec(self) -> int:
        return nvec_for(self.in_features, self.d)


@dataclasses.dataclass
class LayerData:
    spec: LayerSpec
    idx_words: List[np.ndarray]       # uint32 [N][row_words[m]] per book
    row_words: List[int]
    codebooks: List[np.ndarray]       # uint16 (fp16 bits) [K_m][d] per book
    scale: Optional[np.ndarray]       # uint16 (fp16 bits) [N] or None
    bias: Optional[np.ndarray]        # uint16 (fp16 bits) [N] or None
    out_bias: Optional[np.ndarray] = None   # uint16 (fp16 bits) [N] or None

    def nbytes(self) -> int:
        n = sum(w.nbytes for w in self.idx_words) + sum(c.nbytes for c in self.codebooks)
        for a in (self.scale, self.bias, self.out_bias):
            n += 0 if a is None else a.nbytes
        return n


def _unique_rows(book: np.ndarray) -> bool:
    v = np.ascontiguousarray(book).view(np.dtype((np.void, book.dtype.itemsize * book.shape[1])))
    return np.unique(v).shape[0] == book.shape[0]


def _draw_book(rng: np.random.Generator, k: int, d: int, std: float) -> np.ndarray:
    for _ in range(16):
        book = to_f16_bits(rng.standard_normal((k, d), dtype=np.float32) * np.float32(std))
        if _unique_rows(book):
            return book.reshape(k, d)
    raise RuntimeError("could not draw a codebook with unique rows")


def _draw_stream(rng: np.random.Generator, n: int, nvec: int, b: int, row_words: int,
                 pad_garbage: bool = False) -> np.ndarray:
    words = rng.integers(0, 1 << 32, size=(n, row_words), dtype=np.uint64).astype(np.uint32)
    if not pad_garbage:
        used = nvec * b
        full, rem = divmod(used, 32)
        if rem:
            words[:, full] &= np.uint32((1 << rem) - 1)
            full += 1
        words[:, full:] = 0
    return words


def make_layer(spec: LayerSpec, seed: int, row_words: Optional[Sequence[int]] = None,
               pad_garbage: bool = False) -> LayerData:
    """Draw one synthetic layer.  ``row_words`` may over-pad the stream rows
    (each must be a multiple of 4 and at least the minimum);
    ``pad_garbage`` fills the pad bits with random bits instead of zeros."""
    rng = np.random.Generator(np.random.PCG64(seed))
    n, d, nvec = spec.out_features, spec.d, spec.nvec
    books = [_draw_book(rng, 1 << b, d, std) for b, std in zip(spec.log2k, spec.book_std)]
    rws = []
    streams = []
    for m, b in enumerate(spec.log2k):
        rw = row_words_for(nvec, b) if row_words is None else int(row_words[m])
        if rw % 4 or rw < row_words_for(nvec, b):
            raise ValueError("row_words must be a multiple of 4 and cover the row")
        rws.append(rw)
        streams.append(_draw_stream(rng, n, nvec, b, rw, pad_garbage))
    scale = None
    if spec.scale_range is not None:
        lo, hi = spec.scale_range
        scale = to_f16_bits(rng.uniform(lo, hi, size=n).astype(np.float32))
    bias = None
    if spec.bias_std is not None:
        bias = to_f16_bits(rng.standard_normal(n, dtype=np.float32) * np.float32(spec.bias_std))
    out_bias = None
    if spec.out_bias_std is not None:     # drawn last: the other arrays do not depend on it
        out_bias = to_f16_bits(rng.standard_normal(n, dtype=np.float32)
                               * np.float32(spec.out_bias_std))
    return LayerData(spec, streams, rws, books, scale, bias, out_bias)


def make_x(seed: int, rows: int, in_features: int, outlier_frac: float = 0.0,
           outlier_scale: float = 20.0, ld: Optional[int] = None, as_fp16: bool = False) -> np.ndarray:
    """Activations ~N(0, 1) as bf16 bits [rows][ld] (fp16 bits if ``as_fp16``);
    ``round(outlier_frac * in_features)`` distinct columns are scaled by
    ``outlier_scale`` (outlier channels).  Columns past ``in_features`` are 0."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = rng.standard_normal((rows, in_features), dtype=np.float32)
    n_out = int(round(outlier_frac * in_features))
    if n_out:
        cols = rng.choice(in_features, size=n_out, replace=False)
        x[:, cols] *= np.float32(outlier_scale)
    ld = in_features if ld is None else ld
    full = np.zeros((rows, ld), np.float32)
    full[:, :in_features] = x
    return to_f16_bits(full) if as_fp16 else to_bf16_bits(full)


# --------------------------------------------------------------------------
# Named workloads: the layer shapes and distributions of the models the pages
# size (Llama-3 8B, Llama-3 70B, Llama-3.1 405B; "VPTQ Guide", table
# "Configuration Sizing Matrix across Model Architectures").
# --------------------------------------------------------------------------

def make_encode_input(out_features: int, in_features: int, d: int, log2k: Sequence[int],
                      book_std: Sequence[float], seed: int, w_std: float = 0.02):
    """Inputs of the nearest-centroid encoder: fp16 bits of a weight matrix
    W [N][Kin] ~ N(0, w_std) and of one codebook [K_m][d] ~ N(0, std_m) per
    entry of log2k (unique rows).  Draw order: books, then W."""
    rng = np.random.default_rng(seed)
    books = [_draw_book(rng, 1 << b, d, s) for b, s in zip(log2k, book_std)]
    w = to_f16_bits(rng.standard_normal((out_features, in_features), dtype=np.float32)
                    * np.float32(w_std)).reshape(out_features, in_features)
    return w, books


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    layers: Tuple[Tuple[LayerSpec, int], ...]     # (spec, seed)
    batches: Tuple[int, ...]                      # decode B values or prefill M values
    outlier_frac: float = 0.0
    x_seed: int = 1000
    kind: str = "decode"                          # "decode" or "prefill"


def _spec(n, k, d, log2k, std, name):
    return LayerSpec(n, k, d, tuple(log2k), tuple(std), (0.5, 1.5), 1e-3, name)


WORKLOADS = {
    "tiny_512": Workload(
        "tiny_512: W 512x512, d=8, one K=2^16 book (2.0 bpw), B=1",
        ((_spec(512, 512, 8, [16], [0.02], "tiny"), 0),), (1,), 0.0, 1000),
    "llama3_8b_up": Workload(
        "llama3_8b_up: W 14336x4096, d=8, K=2^12 + residual K=2^8 (2.5 bpw), B in {1,4,16}",
        ((_spec(14336, 4096, 8, [12, 8], [0.02, 0.005], "up_proj"), 2),), (1, 4, 16), 0.0, 1002),
    "llama3_70b_mlp": Workload(
        "llama3_70b_mlp: gate/up 28672x8192 + down 8192x28672, d=8, one K=2^16 book (2.0 bpw), "
        "0.1% outlier columns x20, B in {1,2,8,16}",
        ((_spec(28672, 8192, 8, [16], [0.02], "gate_proj"), 3),
         (_spec(28672, 8192, 8, [16], [0.02], "up_proj"), 103),
         (_spec(8192, 28672, 8, [16], [0.02], "down_proj"), 203)),
        (1, 2, 8, 16), 0.001, 1003),
    "prefill_8192": Workload(
        "prefill_8192: x [M,8192], W 8192x8192, d=8, K=2^16 + residual K=2^8 (3.0 bpw), M in {512,2048,4096}",
        ((_spec(8192, 8192, 8, [16, 8], [0.02, 0.005], "proj"), 4),), (512, 2048, 4096), 0.0, 1004,
        "prefill"),
    "llama31_405b": Workload(
        "llama31_405b: q/o 16384^2, k/v 1024x16384, gate/up 53248x16384, down 16384x53248, d=6, "
        "K=2^12 + residual K=2^4 (2.67 bpw), decode B in 1..16, prefill M=1024",
        ((_spec(16384, 16384, 6, [12, 4], [0.02, 0.005], "q_proj"), 5),
         (_spec(1024, 16384, 6, [12, 4], [0.02, 0.005], "k_proj"), 105),
         (_spec(1024, 16384, 6, [12, 4], [0.02, 0.005], "v_proj"), 205),
         (_spec(16384, 16384, 6, [12, 4], [0.02, 0.005], "o_proj"), 305),
         (_spec(53248, 16384, 6, [12, 4], [0.02, 0.005], "gate_proj"), 405),
         (_spec(53248, 16384, 6, [12, 4], [0.02, 0.005], "up_proj"), 505),
         (_spec(16384, 53248, 6, [12, 4], [0.02, 0.005], "down_proj"), 605)),
        tuple(range(1, 17)), 0.0, 1005),
}



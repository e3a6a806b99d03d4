"""Bit-rate and footprint arithmetic for a bit-packed VQ/RVQ layer (host only).

* Index bits per weight: b = sum_m log2(K_m) / d ("VPTQ Guide: Extreme 2-Bit
  Vector Quantization", section "The Information-Theoretic Superiority of
  Vector Quantization"; "Vector Quantization for LLM Weights in Production",
  section "Theoretical Foundations: Scalar vs. Vector Quantization").
* Effective bits per weight with the codebook overhead,
  b_eff = sum_m log2(K_m) / d + (sum_m K_m) * d * 16 / (N * Kin)
  ("VPTQ Guide", section "3. Effective Bit-Width Calculation").
* Stored bytes of the packed format: each stream row is padded to 16 bytes.
"""
from __future__ import annotations

from typing import Optional, Sequence


def index_bits_per_weight(d: int, log2k: Sequence[int]) -> float:
    if d < 1 or not log2k:
        raise ValueError("need d >= 1 and at least one codebook")
    return sum(int(b) for b in log2k) / d


def codebook_bytes(d: int, log2k: Sequence[int]) -> int:
    """fp16 centroids: sum_m K_m * d * 2 bytes."""
    return sum((1 << int(b)) * d * 2 for b in log2k)


def effective_bits_per_weight(out_features: int, in_features: int, d: int,
                              log2k: Sequence[int]) -> float:
    total = out_features * in_features
    if total <= 0:
        raise ValueError("empty layer")
    return index_bits_per_weight(d, log2k) + codebook_bytes(d, log2k) * 8 / total


def stream_row_words(in_features: int, d: int, b: int) -> int:
    nvec = -(-in_features // d)
    return -(-(nvec * b) // 128) * 4


def packed_index_bytes(out_features: int, in_features: int, d: int, log2k: Sequence[int],
                       row_words: Optional[Sequence[int]] = None) -> int:
    """Bytes of the stored index streams (16-byte padded rows)."""
    rws = row_words or [stream_row_words(in_features, d, b) for b in log2k]
    return sum(out_features * rw * 4 for rw in rws)


def footprint_bytes(out_features: int, in_features: int, d: int, log2k: Sequence[int],
                    with_scale: bool = False, with_bias: bool = False) -> int:
    """Stored bytes: packed indices + fp16 codebooks (+ fp16 scale / bias)."""
    n = packed_index_bytes(out_features, in_features, d, log2k) + codebook_bytes(d, log2k)
    return n + 2 * out_features * (int(with_scale) + int(with_bias))

"""Closed forms the pages print for the bit rate and footprint.

* 16-bit index per 8 weights = 2.0 bpw ("VPTQ Guide: Extreme 2-Bit Vector
  Quantization", section "The Information-Theoretic Superiority of Vector
  Quantization"; "Vector Quantization for LLM Weights in Production",
  section "Theoretical Foundations").
* (16 + 8) / 8 = 3.0, 16 / 8 = 2.0 (v8-k65536-woft), (8 + 8) / 8 = 2.0
  (v8-k256-r1-k256), v = 16 with K = 2^16 gives 1.0 ("VPTQ Guide", section
  "3. Effective Bit-Width Calculation").
* R = 2, K = 256, g = 8 gives 2 bpw ("Sub-4-Bit Quantization: AQLM, QuIP#, &
  HQQ", section "AQLM: Additive Quantization").
* Two K = 256, v = 8 fp16 books take 8 KB, and the verification script's 4096 x
  4096 layer stores one byte per vector per book ("VPTQ Guide", section
  "Step 4: Verification and Parity Test Harness"); from its formulas the
  footprint is 2*2,097,152 + 2*4,096 = 4,202,496 bytes, 2.0039 bpw, 7.98x
  smaller than fp16.
"""
import pytest

from bit_packed_index_b200 import bitrate


def test_index_bitrates_from_the_pages():
    assert bitrate.index_bits_per_weight(8, [16]) == 2.0
    assert bitrate.index_bits_per_weight(8, [16, 8]) == 3.0
    assert bitrate.index_bits_per_weight(8, [8, 8]) == 2.0
    assert bitrate.index_bits_per_weight(16, [16]) == 1.0
    assert bitrate.index_bits_per_weight(8, [12, 8]) == 2.5
    assert bitrate.index_bits_per_weight(6, [12, 4]) == pytest.approx(8 / 3)


def test_verification_script_footprint():
    books = bitrate.codebook_bytes(8, [8, 8])
    assert books == 8192                                   # "8 KB"
    idx = bitrate.packed_index_bytes(4096, 4096, 8, [8, 8])
    assert idx == 2 * 2_097_152                            # one byte per vector per book
    total = idx + books
    assert total == 4_202_496
    assert total * 8 / 4096 ** 2 == pytest.approx(2.0039, abs=1e-4)
    assert 4096 ** 2 * 2 / total == pytest.approx(7.98, abs=5e-3)
    assert bitrate.footprint_bytes(4096, 4096, 8, [8, 8]) == total
    assert bitrate.effective_bits_per_weight(4096, 4096, 8, [8, 8]) == pytest.approx(
        total * 8 / 4096 ** 2)


def test_effective_bitrate_formula():
    # b_eff = (log2 K1 + log2 K2) / v + (K1 + K2) * v * 16 / total
    n = k = 8192
    got = bitrate.effective_bits_per_weight(n, k, 8, [16, 8])
    assert got == pytest.approx(3.0 + (65536 + 256) * 8 * 16 / (n * k))


def test_padded_rows():
    # d = 6, Kin = 16384: 2731 vectors of 12 bits = 32772 bits -> 257 x 128 bits
    assert bitrate.stream_row_words(16384, 6, 12) == 257 * 4
    with pytest.raises(ValueError):
        bitrate.index_bits_per_weight(0, [8])

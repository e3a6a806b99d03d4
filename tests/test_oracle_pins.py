"""Pins for the CPU oracle: each test checks it against something other than
itself -- library conversions, a hand-derived fixture, closed forms,
identities with a known answer, an independent numpy restatement, and brute
force on tiny inputs.  A plausible slip in the oracle (a wrong bit order, a
dropped residual term, a swapped scale/bias order, a transposed product, a
tie broken the wrong way) fails at least one of them."""
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from synth import LayerData, LayerSpec

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# -- fp16 / bf16 conversions against numpy and torch --------------------------

def test_f16_to_f32_all_patterns():
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = h.view(np.float16).astype(np.float32)
    got = oracle.f16_to_f32(h)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_f32_to_f16_matches_numpy():
    rng = np.random.default_rng(7)
    parts = [
        rng.standard_normal(400_000).astype(np.float32) * 0.02,
        rng.standard_normal(200_000).astype(np.float32) * 3e4,
        (rng.standard_normal(200_000) * 1e-5).astype(np.float32),      # subnormal range
        (rng.standard_normal(100_000) * 1e-8).astype(np.float32),      # underflow
        rng.uniform(65400, 65600, 50_000).astype(np.float32),           # overflow edge
        np.array([0.0, -0.0, np.inf, -np.inf, 65504, 65519.99, 65520, 65536,
                  2 ** -24, 2 ** -25, 3 * 2 ** -26, 2 ** -14, 2 ** -14 - 2 ** -25],
                 np.float32),
    ]
    # exact midpoints between neighbouring fp16 values (ties to even)
    h = np.arange(0x0001, 0x7bff, dtype=np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).view(np.float16).astype(np.float64)
    mid = ((lo + hi) / 2).astype(np.float32)
    parts += [mid, -mid]
    a = np.concatenate(parts)
    with np.errstate(over="ignore"):
        ref = a.astype(np.float16).view(np.uint16)
    got = oracle.f32_to_f16(a)
    assert np.array_equal(got, ref), np.flatnonzero(got != ref)[:10]


def test_bf16_conversions_match_torch():
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = (h.astype(np.uint32) << 16).view(np.float32)
    got = oracle.bf16_to_f32(h)
    nan = np.isnan(ref)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))
    rng = np.random.default_rng(8)
    a = np.concatenate([
        rng.standard_normal(300_000).astype(np.float32),
        (rng.standard_normal(100_000) * 1e-39).astype(np.float32),     # fp32 subnormals
        np.array([0.0, -0.0, np.inf, -np.inf, 3.3895314e38, 3.4e38], np.float32),
    ])
    # exact ties between neighbouring bf16 values
    hb = np.arange(0x0001, 0x7f7f, 97, dtype=np.uint32)
    mid = ((hb << 16) + (1 << 15)).astype(np.uint32).view(np.float32)
    a = np.concatenate([a, mid, -mid])
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.f32_to_bf16(a)
    assert np.array_equal(got, ref)


# -- index streams ------------------------------------------------------------

def _numpy_unpack(words: np.ndarray, b: int, nvec: int) -> np.ndarray:
    """Independent restatement: expand words to bits (LSB first), regroup."""
    bits = np.unpackbits(words.view(np.uint8), axis=1, bitorder="little")
    f = bits[:, : nvec * b].reshape(words.shape[0], nvec, b).astype(np.uint32)
    return (f << np.arange(b, dtype=np.uint32)).sum(axis=2).astype(np.uint32)


def test_golden_layout():
    with open(os.path.join(GOLDEN, "index_stream_layout.txt")) as fh:
        rows = [ln for ln in fh if ln.strip() and not ln.startswith("#")]
    assert len(rows) == 3
    for ln in rows:
        b, fields, words = (p.split() for p in ln.split("|"))
        b = int(b[0])
        fields = np.array([[int(v) for v in fields]], np.uint32)
        words = np.array([[int(v, 16) for v in words]], np.uint32)
        assert np.array_equal(oracle.pack(fields, b), words)
        assert np.array_equal(oracle.unpack(words, b, fields.shape[1]), fields)


@pytest.mark.parametrize("b", range(1, 17))
def test_unpack_matches_numpy_and_roundtrips(b):
    rng = np.random.default_rng(100 + b)
    for nvec in (1, 7, 31, 32, 33, 129, 1000):
        rw = synth.row_words_for(nvec, b) + 4 * int(rng.integers(0, 3))
        words = rng.integers(0, 1 << 32, size=(5, rw), dtype=np.uint64).astype(np.uint32)
        idx = oracle.unpack(words, b, nvec)
        assert np.array_equal(idx, _numpy_unpack(words, b, nvec))
        assert idx.max() < (1 << b)
        again = oracle.unpack(oracle.pack(idx, b, rw), b, nvec)
        assert np.array_equal(again, idx)


def test_pack_rejects_wide_fields():
    with pytest.raises(ValueError):
        oracle.pack(np.array([[8]], np.uint32), 3)


def test_golden_tile4_layout():
    with open(os.path.join(GOLDEN, "index_stream_tile4.txt")) as fh:
        rows = [ln for ln in fh if ln.strip() and not ln.startswith("#")]
    assert len(rows) == 2
    for ln in rows:
        b, n, nvec, fields, tiles = ln.split("|")
        b, n, nvec = int(b), int(n), int(nvec)
        fields = np.array([int(v) for v in fields.split()], np.uint32).reshape(n, nvec)
        words = np.array([[int(v, 16) for v in t.split()] for t in tiles.split("/")], np.uint32)
        assert np.array_equal(oracle.pack_tile4(fields, b), words)
        assert np.array_equal(oracle.unpack_tile4(words, b, n, nvec), fields)


@pytest.mark.parametrize("b", [1, 3, 4, 7, 8, 12, 16])
def test_tile4_order_holds_the_same_fields(b):
    """Both storage orders carry the same indices: unpacking either gives the
    matrix that was packed, for ragged nvec and padded tiles."""
    rng = np.random.default_rng(300 + b)
    for n, nvec in ((1, 1), (5, 7), (33, 4), (17, 13)):
        idx = rng.integers(0, 1 << b, size=(n, nvec), dtype=np.uint64).astype(np.uint32)
        tw = oracle.tile4_words(n, b) + 4 * int(rng.integers(0, 2))
        tiles = oracle.pack_tile4(idx, b, tw)
        assert tiles.shape == (-(-nvec // 4), tw)
        assert np.array_equal(oracle.unpack_tile4(tiles, b, n, nvec), idx)
        assert np.array_equal(oracle.unpack(oracle.pack(idx, b), b, nvec), idx)
        # every bit past the last record of a tile, and every field of a
        # vector >= nvec, is zero
        bits = np.unpackbits(tiles.view(np.uint8), axis=1, bitorder="little")
        assert not bits[:, n * 4 * b:].any()
        if nvec % 4:
            rec = bits[-1, : n * 4 * b].reshape(n, 4, b)
            assert not rec[:, nvec % 4:, :].any()


def test_tile4_rejects_wide_fields_and_short_tiles():
    with pytest.raises(ValueError):
        oracle.pack_tile4(np.array([[8]], np.uint32), 3)
    with pytest.raises(ValueError):
        oracle.pack_tile4(np.zeros((40, 4), np.uint32), 16, tile_words=4)


# -- dequantisation -----------------------------------------------------------

ONE = np.float16(1.0).view(np.uint16)


def _layer(n, kin, d, books, streams_idx, scale=None, bias=None):
    """A LayerData from explicit books and index arrays (packed by the oracle)."""
    log2k = tuple(int(np.log2(bk.shape[0])) for bk in books)
    spec = LayerSpec(n, kin, d, log2k, tuple(0.0 for _ in books), None, None)
    words = [oracle.pack(ix, b) for ix, b in zip(streams_idx, log2k)]
    return LayerData(spec, words, [w.shape[1] for w in words], list(books), scale, bias)


def test_binary_codebook_identity():
    """d=8, K=256, C[k][e] = bit e of k: W_hat spells out every index's bits."""
    d, n, kin = 8, 37, 8 * 41
    k = np.arange(256, dtype=np.uint32)
    book = np.where((k[:, None] >> np.arange(8)) & 1, ONE, 0).astype(np.uint16)
    rng = np.random.default_rng(1)
    idx = rng.integers(0, 256, size=(n, kin // d), dtype=np.uint32)
    w = oracle.dequant(_layer(n, kin, d, [book], [idx]))
    bits = ((idx[:, :, None] >> np.arange(8)) & 1).reshape(n, kin)
    assert np.array_equal(w, np.where(bits, ONE, 0).astype(np.uint16))


def test_one_hot_identity_and_product():
    """d=8, K=8, C[k] = e_k: y[o] = sum_j x[8j + idx[o][j]]."""
    d, n, nvec = 8, 23, 50
    kin = d * nvec
    book = np.where(np.eye(8, dtype=bool), ONE, 0).astype(np.uint16)
    rng = np.random.default_rng(2)
    idx = rng.integers(0, 8, size=(n, nvec), dtype=np.uint32)
    layer = _layer(n, kin, d, [book], [idx])
    x = synth.make_x(11, 3, kin)
    y = oracle.linear(layer, x)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    cols = np.arange(nvec) * 8 + idx                      # [n][nvec]
    ref = np.stack([xf[:, cols[o]].sum(axis=1) for o in range(n)], axis=1)
    assert np.allclose(y, ref, rtol=1e-13, atol=1e-13)


def test_affine_special_case():
    """All-zero book: W_hat[o][:] = fp16(0 * s[o] + t[o]) = t[o]; y = t[o] * sum(x)."""
    d, n, kin = 6, 19, 6 * 9 + 4
    book = np.zeros((16, d), np.uint16)
    rng = np.random.default_rng(3)
    idx = rng.integers(0, 16, size=(n, -(-kin // d)), dtype=np.uint32)
    scale = synth.to_f16_bits(rng.uniform(0.5, 1.5, n).astype(np.float32))
    bias = synth.to_f16_bits(rng.standard_normal(n).astype(np.float32))
    layer = _layer(n, kin, d, [book], [idx], scale, bias)
    w = oracle.dequant(layer)
    assert np.array_equal(w, np.repeat(bias[:, None], kin, axis=1))
    x = synth.make_x(12, 2, kin)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    tf = bias.view(np.float16).astype(np.float64)
    assert np.allclose(oracle.linear(layer, x), xf.sum(1)[:, None] * tf[None, :], rtol=1e-12)


def test_output_bias_closed_form():
    """All-zero book with an output bias: y[m][o] = t[o] * sum_k x[m][k] + b_out[o]
    (the layer bias t folded into W_hat, then F.linear's output bias once)."""
    d, n, kin = 8, 21, 8 * 7 + 3
    book = np.zeros((16, d), np.uint16)
    rng = np.random.default_rng(31)
    idx = rng.integers(0, 16, size=(n, -(-kin // d)), dtype=np.uint32)
    bias = synth.to_f16_bits(rng.standard_normal(n).astype(np.float32))
    b_out = synth.to_f16_bits(rng.uniform(-4.0, 4.0, n).astype(np.float32))
    layer = _layer(n, kin, d, [book], [idx], None, bias)
    x = synth.make_x(32, 3, kin)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    tf = bias.view(np.float16).astype(np.float64)
    bf = b_out.view(np.float16).astype(np.float64)
    want = xf.sum(1)[:, None] * tf[None, :] + bf[None, :]
    assert np.allclose(oracle.linear(layer, x, out_bias=b_out), want, rtol=1e-12, atol=1e-12)
    # x = 0 leaves exactly the output bias, row by row (also through ``rows``)
    z = np.zeros_like(x)
    assert np.array_equal(oracle.linear(layer, z, out_bias=b_out), np.tile(bf, (3, 1)))
    rows = [20, 0, 7]
    assert np.array_equal(oracle.linear(layer, z, rows=rows, out_bias=b_out), np.tile(bf[rows], (3, 1)))


def test_output_bias_is_added_once_per_output_row():
    """Random two-book layer: linear with b_out equals numpy's x . W_hat^T (from
    the independent dequant restatement) + b_out, and the difference to the
    call without it is b_out in every row of x (not scaled, not per input)."""
    spec = LayerSpec(48, 8 * 40, 8, (12, 8), (0.02, 0.005), out_bias_std=0.5)
    layer = synth.make_layer(spec, seed=33)
    assert layer.out_bias is not None
    x = synth.make_x(34, 5, spec.in_features)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    w = _numpy_dequant(layer).view(np.float16).astype(np.float64)
    bf = layer.out_bias.view(np.float16).astype(np.float64)
    y = oracle.linear(layer, x)                      # the layer's own out_bias
    assert np.allclose(y, xf @ w.T + bf[None, :], rtol=1e-12, atol=1e-12)
    no_bias = oracle.linear(layer, x, out_bias=np.zeros(48, np.uint16))
    assert np.allclose(y - no_bias, np.tile(bf, (5, 1)), rtol=0, atol=1e-12)
    # the same seed without an output bias draws the same weights
    plain = synth.make_layer(LayerSpec(48, 8 * 40, 8, (12, 8), (0.02, 0.005)), seed=33)
    assert plain.out_bias is None
    assert all(np.array_equal(a, b) for a, b in zip(plain.idx_words, layer.idx_words))
    assert np.array_equal(oracle.linear(plain, x), no_bias)


def _numpy_dequant(layer) -> np.ndarray:
    """Independent float32 restatement, vectorised: same operation order."""
    s = layer.spec
    nvec = s.nvec
    acc = None
    for m in range(s.n_books):
        idx = _numpy_unpack(layer.idx_words[m], s.log2k[m], nvec)
        c = layer.codebooks[m].view(np.float16).astype(np.float32)[idx]   # [n][nvec][d]
        acc = c if acc is None else (acc + c).astype(np.float32)
    acc = acc.reshape(s.out_features, nvec * s.d)[:, : s.in_features]
    if layer.scale is not None:
        acc = (acc * layer.scale.view(np.float16).astype(np.float32)[:, None]).astype(np.float32)
    if layer.bias is not None:
        acc = (acc + layer.bias.view(np.float16).astype(np.float32)[:, None]).astype(np.float32)
    return acc.astype(np.float16).view(np.uint16)


@pytest.mark.parametrize("d,log2k,kin,scale,bias", [
    (8, (16,), 512, True, True),
    (8, (12, 8), 1024, True, True),
    (6, (12, 4), 6 * 50 + 4, True, True),
    (6, (12, 4), 6 * 50 + 1, False, True),
    (8, (8, 8), 8 * 33, True, False),
    (5, (7, 3), 5 * 20 + 3, False, False),
    (16, (16,), 16 * 8 + 15, True, True),
    (1, (4, 2), 77, True, True),
])
def test_dequant_matches_numpy_restatement(d, log2k, kin, scale, bias):
    spec = LayerSpec(61, kin, d, log2k, (0.02, 0.005)[: len(log2k)],
                     (0.5, 1.5) if scale else None, 1e-3 if bias else None)
    layer = synth.make_layer(spec, seed=d * 1000 + kin, pad_garbage=True)
    assert np.array_equal(oracle.dequant(layer), _numpy_dequant(layer))


def test_dequant_semantics_are_distinguishable():
    """The restatement pin separates the reading s*(c1+c2)+t from plausible
    slips: bias applied before the scale, or the residual book dropped."""
    spec = LayerSpec(64, 512, 8, (12, 8), (0.02, 0.005))
    layer = synth.make_layer(spec, seed=5)
    w = oracle.dequant(layer)
    s = spec
    i1 = _numpy_unpack(layer.idx_words[0], 12, s.nvec)
    i2 = _numpy_unpack(layer.idx_words[1], 8, s.nvec)
    c1 = layer.codebooks[0].view(np.float16).astype(np.float32)[i1].reshape(64, 512)
    c2 = layer.codebooks[1].view(np.float16).astype(np.float32)[i2].reshape(64, 512)
    sc = layer.scale.view(np.float16).astype(np.float32)[:, None]
    t = layer.bias.view(np.float16).astype(np.float32)[:, None]
    bias_first = ((c1 + c2 + t) * sc).astype(np.float16).view(np.uint16)
    no_residual = (c1 * sc + t).astype(np.float16).view(np.uint16)
    assert (w != bias_first).mean() > 0.5
    assert (w != no_residual).mean() > 0.5


def test_rows_and_linear_consistent():
    spec = LayerSpec(40, 200, 8, (12, 8), (0.02, 0.005))
    layer = synth.make_layer(spec, seed=9)
    w = oracle.dequant(layer)
    rows = [3, 0, 39, 17]
    assert np.array_equal(oracle.dequant(layer, rows), w[rows])
    x = synth.make_x(13, 4, 200)
    assert np.array_equal(oracle.linear(layer, x, rows), oracle.linear(layer, x)[:, rows])


# -- products -----------------------------------------------------------------

def test_matmul_matches_numpy_float64():
    rng = np.random.default_rng(4)
    for M, N, K in [(1, 33, 100), (7, 64, 257), (16, 5, 1000)]:
        x = synth.make_x(int(rng.integers(1 << 30)), M, K)
        w = synth.to_f16_bits(rng.standard_normal((N, K)).astype(np.float32) * 0.02)
        y = oracle.matmul(x, w)
        xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        ref = xf @ w.view(np.float16).astype(np.float64).T
        assert np.allclose(y, ref, rtol=1e-12, atol=1e-14 * np.abs(ref).max())
        # fp16 activations
        xh = synth.make_x(5, M, K, as_fp16=True)
        ref = xh.view(np.float16).astype(np.float64) @ w.view(np.float16).astype(np.float64).T
        assert np.allclose(oracle.matmul(xh, w, x_is_fp16=True), ref, rtol=1e-12,
                           atol=1e-14 * np.abs(ref).max())


def test_linear_is_x_times_dequant_transpose_and_rows_independent():
    spec = LayerSpec(50, 6 * 30 + 2, 6, (12, 4), (0.02, 0.005))
    layer = synth.make_layer(spec, seed=6)
    x = synth.make_x(14, 6, spec.in_features, outlier_frac=0.01)
    w = oracle.dequant(layer)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ref = xf @ w.view(np.float16).astype(np.float64).T
    y = oracle.linear(layer, x)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-14 * np.abs(ref).max())
    for b in range(6):      # batch-row independence
        assert np.array_equal(oracle.linear(layer, x[b:b + 1])[0], y[b])


# -- encoders -----------------------------------------------------------------

def test_encode_recovers_generating_indices():
    spec = LayerSpec(32, 64, 8, (8,), (0.02,))
    book = synth.make_layer(spec, seed=21).codebooks[0]
    rng = np.random.default_rng(22)
    idx = rng.integers(0, 256, size=512, dtype=np.uint32)
    v = book.view(np.float16).astype(np.float64)[idx]
    assert np.array_equal(oracle.encode(v, book), idx)
    # a perturbed copy agrees with numpy's argmin (first minimum on ties)
    v2 = v + rng.standard_normal(v.shape) * 0.004
    dist = ((v2[:, None, :] - book.view(np.float16).astype(np.float64)[None]) ** 2).sum(-1)
    assert np.array_equal(oracle.encode(v2, book), dist.argmin(1).astype(np.uint32))


def test_encode_ties_go_to_lowest_index():
    book = np.array([[ONE, 0], [0, ONE], [ONE, 0]], np.uint16)     # rows 0 and 2 equal
    v = np.array([[1.0, 0.0], [0.5, 0.5]])
    assert list(oracle.encode(v, book)) == [0, 0]


def test_two_book_encoders():
    spec = LayerSpec(8, 8, 4, (4, 3), (0.3, 0.01))
    L = synth.make_layer(spec, seed=23)
    b1, b2 = L.codebooks
    rng = np.random.default_rng(24)
    i1 = rng.integers(0, 16, 300, dtype=np.uint32)
    i2 = rng.integers(0, 8, 300, dtype=np.uint32)
    c1 = b1.view(np.float16).astype(np.float64)
    c2 = b2.view(np.float16).astype(np.float64)
    v = c1[i1] + c2[i2]
    j1, j2 = oracle.encode_joint(v, b1, b2)
    assert np.array_equal(c1[j1] + c2[j2], v)           # the generating W_hat
    g1, g2 = oracle.encode_residual(v, b1, b2)           # greedy cascade
    assert np.array_equal(g1, oracle.encode(v, b1))
    r = v - c1[g1]
    dist = ((r[:, None, :] - c2[None]) ** 2).sum(-1)
    assert np.array_equal(g2, dist.argmin(1).astype(np.uint32))


# -- Hessian-weighted encoding --------------------------------------------------
# D_H(v, c) = (v - c)^T H_v (v - c), H_v the sub-matrix of H on the vector's
# channels ("VPTQ Guide", section "1. Second-Order Hessian-Weighted Optimization").

def _f16(vals) -> np.ndarray:
    return np.asarray(vals, np.float16).view(np.uint16)


def _spd(rng, n: int) -> np.ndarray:
    a = rng.standard_normal((n, n))
    return a @ a.T / n + 0.05 * np.eye(n)


def test_encode_h_with_identity_is_the_plain_encoder():
    """H_v = I gives the plain squared distance operation for operation (the
    products by 0 and 1 are exact), so the indices agree bit for bit, also
    for 4 I (a power of two scales every distance exactly), and the weighted
    cascade with I is the plain cascade."""
    spec = LayerSpec(8, 64, 8, (10, 6), (0.05, 0.01))
    L = synth.make_layer(spec, seed=41)
    b1, b2 = L.codebooks
    rng = np.random.default_rng(42)
    v = rng.standard_normal((700, 8)) * 0.05
    eye = np.broadcast_to(np.eye(8), (700, 8, 8))
    assert np.array_equal(oracle.encode_h(v, eye, b1), oracle.encode(v, b1))
    assert np.array_equal(oracle.encode_h(v, 4 * eye, b1), oracle.encode(v, b1))
    g1, g2 = oracle.encode_h_residual(v, eye, b1, b2)
    p1, p2 = oracle.encode_residual(v, b1, b2)
    assert np.array_equal(g1, p1) and np.array_equal(g2, p2)


def test_encode_h_diagonal_hand_worked():
    """Book (1, 0), (0, 1.5), (3, 3); D_H = sum_e H_ee (v_e - c_e)^2 for a
    diagonal H, worked by hand:
      v = (0, 0),     H = I:             1,     2.25,  18      -> 0
      v = (0, 0),     H = diag(4, 1):    4,     2.25,  45      -> 1
      v = (0, 0),     H = diag(1, 4):    1,     9,     45      -> 0
      v = (0.9, 1.2), H = I:             1.45,  0.9,   7.65    -> 1
      v = (0.9, 1.2), H = diag(10, 0.1): 0.244, 8.109, 44.424  -> 0"""
    book = _f16([[1, 0], [0, 1.5], [3, 3]])
    cases = [((0.0, 0.0), (1.0, 1.0), 0), ((0.0, 0.0), (4.0, 1.0), 1), ((0.0, 0.0), (1.0, 4.0), 0),
             ((0.9, 1.2), (1.0, 1.0), 1), ((0.9, 1.2), (10.0, 0.1), 0)]
    for v, hd, want in cases:
        assert list(oracle.encode_h(np.array([v]), np.diag(hd)[None], book)) == [want], (v, hd)
    # the same vectors in one call, each with its own sub-matrix
    vs = np.array([c[0] for c in cases])
    hs = np.stack([np.diag(c[1]) for c in cases])
    assert list(oracle.encode_h(vs, hs, book)) == [c[2] for c in cases]


def test_encode_h_off_diagonal_hand_worked():
    """H = [[1, 0.75], [0.75, 1]], v = 0: (1, 1) -> 1 + 1 + 2 * 0.75 = 3.5;
    (1, -1.25) -> 1 + 1.5625 - 2 * 0.75 * 1.25 = 0.6875: picks 1, where the
    plain distances 2 and 2.5625 pick 0.  The cross term's sign matters: with
    -0.75 off the diagonal the distances become 0.5 and 4.4375 (picks 0)."""
    book = _f16([[1, 1], [1, -1.25]])
    v = np.zeros((1, 2))
    assert list(oracle.encode(v, book)) == [0]
    assert list(oracle.encode_h(v, np.array([[[1.0, 0.75], [0.75, 1.0]]]), book)) == [1]
    assert list(oracle.encode_h(v, np.array([[[1.0, -0.75], [-0.75, 1.0]]]), book)) == [0]
    # a non-symmetric H weighs like its symmetric part: (v-c)^T H (v-c)
    assert list(oracle.encode_h(v, np.array([[[1.0, 1.5], [0.0, 1.0]]]), book)) == [1]


def test_encode_h_ties_go_to_lowest_index():
    book = _f16([[1, 0], [0, 1], [1, 0]])
    h = np.array([[[2.0, 0.0], [0.0, 2.0]]])
    assert list(oracle.encode_h(np.array([[1.0, 0.0]]), h, book)) == [0]
    assert list(oracle.encode_h(np.array([[0.5, 0.5]]), h, book)) == [0]


@pytest.mark.parametrize("d,kin", [(8, 8 * 12), (6, 6 * 10 + 4)])
def test_encode_h_matches_numpy_brute_force_on_layer_blocks(d, kin):
    """A random SPD Hessian of a small layer: the oracle with each vector's
    sub-matrix (hessian_blocks) agrees with numpy's einsum distances and
    argmin, for whole vectors and the partial last one; the chosen distance is
    numpy's minimum.  Taking the neighbouring block instead changes answers."""
    rng = np.random.default_rng(43 + d)
    rows = 9
    h = _spd(rng, kin)
    book = synth.to_f16_bits(rng.standard_normal((64, d)).astype(np.float32) * 0.3).reshape(64, d)
    w = rng.standard_normal((rows, kin)) * 0.3
    full, last = oracle.hessian_blocks(h, kin, d, rows)
    nfull, rem = kin // d, kin % d
    assert (rem == 0) == (last is None)
    v = w[:, :nfull * d].reshape(rows * nfull, d)
    got = oracle.encode_h(v, full, book)
    c = book.view(np.float16).astype(np.float64)
    jj = np.tile(np.arange(nfull), rows)
    t = v[:, None, :] - c[None]                                   # [nv][K][d]
    blocks = np.stack([h[j * d:(j + 1) * d, j * d:(j + 1) * d] for j in jj])
    dist = np.einsum("nke,nef,nkf->nk", t, blocks, t)
    assert np.array_equal(got, dist.argmin(1).astype(np.uint32))
    chosen = dist[np.arange(len(got)), got]
    assert np.allclose(chosen, dist.min(1), rtol=1e-12, atol=0)
    # the sub-matrix is the vector's own: the neighbouring block moves answers
    shifted = np.stack([h[((j + 1) % nfull) * d:((j + 1) % nfull + 1) * d,
                          ((j + 1) % nfull) * d:((j + 1) % nfull + 1) * d] for j in jj])
    assert (oracle.encode_h(v, shifted, book) != got).mean() > 0.05
    # and the weighting moves answers against the plain distance
    assert (oracle.encode(v, book) != got).mean() > 0.05
    if rem:
        vl = np.ascontiguousarray(w[:, nfull * d:])
        bl = np.ascontiguousarray(book[:, :rem])
        gl = oracle.encode_h(vl, last, bl)
        hl = h[nfull * d:, nfull * d:]
        tl = vl[:, None, :] - bl.view(np.float16).astype(np.float64)[None]
        dl = np.einsum("nke,ef,nkf->nk", tl, hl, tl)
        assert np.array_equal(gl, dl.argmin(1).astype(np.uint32))


def test_encode_h_residual_matches_numpy():
    rng = np.random.default_rng(47)
    d = 8
    spec = LayerSpec(8, 64, d, (6, 4), (0.3, 0.05))
    b1, b2 = synth.make_layer(spec, seed=48).codebooks
    v = rng.standard_normal((200, d)) * 0.3
    hb = np.stack([_spd(rng, d) for _ in range(200)])
    g1, g2 = oracle.encode_h_residual(v, hb, b1, b2)
    c1 = b1.view(np.float16).astype(np.float64)
    c2 = b2.view(np.float16).astype(np.float64)
    t1 = v[:, None] - c1[None]
    assert np.array_equal(g1, np.einsum("nke,nef,nkf->nk", t1, hb, t1).argmin(1))
    r = v - c1[g1]
    t2 = r[:, None] - c2[None]
    assert np.array_equal(g2, np.einsum("nke,nef,nkf->nk", t2, hb, t2).argmin(1))


def test_hessian_blocks_pick_the_vector_channels():
    kin, d, rows = 14, 4, 2
    h = np.arange(kin)[:, None] * 100.0 + np.arange(kin)[None, :]
    full, last = oracle.hessian_blocks(h, kin, d, rows)
    assert full.shape == (rows * 3, d, d) and last.shape == (rows, 2, 2)
    assert full[1][0, 0] == 4 * 100 + 4 and full[1][3, 2] == 7 * 100 + 6
    assert full[3 + 2][1, 3] == 9 * 100 + 11                     # row 1, vector 2
    assert last[1].tolist() == [[1212.0, 1213.0], [1312.0, 1313.0]]


# -- randomized Hadamard transform ----------------------------------------------

def _signs(n, seed):
    rng = np.random.default_rng(seed)
    bits = rng.integers(0, 2, size=n).astype(np.uint8)
    words = np.packbits(np.concatenate([bits, np.zeros((-n) % 32, np.uint8)]), bitorder="little")
    return words.view(np.uint32), np.where(bits == 1, -1.0, 1.0)


def test_rht_hand_worked_example():
    """H_4 = [[1,1,1,1],[1,-1,1,-1],[1,1,-1,-1],[1,-1,-1,1]] (Sylvester), signs
    (+1, -1, +1, +1): x = (1, 2, 3, 4) -> H (1, -2, 3, 4) / 2 = (3, 1, -4, 2)."""
    x = np.array([[1.0, 2.0, 3.0, 4.0]])
    signs = np.array([0b0010], np.uint32)
    assert np.array_equal(oracle.rht(x, signs), [[3.0, 1.0, -4.0, 2.0]])
    assert np.array_equal(oracle.rht(x, np.zeros(1, np.uint32)), [[5.0, -1.0, -2.0, 0.0]])
    # the inverse undoes it: signs applied after H
    assert np.allclose(oracle.rht(np.array([[3.0, 1.0, -4.0, 2.0]]), signs, inverse=True), x, atol=1e-15)


def test_rht_block_rule():
    """Blocks: the largest power of two dividing n, at most 2^15."""
    for n, b in [(1, 1), (7, 1), (12, 4), (6, 2), (8192, 8192), (28672, 4096), (53248, 4096),
                 (16384, 16384), (1 << 20, 32768), (3 * 32768, 32768)]:
        assert oracle.rht_block(n) == b, n


@pytest.mark.parametrize("n", [8, 24, 96, 1024 + 512])
def test_rht_matches_a_library_hadamard_and_is_orthogonal(n):
    """Against scipy's Sylvester Hadamard matrix, block-diagonal with random
    signs; forward then inverse returns x; norms are preserved."""
    from scipy.linalg import hadamard, block_diag
    words, s = _signs(n, 70 + n)
    b = oracle.rht_block(n)
    V = block_diag(*[hadamard(b)] * (n // b)) @ np.diag(s) / np.sqrt(b)
    rng = np.random.default_rng(n)
    x = rng.standard_normal((3, n))
    y = oracle.rht(x, words)
    assert np.allclose(y, x @ V.T, atol=1e-12)
    assert np.allclose(oracle.rht(y, words, inverse=True), x, atol=1e-12)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    assert np.allclose(V @ V.T, np.eye(n), atol=1e-12)


def test_rht_layer_identity():
    """W x = U^T ((U W V^T) (V x)) for orthogonal U, V (the QuIP# identity)."""
    rng = np.random.default_rng(5)
    N, K = 48, 40                      # blocks of 16 and 8
    W = rng.standard_normal((N, K))
    x = rng.standard_normal(K)
    su, _ = _signs(N, 6)
    sv, _ = _signs(K, 7)
    WVt = oracle.rht(W, sv)                              # rows: W V^T
    Wt = oracle.rht(WVt.T.copy(), su).T                  # columns: U (W V^T)
    xt = oracle.rht(x[None, :], sv)[0]                   # V x
    y = oracle.rht((Wt @ xt)[None, :], su, inverse=True)[0]
    assert np.allclose(y, W @ x, atol=1e-12)


# -- Hessian collection -----------------------------------------------------------

def test_hessian_closed_forms():
    """All-ones tokens: H = 2 n J, h = 2 J, damp = 0.01 * 2 -> 2 J + 0.02 I.
    One-hot tokens e_(t mod d): h = 2 diag(counts) / n + 0.01 * mean."""
    d, n = 8, 40
    ones = oracle.f32_to_bf16(np.ones((n, d), np.float32))
    h = oracle.hessian(ones)
    assert np.allclose(h, 2.0 * np.ones((d, d)) + 0.02 * np.eye(d), atol=1e-15)
    onehot = np.zeros((n, d), np.float32)
    onehot[np.arange(n), np.arange(n) % d] = 1.0
    h = oracle.hessian(oracle.f32_to_bf16(onehot))
    counts = np.bincount(np.arange(n) % d, minlength=d)
    base = 2.0 * np.diag(counts) / n
    assert np.allclose(h, base + 0.01 * np.trace(base) / d * np.eye(d), atol=1e-15)


def test_hessian_matches_numpy():
    """Against numpy: 2 X^T X / n (fp64 matmul) plus 0.01 * mean(diag) I; symmetric."""
    rng = np.random.default_rng(9)
    n, d = 300, 48
    xb = oracle.f32_to_bf16(rng.standard_normal((n, d), dtype=np.float32))
    x = oracle.bf16_to_f32(xb).astype(np.float64)
    h0 = 2.0 * x.T @ x / n
    ref = h0 + 0.01 * np.mean(np.diag(h0)) * np.eye(d)
    h = oracle.hessian(xb)
    assert np.allclose(h, ref, rtol=1e-13, atol=1e-13)
    assert np.array_equal(h, h.T)
    xf = oracle.f32_to_f16(rng.standard_normal((n, d), dtype=np.float32))
    x = oracle.f16_to_f32(xf).astype(np.float64)
    h0 = 2.0 * x.T @ x / n
    assert np.allclose(oracle.hessian(xf, x_is_fp16=True), h0 + 0.01 * np.mean(np.diag(h0)) * np.eye(d),
                       rtol=1e-13, atol=1e-13)

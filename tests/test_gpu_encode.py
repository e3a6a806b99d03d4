"""GPU parity for the nearest-centroid encoder (vq_encode), through the C ABI.

The encoder's result is an integer per vector, fixed by the definition
idx = argmin_k sum_e (v_e - C[k][e])^2 in fp64, ties to the lowest k (the
oracle's brute force); the packed streams must equal the oracle's packer word
for word.  Cases: one book and the two-book greedy cascade; d = 1, 6, 8, 14;
books from 2^3 to 2^16 entries (smaller than one staged block of 1024, and
not); partial last vectors; exact ties (duplicate centroids, midpoints);
weights far larger than the centroids; a 4096 x 4096 layer on sampled rows;
and the fixed point encode(dequant(encode(W))) = encode(W)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._util import sample_rows

pytestmark = pytest.mark.gpu


def _vq():
    from bit_packed_index_b200 import vq
    return vq


def _dev16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.float16)


def _oracle_idx(w_bits, books, d, rows=None):
    """Per book, idx [len(rows)][nvec] from the oracle's encoders."""
    w_bits = w_bits if rows is None else w_bits[rows]
    n, kin = w_bits.shape
    nvec, nfull, rem = -(-kin // d), kin // d, kin % d
    wf = oracle.f16_to_f32(w_bits).astype(np.float64)
    out = [np.zeros((n, nvec), np.uint32) for _ in books]
    parts = []
    if nfull:
        parts.append((slice(0, nfull), wf[:, :nfull * d].reshape(n * nfull, d), books))
    if rem:
        parts.append((slice(nfull, nfull + 1), np.ascontiguousarray(wf[:, nfull * d:]),
                      [np.ascontiguousarray(b[:, :rem]) for b in books]))
    for cols, v, bk in parts:
        width = cols.stop - cols.start
        if len(books) == 1:
            out[0][:, cols] = oracle.encode(v, bk[0]).reshape(n, width)
        else:
            i1, i2 = oracle.encode_residual(v, bk[0], bk[1])
            out[0][:, cols] = i1.reshape(n, width)
            out[1][:, cols] = i2.reshape(n, width)
    return out


def _gpu_encode(w_bits, books, log2k, d):
    vq = _vq()
    n, kin = w_bits.shape
    ws = torch.full((max(256, vq.encode_workspace_size(n, kin, log2k, d)),), 0x5A, dtype=torch.uint8,
                    device="cuda")                      # stale workspace contents are fine
    layer = vq.encode(_dev16(w_bits), [_dev16(b) for b in books], log2k, d, workspace=ws)
    torch.cuda.synchronize()
    ctrl = ws[:16].view(torch.int32).cpu().numpy()
    streams = [t.cpu().numpy().view(np.uint32) for t in layer.idx]
    return layer, streams, ctrl


def _check(w_bits, books, log2k, d):
    n, kin = w_bits.shape
    nvec = -(-kin // d)
    layer, streams, ctrl = _gpu_encode(w_bits, books, log2k, d)
    assert ctrl[0] == 0                                 # device status word
    ref = _oracle_idx(w_bits, books, d)
    for m, b in enumerate(log2k):
        got = oracle.unpack(streams[m], b, nvec)
        bad = np.argwhere(got != ref[m])
        assert bad.size == 0, f"book {m}: {len(bad)} of {got.size} differ, first {bad[:4].tolist()}"
        assert np.array_equal(streams[m], oracle.pack(ref[m], b, streams[m].shape[1]))
    return layer, ctrl


SPECS = [
    # N, Kin, d, log2k, book std
    (1, 8, 8, (4,), (0.02,)),                    # K = 16: one padded staged block
    (37, 8 * 21 + 3, 8, (10,), (0.02,)),         # partial last vector
    (64, 6 * 50 + 4, 6, (12,), (0.02,)),         # d = 6 as in the 405B layers
    (130, 64, 8, (16,), (0.02,)),                # K = 2^16, 1040 vectors: a ragged last block
    (20, 14 * 10, 14, (8,), (0.5,)),             # largest d
    (50, 33, 1, (3,), (1.0,)),                   # d = 1, K = 8
    (3, 5, 8, (6,), (0.02,)),                    # Kin < d: only partial vectors
    (40, 8 * 30 + 5, 8, (12, 8), (0.02, 0.005)), # two books, greedy residual
    (33, 6 * 20 + 2, 6, (12, 4), (0.02, 0.005)), # 405B-style pair, partial vector
    (16, 128, 8, (16, 16), (0.02, 0.005)),       # two 2^16 books
]


@pytest.mark.parametrize("i", range(len(SPECS)))
def test_encode_matches_the_oracle(i):
    n, kin, d, log2k, std = SPECS[i]
    w, books = synth.make_encode_input(n, kin, d, log2k, std, seed=3100 + i)
    _check(w, books, list(log2k), d)


def test_exact_ties_go_to_the_lowest_index():
    """Duplicate centroids and vectors midway between two centroids: the
    tensor-core margin is zero, the exact pass decides, ties to the lowest k."""
    d, K = 8, 16
    rng = np.random.default_rng(3200)
    book = rng.integers(-3, 4, size=(K, d)).astype(np.float32)
    book[9] = book[4]                                  # a duplicate pair (4 wins)
    book[12] = book[2]
    vecs = [book[4], book[2], book[9]]
    for a, b in [(0, 1), (3, 5), (7, 11), (6, 13)]:
        vecs.append((book[a] + book[b]) / 2)           # exact midpoints (integers / 2)
    vecs += [book[k] for k in range(K)]
    w = synth.to_f16_bits(np.stack(vecs).reshape(1, -1))
    _check(w, [synth.to_f16_bits(book).reshape(K, d)], [4], d)


def test_all_equal_centroids_and_large_weights():
    """A book whose rows are all equal (every vector ties: index 0), and
    weights 10^4 times the centroids (fp16 cannot hold the scaled operand:
    those vectors go to the exact pass)."""
    d = 8
    book = synth.to_f16_bits(np.full((256, d), 0.25, np.float32)).reshape(256, d)
    w, _ = synth.make_encode_input(8, 64, d, [8], [0.02], seed=3210)
    _check(w, [book], [8], d)
    w2, books = synth.make_encode_input(8, 8 * 16, d, [10], [0.01], seed=3211, w_std=100.0)
    _check(w2, books, [10], d)


def test_recovers_generating_indices_and_is_a_fixed_point():
    """W = C[idx] exactly (unique rows): the encoder returns idx; and the
    dequantised encoding of any W encodes to itself."""
    vq = _vq()
    d, b, n, kin = 8, 12, 96, 8 * 64
    w, books = synth.make_encode_input(n, kin, d, [b], [0.02], seed=3220)
    rng = np.random.default_rng(3221)
    idx = rng.integers(0, 1 << b, size=(n, kin // d)).astype(np.uint32)
    wc = books[0][idx].reshape(n, kin)
    layer, _ = _check(wc, books, [b], d)
    got = oracle.unpack(layer.idx[0].cpu().numpy().view(np.uint32), b, kin // d)
    assert np.array_equal(got, idx)
    # fixed point on a random W
    layer, _ = _check(w, books, [b], d)
    w_hat = vq.dequant(layer)
    layer2 = vq.encode(w_hat, layer.codebooks, [b], d)
    assert torch.equal(layer2.idx[0], layer.idx[0])


def test_large_layer_sampled_rows():
    """A 4096 x 4096 layer, d = 8, K = 2^16 (2M vectors) encoded whole; the
    oracle checks a sample of rows."""
    n, kin, d, b = 4096, 4096, 8, 16
    w, books = synth.make_encode_input(n, kin, d, [b], [0.02], seed=3230)
    layer, streams, ctrl = _gpu_encode(w, books, [b], d)
    assert ctrl[0] == 0
    rows = sample_rows(n, 6, 3231)
    ref = _oracle_idx(w, books, d, rows)[0]
    got = oracle.unpack(streams[0][rows], b, kin // d)
    assert np.array_equal(got, ref)
    # vectors the tensor-core pass left to the exact pass: a small share
    assert 0 <= ctrl[1] < 0.05 * n * (kin // d), ctrl[1]


def test_empty_shapes():
    vq = _vq()
    book = _dev16(synth.make_encode_input(1, 8, 8, [4], [0.02], 1)[1][0])
    for n, kin in ((0, 16), (4, 0)):
        w = torch.zeros((n, kin), dtype=torch.float16, device="cuda")
        layer = vq.encode(w, [book], [4], 8)
        torch.cuda.synchronize()
        assert layer.idx[0].shape[0] == n
        if n:
            assert int(layer.idx[0].abs().sum()) == 0

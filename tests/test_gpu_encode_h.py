"""GPU parity for the Hessian-weighted encoder (vq_encode with a Hessian),
through the C ABI, against the oracle's brute force.

The result is an integer per vector fixed by the definition
idx = argmin_k (v - C[k])^T H_v (v - C[k]) in fp64 (H_v the sub-matrix of H
on the vector's channels), ties to the lowest k ("VPTQ Guide", section
"1. Second-Order Hessian-Weighted Optimization"); the packed streams must
equal the oracle's packer word for word.  Hessians come from synthetic
activations with outlier channels (H = 2 X^T X / n + 0.01 mean(diag) I,
rounded to fp32 as vq_hessian returns it).  Cases: one book and the weighted cascade;
d = 6 and 8; books from 2^4 to 2^16 entries; partial last vectors; more
rows than one 128-row block (ragged); H = I against the plain encoder;
a non-symmetric and an indefinite H; exact ties; a 4096 x 4096 layer on
sampled rows."""
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


def _hessian32(kin: int, seed: int, tokens: int = 256, outliers: float = 0.02) -> np.ndarray:
    """fp32 H = 2 X^T X / n + 0.01 mean(diag) I of synthetic bf16 activations
    with outlier channels (the collector's formula, in numpy's fp64 matmul,
    rounded once): an input of the encoder, whose result is then fixed."""
    x = oracle.bf16_to_f32(synth.make_x(seed, tokens, kin, outlier_frac=outliers)).astype(np.float64)
    h = 2.0 * (x.T @ x) / tokens
    h[np.diag_indices(kin)] += 0.01 * np.diag(h).mean()
    return h.astype(np.float32)


def _oracle_idx_h(w_bits, books, d, h32, rows=None):
    """Per book, idx [len(rows)][nvec] from the oracle's weighted encoders."""
    w_bits = w_bits if rows is None else w_bits[rows]
    n, kin = w_bits.shape
    nvec, nfull, rem = -(-kin // d), kin // d, kin % d
    wf = oracle.f16_to_f32(w_bits).astype(np.float64)
    full, last = oracle.hessian_blocks(h32.astype(np.float64), kin, d, n)
    out = [np.zeros((n, nvec), np.uint32) for _ in books]
    parts = []
    if nfull:
        parts.append((slice(0, nfull), wf[:, :nfull * d].reshape(n * nfull, d), full, books))
    if rem:
        parts.append((slice(nfull, nfull + 1), np.ascontiguousarray(wf[:, nfull * d:]), last,
                      [np.ascontiguousarray(b[:, :rem]) for b in books]))
    for cols, v, hb, bk in parts:
        width = cols.stop - cols.start
        if len(books) == 1:
            out[0][:, cols] = oracle.encode_h(v, hb, bk[0]).reshape(n, width)
        else:
            i1, i2 = oracle.encode_h_residual(v, hb, bk[0], bk[1])
            out[0][:, cols] = i1.reshape(n, width)
            out[1][:, cols] = i2.reshape(n, width)
    return out


def _gpu_encode_h(w_bits, books, log2k, d, h32):
    vq = _vq()
    n, kin = w_bits.shape
    size = vq.encode_workspace_size(n, kin, log2k, d, hessian=True)
    ws = torch.full((max(256, size),), 0x5A, dtype=torch.uint8, device="cuda")   # stale contents
    h = torch.from_numpy(np.ascontiguousarray(h32)).cuda()
    layer = vq.encode(_dev16(w_bits), [_dev16(b) for b in books], log2k, d, workspace=ws, hessian=h)
    torch.cuda.synchronize()
    ctrl = ws[:16].view(torch.int32).cpu().numpy()
    streams = [t.cpu().numpy().view(np.uint32) for t in layer.idx]
    return layer, streams, ctrl


def _check(w_bits, books, log2k, d, h32):
    n, kin = w_bits.shape
    nvec = -(-kin // d)
    layer, streams, ctrl = _gpu_encode_h(w_bits, books, log2k, d, h32)
    assert ctrl[0] == 0                                 # device status word
    ref = _oracle_idx_h(w_bits, books, d, h32)
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
    (130, 64, 8, (16,), (0.02,)),                # K = 2^16, two 128-row blocks per channel block
    (300, 8 * 16, 8, (8,), (0.02,)),             # 300 rows: 128 + 128 + 44
    (3, 5, 8, (6,), (0.02,)),                    # Kin < d: only partial vectors
    (40, 8 * 30 + 5, 8, (12, 8), (0.02, 0.005)), # two books, weighted cascade
    (33, 6 * 20 + 2, 6, (12, 4), (0.02, 0.005)), # 405B-style pair, partial vector
    (16, 128, 8, (16, 16), (0.02, 0.005)),       # two 2^16 books
]


@pytest.mark.parametrize("i", range(len(SPECS)))
def test_encode_h_matches_the_oracle(i):
    n, kin, d, log2k, std = SPECS[i]
    w, books = synth.make_encode_input(n, kin, d, log2k, std, seed=5100 + i)
    _check(w, books, list(log2k), d, _hessian32(kin, 5150 + i))


def test_identity_hessian_is_the_plain_encoder():
    """H = I: the weighted streams equal the plain encoder's, word for word."""
    vq = _vq()
    n, kin, d = 96, 8 * 40 + 3, 8
    w, books = synth.make_encode_input(n, kin, d, [12, 8], [0.02, 0.005], seed=5200)
    layer, _ = _check(w, books, [12, 8], d, np.eye(kin, dtype=np.float32))
    plain = vq.encode(_dev16(w), [_dev16(b) for b in books], [12, 8], d)
    torch.cuda.synchronize()
    for a, b in zip(layer.idx, plain.idx):
        assert torch.equal(a, b)


def test_non_symmetric_and_indefinite_hessians():
    """The definition takes H as given: a non-symmetric H (weighs like its
    symmetric part) and an indefinite one (negative directions: distances may
    be negative) are both decided exactly."""
    n, kin, d = 50, 8 * 24, 8
    w, books = synth.make_encode_input(n, kin, d, [10], [0.02], seed=5300)
    h = _hessian32(kin, 5301).astype(np.float64)
    rng = np.random.default_rng(5302)
    skew = rng.standard_normal((kin, kin)) * 0.1 * np.abs(h).mean()
    _check(w, books, [10], d, (h + skew - skew.T).astype(np.float32))
    shifted = h - 2.0 * np.diag(h).mean() * np.eye(kin)          # many negative eigenvalues
    assert np.linalg.eigvalsh(shifted).min() < 0
    _check(w, books, [10], d, shifted.astype(np.float32))


def test_exact_ties_go_to_the_lowest_index():
    """Duplicate centroids and exact midpoints under a diagonal H: zero
    margins, the exact pass decides, ties to the lowest k."""
    d, K = 8, 16
    rng = np.random.default_rng(5400)
    book = rng.integers(-3, 4, size=(K, d)).astype(np.float32)
    book[9] = book[4]
    book[12] = book[2]
    vecs = [book[4], book[2], book[9]]
    for a, b in [(0, 1), (3, 5), (7, 11), (6, 13)]:
        vecs.append((book[a] + book[b]) / 2)
    vecs += [book[k] for k in range(K)]
    w = synth.to_f16_bits(np.stack(vecs).reshape(1, -1))
    kin = w.shape[1]
    h = np.diag(rng.choice([0.5, 1.0, 2.0, 4.0], size=kin)).astype(np.float32)
    _check(w, [synth.to_f16_bits(book).reshape(K, d)], [4], d, h)


def test_large_layer_sampled_rows():
    """A 4096 x 4096 layer, d = 8, K = 2^16 (2M vectors) with the Hessian of
    1024 synthetic tokens, encoded whole; the oracle checks sampled rows."""
    n, kin, d, b = 4096, 4096, 8, 16
    w, books = synth.make_encode_input(n, kin, d, [b], [0.02], seed=5500)
    h32 = _hessian32(kin, 5501, tokens=1024)
    layer, streams, ctrl = _gpu_encode_h(w, books, [b], d, h32)
    assert ctrl[0] == 0
    rows = sample_rows(n, 4, 5502)
    ref = _oracle_idx_h(w, books, d, h32, rows)[0]
    got = oracle.unpack(streams[0][rows], b, kin // d)
    assert np.array_equal(got, ref)
    assert 0 <= ctrl[1] < 0.05 * n * (kin // d), ctrl[1]


def test_rejects_wide_vectors_and_short_strides():
    vq = _vq()
    w, books = synth.make_encode_input(4, 40, 10, [4], [0.02], seed=5600)
    h = torch.eye(40, dtype=torch.float32, device="cuda")
    with pytest.raises(vq.VQError) as e:
        vq.encode(_dev16(w), [_dev16(books[0])], [4], 10, hessian=h)
    assert e.value.status == vq.VQ_ERR_UNSUPPORTED
    with pytest.raises(vq.VQError) as e:
        vq.encode(_dev16(np.ascontiguousarray(w[:, :32])), [_dev16(np.ascontiguousarray(books[0][:, :8]))], [4], 8,
                  hessian=torch.eye(16, dtype=torch.float32, device="cuda"))   # ldh 16 < Kin 32
    assert e.value.status == vq.VQ_ERR_INVALID_ARG

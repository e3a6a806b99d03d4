"""GPU parity for the tiled index order (VQ_IDX_TILE4), through the C ABI.

- vq_repack_tile4 writes, word for word, what the oracle's tiled packer
  writes for the same indices;
- layers whose tiled streams come from the oracle's packer (not from the
  library) give vq_dequant bit-exact and vq_gemv / vq_gemm within the bar, so
  the kernels read the documented order and not just whatever repack writes;
- the lookup-table GEMVs (batch 1: one 2^16-entry book at d = 8, sliced; or
  books of up to 2^12 entries at d = 6 or 8, whole) are checked on ragged
  shapes, every block-row size they compile for, both activation types, every
  output type, scale/bias present and absent, large and small activation
  magnitudes, and the 70B / 405B / 8B decode shapes on sampled rows; the
  split-K gather kernel reading tiled records on every other case."""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth import LayerSpec, WORKLOADS
from tests._util import assert_close, sample_rows

pytestmark = pytest.mark.gpu


def _vq():
    from bit_packed_index_b200 import vq
    return vq


def _x_dev(x_bits: np.ndarray, fp16: bool = False) -> torch.Tensor:
    t = torch.from_numpy(x_bits.view(np.int16)).cuda()
    return t.view(torch.float16 if fp16 else torch.bfloat16)


def _w_bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def _garbage(tiles, b, n, nvec, seed):
    """Random bits wherever the format says bits are ignored: fields of vectors
    >= nvec in the last tile, and every bit past the N records of a tile."""
    rng = np.random.default_rng(seed)
    bits = np.unpackbits(tiles.view(np.uint8), axis=1, bitorder="little")
    bits[:, n * 4 * b:] = rng.integers(0, 2, size=bits[:, n * 4 * b:].shape, dtype=np.uint8)
    if nvec % 4:
        rec = bits[-1, : n * 4 * b].reshape(n, 4, b)
        rec[:, nvec % 4:, :] = rng.integers(0, 2, size=rec[:, nvec % 4:, :].shape, dtype=np.uint8)
        bits[-1, : n * 4 * b] = rec.reshape(-1)
    return np.packbits(bits, axis=1, bitorder="little").view(np.uint32).reshape(tiles.shape)


def _oracle_tiled_layer(data, extra_words=0, garbage=False):
    """A device layer whose tiled streams the oracle packed (never the library);
    with ``garbage`` every ignored bit is random."""
    vq = _vq()
    s = data.spec
    tiles = []
    for m, b in enumerate(s.log2k):
        idx = oracle.unpack(data.idx_words[m], b, s.nvec)
        t = oracle.pack_tile4(idx, b, oracle.tile4_words(s.out_features, b) + extra_words)
        if garbage:
            t = _garbage(t, b, s.out_features, s.nvec, seed=77 + m)
            assert np.array_equal(oracle.unpack_tile4(t, b, s.out_features, s.nvec), idx)
        tiles.append(t)
    layer = vq.Layer.from_host(s.out_features, s.in_features, s.d, s.log2k, tiles,
                               data.codebooks, data.scale, data.bias)
    layer.layout = "tile4"
    return layer


REPACK_SPECS = [
    LayerSpec(37, 8 * 45 + 3, 8, (16,), (0.02,)),
    LayerSpec(29, 6 * 50 + 4, 6, (12, 4), (0.02, 0.005)),
    LayerSpec(33, 7 * 9 + 2, 7, (3, 5), (0.02, 0.005)),
    LayerSpec(1, 1, 1, (1,), (0.02,)),
    LayerSpec(1000, 8 * 4, 8, (16,), (0.02,)),
    LayerSpec(17, 16 * 5, 16, (13, 2), (0.02, 0.005)),
]


@pytest.mark.parametrize("i", range(len(REPACK_SPECS)))
@pytest.mark.parametrize("extra", [0, 8])
def test_repack_matches_the_oracle_packer(i, extra):
    vq = _vq()
    spec = REPACK_SPECS[i]
    data = synth.make_layer(spec, seed=2100 + i, pad_garbage=True)
    rows = vq.Layer.from_synth(data)
    tw = [vq.tile4_words(spec.out_features, b) + extra for b in spec.log2k]
    tiled = vq.repack_tile4(rows, tile_words=tw)
    assert [tuple(t.shape) for t in tiled.idx] == [(-(-spec.nvec // 4), w) for w in tw]
    torch.cuda.synchronize()
    for m, b in enumerate(spec.log2k):
        idx = oracle.unpack(data.idx_words[m], b, spec.nvec)
        want = oracle.pack_tile4(idx, b, tw[m])
        got = tiled.idx[m].cpu().numpy().view(np.uint32)
        assert np.array_equal(got, want)


def test_repack_overwrites_every_word():
    vq = _vq()
    spec = LayerSpec(50, 8 * 13, 8, (16,), (0.02,))
    data = synth.make_layer(spec, seed=2200)
    rows = vq.Layer.from_synth(data)
    tw = vq.tile4_words(50, 16) + 4
    dst = torch.full((4, tw), -1, dtype=torch.int32, device="cuda")
    import ctypes as C
    ptrs = (C.c_void_p * 2)(dst.data_ptr(), 0)
    words = (C.c_int64 * 2)(tw, 0)
    assert vq.lib().vq_repack_tile4(C.byref(rows.desc()), ptrs, words, None) == vq.VQ_OK
    torch.cuda.synchronize()
    want = oracle.pack_tile4(oracle.unpack(data.idx_words[0], 16, spec.nvec), 16, tw)
    assert np.array_equal(dst.cpu().numpy().view(np.uint32), want)


DQ_SPECS = REPACK_SPECS + [
    LayerSpec(300, 1000, 8, (12, 8), (0.02, 0.005)),
    LayerSpec(130, 6 * 200 + 1, 6, (16,), (0.02,), None, None),
    LayerSpec(64, 510, 6, (12, 4), (0.02, 0.005), None, 1e-3),
]


@pytest.mark.parametrize("i", range(len(DQ_SPECS)))
def test_dequant_tiled_bit_exact(i):
    spec = DQ_SPECS[i]
    data = synth.make_layer(spec, seed=2300 + i)
    want = oracle.dequant(data)
    for layer in (_oracle_tiled_layer(data, extra_words=4 * (i % 2)),
                  _vq().repack_tile4(_vq().Layer.from_synth(data))):
        w = _vq().dequant(layer)
        torch.cuda.synchronize()
        assert np.array_equal(_w_bits(w), want)


# Lookup-table kernel cases: (N, Kin, scale/bias) covering N below one block
# row, N on and just past the 1024 * 8 * {1, 2, 4} boundaries of the
# per-thread row batches, nvec not a multiple of 4, and Kin not a multiple
# of 8 (a partial last vector).
LUT_SPECS = [
    LayerSpec(1, 8, 8, (16,), (0.02,)),
    LayerSpec(777, 8 * 125, 8, (16,), (0.02,)),
    LayerSpec(1000, 1001, 8, (16,), (0.02,)),
    LayerSpec(8192, 8 * 64, 8, (16,), (0.02,), None, None),
    LayerSpec(8193, 8 * 66 + 5, 8, (16,), (0.02,)),
    LayerSpec(16385, 8 * 33, 8, (16,), (0.02,), (0.5, 1.5), None),
    LayerSpec(40000, 8 * 20, 8, (16,), (0.02,), None, 1e-3),
    LayerSpec(65536, 8 * 8, 8, (16,), (0.02,)),
]


@pytest.mark.parametrize("i", range(len(LUT_SPECS)))
def test_lut_gemv(i):
    vq = _vq()
    spec = LUT_SPECS[i]
    data = synth.make_layer(spec, seed=2400 + i)
    layer = _oracle_tiled_layer(data)
    nws = vq.gemv_workspace_size(layer, 1)
    assert nws > 0                                          # the lookup-table plan
    ws = torch.full((nws,), 0x55, dtype=torch.uint8, device="cuda")   # stale contents are fine
    for fp16 in (False, True):
        x = synth.make_x(2450 + i, 1, spec.in_features, outlier_frac=0.01, as_fp16=fp16)
        ref = oracle.linear(data, x, x_is_fp16=fp16)
        for od in (torch.float32, torch.bfloat16, torch.float16):
            y = vq.gemv(layer, _x_dev(x, fp16), out_dtype=od, workspace=ws)
            assert_close(_f64(y), ref, str(od).split(".")[-1])


@pytest.mark.parametrize("mag", [1e-3, 1.0, 1e3])
def test_lut_gemv_activation_magnitudes(mag):
    """The per-group power-of-two scaling keeps the fp16 table in range and
    precise for small and large activations alike."""
    vq = _vq()
    spec = LayerSpec(3000, 8 * 300, 8, (16,), (0.02,))
    data = synth.make_layer(spec, seed=2500)
    layer = _oracle_tiled_layer(data)
    x = synth.make_x(2501, 1, spec.in_features, outlier_frac=0.01)
    xf = oracle.bf16_to_f32(x) * np.float32(mag)
    xb = oracle.f32_to_bf16(xf)
    ref = oracle.linear(data, xb)
    y = vq.gemv(layer, _x_dev(xb), out_dtype=torch.float32)
    assert_close(_f64(y), ref, "float32")


def test_lut_gemv_all_zero_input_and_single_outlier():
    vq = _vq()
    spec = LayerSpec(2000, 8 * 100, 8, (16,), (0.02,))
    data = synth.make_layer(spec, seed=2510)
    layer = _oracle_tiled_layer(data)
    x = np.zeros((1, spec.in_features), np.uint16)
    y = vq.gemv(layer, _x_dev(x), out_dtype=torch.float32)
    assert_close(_f64(y), oracle.linear(data, x), "float32")
    x = oracle.f32_to_bf16(np.zeros((1, spec.in_features), np.float32))
    x[0, 437] = oracle.f32_to_bf16(np.array([300.0], np.float32))[0]
    y = vq.gemv(layer, _x_dev(x), out_dtype=torch.float32)
    assert_close(_f64(y), oracle.linear(data, x), "float32")


# Batches 1..16 on tiled layers: small batches of table-eligible layers run one
# table pass per row of x, everything else the split-K gather kernel reading
# tiled records.
SPLITK_SPECS = [
    LayerSpec(300, 8 * 300 + 5, 8, (16,), (0.02,)),
    LayerSpec(300, 8 * 300 + 5, 8, (16, 8), (0.02, 0.005)),
    LayerSpec(300, 6 * 600 + 4, 6, (12, 4), (0.02, 0.005)),
    LayerSpec(129, 7 * 30 + 1, 7, (9,), (0.02,), None, None),
    LayerSpec(70, 16 * 20, 16, (16, 3), (0.02, 0.005)),
]


@pytest.mark.parametrize("i", range(len(SPLITK_SPECS)))
@pytest.mark.parametrize("batch", [1, 2, 5, 16])
def test_tiled_gemv_batches(i, batch):
    vq = _vq()
    spec = SPLITK_SPECS[i]
    data = synth.make_layer(spec, seed=2600 + i)
    layer = _oracle_tiled_layer(data)
    x = synth.make_x(2650 + i, batch, spec.in_features, outlier_frac=0.01)
    ref = oracle.linear(data, x)
    y = vq.gemv(layer, _x_dev(x), out_dtype=torch.float32)
    assert_close(_f64(y), ref, "float32")


def test_tiled_gemm_staged():
    vq = _vq()
    for i, spec in enumerate([LayerSpec(300, 8 * 130 + 8, 8, (16, 8), (0.02, 0.005)),
                              LayerSpec(257, 6 * 100 + 2, 6, (12, 4), (0.02, 0.005))]):
        data = synth.make_layer(spec, seed=2700 + i)
        layer = _oracle_tiled_layer(data)
        ld = -(-spec.in_features // 8) * 8           # vq_gemm wants ldx % 8 == 0
        x = synth.make_x(2750 + i, 200, spec.in_features, outlier_frac=0.01, ld=ld)
        ref = oracle.linear(data, x[:, :spec.in_features])
        y = vq.gemm(layer, _x_dev(x)[:, :spec.in_features], out_dtype=torch.float32)
        assert_close(_f64(y), ref, "float32")


def test_noalloc_on_a_tiled_layer_shrinks_the_grid():
    """28672 rows need about 17 MB of per-block sums on 148 blocks; the no-alloc
    entry point runs the same kernel on as many blocks as its 8 MB scratch holds."""
    vq = _vq()
    spec, seed = WORKLOADS["llama3_70b_mlp"].layers[0]
    data = synth.make_layer(spec, seed)
    layer = vq.repack_tile4(vq.Layer.from_synth(data))
    assert vq.gemv_workspace_size(layer, 1) > vq.NOALLOC_SCRATCH_BYTES
    x = synth.make_x(2800, 1, spec.in_features, outlier_frac=0.001)
    rows = sample_rows(spec.out_features, 256, 2801)
    ref = oracle.linear(data, x, rows)
    out = torch.empty((1, spec.out_features), dtype=torch.float32, device="cuda")
    vq.gemv_noalloc(layer, _x_dev(x), out=out)
    assert_close(_f64(out[:, torch.from_numpy(rows).cuda()]), ref, "float32")
    y = vq.gemv(layer, _x_dev(x), out_dtype=torch.float32)
    assert_close(_f64(y[:, torch.from_numpy(rows).cuda()]), ref, "float32")


@pytest.mark.parametrize("li", [0, 1, 2])
def test_70b_decode_layers_tiled(li):
    """The 2-bpw 70B MLP layers in the tiled order: dequant bit-exact on sampled
    rows; batch 1 (lookup table) and batch 4 (split-K gather kernel) on sampled rows."""
    vq = _vq()
    w = WORKLOADS["llama3_70b_mlp"]
    spec, seed = w.layers[li]
    data = synth.make_layer(spec, seed)
    layer = vq.repack_tile4(vq.Layer.from_synth(data))
    rows = sample_rows(spec.out_features, 192, seed + 2)
    rd = torch.from_numpy(rows).cuda()
    wh = vq.dequant(layer)
    assert np.array_equal(_w_bits(wh[rd]), oracle.dequant(data, rows))
    del wh
    x = synth.make_x(w.x_seed + li, 4, spec.in_features, w.outlier_frac)
    ref = oracle.linear(data, x, rows)
    for b in (1, 4):
        y = vq.gemv(layer, _x_dev(x)[:b], out_dtype=torch.bfloat16)
        assert_close(_f64(y[:, rd]), ref[:b], "bfloat16")


# Small-book lookup tables: d = 6 and 8, one and two books, books smaller than
# one 16-centroid tile, odd field widths, ragged N / nvec / Kin.
SMALL_LUT_SPECS = [
    LayerSpec(777, 6 * 130 + 4, 6, (12, 4), (0.02, 0.005)),
    LayerSpec(1000, 8 * 125, 8, (12, 8), (0.02, 0.005)),
    LayerSpec(513, 8 * 61 + 3, 8, (12,), (0.02,), None, None),
    LayerSpec(300, 6 * 77, 6, (9,), (0.02,), (0.5, 1.5), None),
    LayerSpec(9000, 6 * 20 + 5, 6, (3, 5), (0.02, 0.005)),
    LayerSpec(17000, 8 * 9, 8, (7, 11), (0.02, 0.005)),
    LayerSpec(65536, 6 * 5, 6, (12, 4), (0.02, 0.005)),
]


@pytest.mark.parametrize("i", range(len(SMALL_LUT_SPECS)))
def test_small_book_lut_gemv(i):
    vq = _vq()
    spec = SMALL_LUT_SPECS[i]
    data = synth.make_layer(spec, seed=2900 + i)
    layer = _oracle_tiled_layer(data)
    assert vq.gemv_workspace_size(layer, 1) > 0            # a lookup-table plan
    for fp16 in (False, True):
        x = synth.make_x(2950 + i, 1, spec.in_features, outlier_frac=0.01, as_fp16=fp16)
        ref = oracle.linear(data, x, x_is_fp16=fp16)
        for od in (torch.float32, torch.bfloat16):
            y = vq.gemv(layer, _x_dev(x, fp16), out_dtype=od)
            assert_close(_f64(y), ref, str(od).split(".")[-1])


@pytest.mark.parametrize("name,li", [("llama31_405b", 4), ("llama31_405b", 6), ("llama31_405b", 1),
                                     ("llama3_8b_up", 0)])
def test_small_book_decode_layers_tiled(name, li):
    vq = _vq()
    w = WORKLOADS[name]
    spec, seed = w.layers[li]
    data = synth.make_layer(spec, seed)
    layer = vq.repack_tile4(vq.Layer.from_synth(data))
    rows = sample_rows(spec.out_features, 192, seed + 3)
    x = synth.make_x(w.x_seed + li, 1, spec.in_features, w.outlier_frac)
    ref = oracle.linear(data, x, rows)
    y = vq.gemv(layer, _x_dev(x), out_dtype=torch.bfloat16)
    assert_close(_f64(y[:, torch.from_numpy(rows).cuda()]), ref, "bfloat16")


GARBAGE_SPECS = [
    LayerSpec(1001, 8 * 33 + 3, 8, (16,), (0.02,)),            # 2^16 table kernel
    LayerSpec(777, 6 * 31 + 4, 6, (12, 4), (0.02, 0.005)),     # paired small-book kernel
    LayerSpec(301, 7 * 13 + 2, 7, (9, 3), (0.02, 0.005)),      # split-K kernel
]


@pytest.mark.parametrize("i", range(len(GARBAGE_SPECS)))
def test_ignored_bits_are_ignored(i):
    """Random bits in every bit the tiled format ignores change nothing: dequant
    stays bit-exact and the products stay within the bar, at batch 1 and 3."""
    vq = _vq()
    spec = GARBAGE_SPECS[i]
    data = synth.make_layer(spec, seed=3000 + i)
    layer = _oracle_tiled_layer(data, extra_words=4, garbage=True)
    w = vq.dequant(layer)
    torch.cuda.synchronize()
    assert np.array_equal(_w_bits(w), oracle.dequant(data))
    for batch in (1, 3):
        x = synth.make_x(3050 + i, batch, spec.in_features, outlier_frac=0.01)
        y = vq.gemv(layer, _x_dev(x), out_dtype=torch.float32)
        assert_close(_f64(y), oracle.linear(data, x), "float32")


def test_table_batch_limit_override(monkeypatch):
    """VQ_LUT_MAX_BATCH moves a batch between the per-row table passes (a
    workspace of per-block row sums) and the split-K kernel (split partials);
    both give the same products within the bar."""
    vq = _vq()
    spec = LayerSpec(2000, 6 * 100 + 2, 6, (12, 4), (0.02, 0.005))
    data = synth.make_layer(spec, seed=3100)
    layer = _oracle_tiled_layer(data)
    x = synth.make_x(3101, 5, spec.in_features, outlier_frac=0.01)
    ref = oracle.linear(data, x)
    sizes = {}
    for limit in ("0", "16"):
        monkeypatch.setenv("VQ_LUT_MAX_BATCH", limit)
        sizes[limit] = vq.gemv_workspace_size(layer, 5)
        y = vq.gemv(layer, _x_dev(x), out_dtype=torch.float32)
        assert_close(_f64(y), ref, "float32")
    assert sizes["16"] % ((spec.out_features + 1) * 4) == 0
    assert sizes["0"] != sizes["16"]


def test_tiled_small_batch_strided_x_and_y():
    """The per-row table passes honour the row strides of x and y."""
    vq = _vq()
    for i, spec in enumerate([LayerSpec(700, 8 * 60, 8, (16,), (0.02,)),
                              LayerSpec(500, 6 * 70 + 2, 6, (12, 4), (0.02, 0.005))]):
        data = synth.make_layer(spec, seed=3200 + i)
        layer = _oracle_tiled_layer(data)
        x = synth.make_x(3210 + i, 2, spec.in_features, outlier_frac=0.01, ld=spec.in_features + 40)
        ref = oracle.linear(data, x[:, :spec.in_features])
        ybuf = torch.zeros((2, spec.out_features + 24), dtype=torch.float32, device="cuda")
        vq.gemv(layer, _x_dev(x)[:, :spec.in_features], out=ybuf[:, :spec.out_features])
        assert_close(_f64(ybuf[:, :spec.out_features]), ref, "float32")
        assert (ybuf[:, spec.out_features:] == 0).all()


# Layers that share x through vq_gemv_multi: tiled 2^16-book layers at batch
# 1 run as one table launch (rows of all layers in one task list); any other
# mix runs the layers one after another.
MULTI_SETS = [
    [LayerSpec(3000, 8 * 100 + 3, 8, (16,), (0.02,)), LayerSpec(777, 8 * 100 + 3, 8, (16,), (0.02,))],
    [LayerSpec(8193, 8 * 40, 8, (16,), (0.02,), None, None), LayerSpec(300, 8 * 40, 8, (16,), (0.02,)),
     LayerSpec(20000, 8 * 40, 8, (16,), (0.02,), (0.5, 1.5), None)],
    [LayerSpec(5000, 8 * 33, 8, (16,), (0.02,)) for _ in range(4)],
    # not fusable: a small-book layer in the set
    [LayerSpec(3000, 8 * 64, 8, (16,), (0.02,)), LayerSpec(900, 8 * 64, 8, (12, 8), (0.02, 0.005))],
    # paired-row small-book layers: q/k/v-like (d = 6, 2^12 + 2^4) and gate/up-like (d = 8, 2^12 + 2^8)
    [LayerSpec(9000, 6 * 50 + 4, 6, (12, 4), (0.02, 0.005)), LayerSpec(1024, 6 * 50 + 4, 6, (12, 4), (0.02, 0.005)),
     LayerSpec(1023, 6 * 50 + 4, 6, (12, 4), (0.02, 0.005))],
    [LayerSpec(14336, 8 * 40, 8, (12, 8), (0.02, 0.005)), LayerSpec(14335, 8 * 40, 8, (12, 8), (0.02, 0.005))],
    [LayerSpec(700, 6 * 30, 6, (12, 4), (0.02, 0.005)) for _ in range(4)],
]


@pytest.mark.parametrize("i", range(len(MULTI_SETS)))
@pytest.mark.parametrize("batch", [1, 3])
def test_gemv_multi_matches_the_oracle(i, batch):
    vq = _vq()
    specs = MULTI_SETS[i]
    datas = [synth.make_layer(s, seed=2900 + 10 * i + k) for k, s in enumerate(specs)]
    layers = [_oracle_tiled_layer(d) for d in datas]
    assert vq.gemv_multi_workspace_size(layers, batch) > 0
    for fp16 in (False, True):
        x = synth.make_x(2950 + i, batch, specs[0].in_features, outlier_frac=0.01, as_fp16=fp16)
        for od in (torch.float32, torch.bfloat16):
            ys = vq.gemv_multi(layers, _x_dev(x, fp16), out_dtype=od)
            for y, d in zip(ys, datas):
                assert_close(_f64(y), oracle.linear(d, x, x_is_fp16=fp16), str(od).split(".")[-1])


def test_gemv_multi_70b_gate_up_sampled():
    """The 70B gate/up pair (2 x 28672 rows = all eight row-sum batches) as one launch."""
    vq = _vq()
    w = WORKLOADS["llama3_70b_mlp"]
    datas, layers = [], []
    for li in (0, 1):
        spec, seed = w.layers[li]
        datas.append(synth.make_layer(spec, seed))
        layers.append(vq.repack_tile4(vq.Layer.from_synth(datas[-1])))
    x = synth.make_x(w.x_seed, 1, layers[0].in_features, w.outlier_frac)
    rows = sample_rows(layers[0].out_features, 192, 2990)
    rd = torch.from_numpy(rows).cuda()
    ys = vq.gemv_multi(layers, _x_dev(x), out_dtype=torch.bfloat16)
    for y, d in zip(ys, datas):
        assert_close(_f64(y[:, rd]), oracle.linear(d, x, rows), "bfloat16")


def test_gemv_multi_405b_qkv_sampled():
    """The 405B q/k/v projections (16384 + 1024 + 1024 rows, d = 6) as one launch."""
    vq = _vq()
    w = WORKLOADS["llama31_405b"]
    datas, layers = [], []
    for li in (0, 1, 2):
        spec, seed = w.layers[li]
        datas.append(synth.make_layer(spec, seed))
        layers.append(vq.repack_tile4(vq.Layer.from_synth(datas[-1])))
    x = synth.make_x(w.x_seed, 1, layers[0].in_features, w.outlier_frac)
    ys = vq.gemv_multi(layers, _x_dev(x), out_dtype=torch.bfloat16)
    for k, (y, d) in enumerate(zip(ys, datas)):
        rows = sample_rows(layers[k].out_features, 128, 2995 + k)
        rd = torch.from_numpy(rows).cuda()
        assert_close(_f64(y[:, rd]), oracle.linear(d, x, rows), "bfloat16")

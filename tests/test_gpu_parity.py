"""GPU parity: vq_dequant bit-exact and vq_gemv within the normwise bar,
against the CPU oracle on the same seeded inputs, through the C ABI.

Small cases run in full (several tiles, ragged tails); the full-size layers
of the named workloads are compared on sampled output rows, which the
oracle computes one by one."""
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


def _dev_layer(data):
    return _vq().Layer.from_synth(data)


def _x_dev(x_bits: np.ndarray, fp16: bool = False) -> torch.Tensor:
    t = torch.from_numpy(x_bits.view(np.int16)).cuda()
    return t.view(torch.float16 if fp16 else torch.bfloat16)


def _w_bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


# -- vq_dequant: bit-exact ----------------------------------------------------

SMALL_SPECS = (
    [LayerSpec(37, 8 * 45 + 3, 8, (b,), (0.02,)) for b in range(1, 17)]
    + [LayerSpec(29, 5 * d + d // 2 + 1, d, (5, 3), (0.02, 0.005)) for d in range(1, 17)]
    + [
        LayerSpec(300, 1000, 8, (12, 8), (0.02, 0.005)),
        LayerSpec(130, 6 * 200 + 4, 6, (12, 4), (0.02, 0.005)),
        LayerSpec(130, 6 * 200 + 1, 6, (16,), (0.02,)),
        LayerSpec(257, 2056, 8, (16, 16), (0.02, 0.005)),
        LayerSpec(64, 512, 8, (16,), (0.02,), None, None),
        LayerSpec(64, 512, 8, (12, 8), (0.02, 0.005), (0.5, 1.5), None),
        LayerSpec(64, 510, 6, (12, 4), (0.02, 0.005), None, 1e-3),
        LayerSpec(1, 1, 1, (1,), (0.02,)),
        LayerSpec(3, 17, 16, (16, 2), (0.02, 0.005)),
    ])


@pytest.mark.parametrize("i", range(len(SMALL_SPECS)))
def test_dequant_bit_exact_small(i):
    spec = SMALL_SPECS[i]
    data = synth.make_layer(spec, seed=500 + i, pad_garbage=(i % 2 == 1))
    w = _vq().dequant(_dev_layer(data))
    torch.cuda.synchronize()
    assert np.array_equal(_w_bits(w), oracle.dequant(data))


def test_dequant_overpadded_rows_and_strided_output():
    spec = LayerSpec(100, 777, 8, (12, 8), (0.02, 0.005))
    data = synth.make_layer(spec, seed=77, row_words=[300, 200], pad_garbage=True)
    layer = _dev_layer(data)
    buf = torch.full((100, 800), -1, dtype=torch.int16, device="cuda")
    out = buf.view(torch.float16)[:, :777]
    _vq().dequant(layer, out=out)
    got = buf.cpu().numpy().view(np.uint16)
    assert np.array_equal(got[:, :777], oracle.dequant(data))
    assert (got[:, 777:] == 0xFFFF).all()          # columns past Kin untouched


def _workload_layers(name):
    w = WORKLOADS[name]
    return [(spec, seed) for spec, seed in w.layers]


FULL_SIZE = [(name, i) for name in WORKLOADS for i in range(len(WORKLOADS[name].layers))]


@pytest.mark.parametrize("name,li", FULL_SIZE)
def test_dequant_bit_exact_workloads(name, li):
    spec, seed = WORKLOADS[name].layers[li]
    data = synth.make_layer(spec, seed)
    layer = _dev_layer(data)
    w = _vq().dequant(layer)
    rows = sample_rows(spec.out_features, 192, seed)
    got = _w_bits(w[torch.from_numpy(rows).cuda()])
    assert np.array_equal(got, oracle.dequant(data, rows))


# -- vq_gemv -----------------------------------------------------------------

@pytest.mark.parametrize("i", range(len(SMALL_SPECS)))
@pytest.mark.parametrize("batch", [1, 3, 16])
def test_gemv_small(i, batch):
    spec = SMALL_SPECS[i]
    data = synth.make_layer(spec, seed=900 + i)
    x = synth.make_x(40 + i, batch, spec.in_features, outlier_frac=0.01)
    ref = oracle.linear(data, x)
    y = _vq().gemv(_dev_layer(data), _x_dev(x), out_dtype=torch.float32)
    assert_close(_f64(y), ref, "float32")


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float16, torch.float32])
def test_gemv_output_types_and_fp16_input(out_dtype):
    spec = LayerSpec(500, 3000, 8, (12, 8), (0.02, 0.005))
    data = synth.make_layer(spec, seed=31)
    layer = _dev_layer(data)
    for fp16 in (False, True):
        x = synth.make_x(32, 5, 3000, as_fp16=fp16)
        ref = oracle.linear(data, x, x_is_fp16=fp16)
        y = _vq().gemv(layer, _x_dev(x, fp16), out_dtype=out_dtype)
        assert_close(_f64(y), ref, str(out_dtype).split(".")[-1])
    # the bf16 output is the fp32 result rounded once (oracle rounding)
    x = synth.make_x(33, 2, 3000)
    y32 = _vq().gemv(layer, _x_dev(x), out_dtype=torch.float32).cpu().numpy()
    yb = _vq().gemv(layer, _x_dev(x), out_dtype=torch.bfloat16)
    assert np.array_equal(yb.view(torch.int16).cpu().numpy().view(np.uint16), oracle.f32_to_bf16(y32))


# Specialised kernels: every supported (d, index widths) pair, ragged
# rows and columns, partial 256-vector chunks, and narrow layers that take the
# split along the input dimension.
FAST_SPECS = [
    LayerSpec(300, 8 * 300 + 5, 8, (16,), (0.02,)),
    LayerSpec(300, 8 * 300 + 5, 8, (16, 8), (0.02, 0.005)),
    LayerSpec(300, 8 * 300 + 5, 8, (12, 8), (0.02, 0.005)),
    LayerSpec(300, 8 * 300 + 5, 8, (8, 8), (0.02, 0.005)),
    LayerSpec(257, 8 * 700, 8, (8,), (0.02,), None, None),
    LayerSpec(300, 6 * 600 + 4, 6, (12, 4), (0.02, 0.005)),
    LayerSpec(129, 6 * 300 + 1, 6, (12,), (0.02,)),
    LayerSpec(64, 8 * 4000, 8, (16,), (0.02,)),
    LayerSpec(40, 6 * 3000 + 2, 6, (12, 4), (0.02, 0.005)),
    LayerSpec(1, 8, 8, (16,), (0.02,)),
]


@pytest.mark.parametrize("i", range(len(FAST_SPECS)))
@pytest.mark.parametrize("batch", [1, 2, 3, 5, 16])
def test_gemv_specialised_kernels(i, batch):
    """Single-row (batch 1) and batched (2..16) kernels."""
    spec = FAST_SPECS[i]
    data = synth.make_layer(spec, seed=1300 + i, pad_garbage=True)
    layer = _dev_layer(data)
    for fp16 in (False, True):
        x = synth.make_x(90 + i, batch, spec.in_features, outlier_frac=0.01, as_fp16=fp16)
        ref = oracle.linear(data, x, x_is_fp16=fp16)
        y = _vq().gemv(layer, _x_dev(x, fp16), out_dtype=torch.float32)
        assert_close(_f64(y), ref, "float32")


def test_gemv_strided_x_and_y():
    spec = LayerSpec(70, 600, 6, (12, 4), (0.02, 0.005))
    data = synth.make_layer(spec, seed=34)
    x = synth.make_x(35, 4, 600, ld=640)
    ref = oracle.linear(data, x[:, :600])
    ybuf = torch.zeros((4, 96), dtype=torch.float32, device="cuda")
    _vq().gemv(_dev_layer(data), _x_dev(x)[:, :600], out=ybuf[:, :70])
    assert_close(_f64(ybuf[:, :70]), ref, "float32")
    assert (ybuf[:, 70:] == 0).all()


def _decode_cases():
    for name in ("tiny_512", "llama3_8b_up", "llama3_70b_mlp", "llama31_405b"):
        w = WORKLOADS[name]
        batches = w.batches if name != "llama31_405b" else (1, 4, 16)
        for li in range(len(w.layers)):
            yield name, li, batches


@pytest.mark.parametrize("name,li,batches", list(_decode_cases()))
def test_gemv_workloads(name, li, batches):
    w = WORKLOADS[name]
    spec, seed = w.layers[li]
    data = synth.make_layer(spec, seed)
    layer = _dev_layer(data)
    bmax = max(batches)
    x = synth.make_x(w.x_seed + li, bmax, spec.in_features, w.outlier_frac)
    rows = sample_rows(spec.out_features, 256, seed + 1)
    ref = oracle.linear(data, x, rows)
    xd = _x_dev(x)
    for b in batches:
        for od in (torch.float32, torch.bfloat16):
            y = _vq().gemv(layer, xd[:b], out_dtype=od)
            got = _f64(y[:, torch.from_numpy(rows).cuda()])
            assert_close(got, ref[:b], str(od).split(".")[-1])


def test_gemv_every_batch_on_kv_shape():
    spec, seed = WORKLOADS["llama31_405b"].layers[1]       # k_proj 1024 x 16384
    data = synth.make_layer(spec, seed)
    layer = _dev_layer(data)
    x = synth.make_x(77, 16, spec.in_features)
    ref = oracle.linear(data, x)
    xd = _x_dev(x)
    for b in range(1, 17):
        y = _vq().gemv(layer, xd[:b], out_dtype=torch.float32)
        assert_close(_f64(y), ref[:b], "float32")


# -- degenerate cases and argument errors -----------------------------------

def test_gemv_empty_and_degenerate():
    vq = _vq()
    spec = LayerSpec(8, 16, 8, (4,), (0.02,))
    data = synth.make_layer(spec, seed=3)
    layer = _dev_layer(data)
    x = _x_dev(synth.make_x(1, 16, 16))
    y = vq.gemv(layer, x[:0], out_dtype=torch.float32)           # batch 0
    assert y.shape == (0, 8)
    # in_features = 0: y = 0 for every row
    spec0 = LayerSpec(5, 0, 8, (4,), (0.02,))
    d0 = synth.make_layer(spec0, seed=4)
    l0 = _dev_layer(d0)
    y0 = torch.full((2, 5), 7.0, device="cuda")
    vq.gemv(l0, torch.zeros((2, 8), dtype=torch.bfloat16, device="cuda"), out=y0)
    assert (y0 == 0).all()


def test_argument_errors():
    vq = _vq()
    spec = LayerSpec(64, 256, 8, (8,), (0.02,))
    data = synth.make_layer(spec, seed=5)
    layer = _dev_layer(data)
    x = _x_dev(synth.make_x(2, 17, 256))
    with pytest.raises(vq.VQError) as e:
        vq.gemv(layer, x)                                      # batch 17
    assert e.value.status == vq.VQ_ERR_UNSUPPORTED
    bad = vq.Layer(64, 256, 8, [8], [layer.idx[0][:, :4].contiguous()], layer.codebooks)  # short rows
    with pytest.raises(vq.VQError) as e:
        vq.dequant(bad)
    assert e.value.status == vq.VQ_ERR_INVALID_ARG
    shifted = torch.empty(2049, dtype=torch.float16, device="cuda")
    shifted[1:] = layer.codebooks[0].reshape(-1)
    mis = vq.Layer(64, 256, 8, [8], layer.idx, [shifted[1:].view(256, 8)])      # 2-byte offset
    with pytest.raises(vq.VQError) as e:
        vq.dequant(mis)
    assert e.value.status == vq.VQ_ERR_ALIGNMENT
    big = synth.make_layer(LayerSpec(4096, 2048, 8, (8,), (0.02,)), seed=6)
    bl = _dev_layer(big)
    need = vq.gemv_workspace_size(bl, 16)
    if need:
        with pytest.raises(vq.VQError) as e:
            vq.gemv(bl, _x_dev(synth.make_x(3, 16, 2048)),
                    workspace=torch.empty(need // 2, dtype=torch.uint8, device="cuda"))
        assert e.value.status == vq.VQ_ERR_WORKSPACE

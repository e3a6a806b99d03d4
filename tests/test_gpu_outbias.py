"""GPU parity of the optional output bias (vq_layer_desc.out_bias, ABI 4):
y = x . W_hat^T + b_out, against the oracle's fp64 sum plus b_out, through
every epilogue that writes y.

Each case runs with and without the bias, on the same layer and x:
  vq_gemv    row order: batch 1 (single-row kernel) and 5 (batched kernel)
             on small books; 2^16 book at batch 1 (single-row) and 2..16
             (tensor-core kernel); d = 4 (split-K gather kernel); narrow and
             wide layers, so K splits with a summing pass occur;
             tiled order: 2^16 book at batch 1 and 2 (table kernel, one pass
             per row of x), 3 and 16 (tensor-core kernel); 2^12 books at
             batch 1 and 4 (small-book table kernels); 2^12 book at batch 12
             (split-K gather kernel on the tiled order);
  vq_gemv_multi  fused table launches (2^16 set, 2^12 + 2^8 set) and the
             unfused row-order fallback;
  vq_gemm    fused and staged forms, bf16 and fp16 x, a ragged tile;
  vq_gemv_rht  the bias lands on y, after the inverse transform;
  Kin = 0    y is b_out exactly (gemv and gemm).
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import synth
from synth import LayerSpec
from tests._util import assert_close

pytestmark = pytest.mark.gpu

_TORCH = {"bfloat16": torch.bfloat16, "float16": torch.float16, "float32": torch.float32}


def _vq():
    from bit_packed_index_b200 import vq
    return vq


def _x_dev(x_bits: np.ndarray, fp16: bool = False) -> torch.Tensor:
    t = torch.from_numpy(x_bits.view(np.int16)).cuda()
    return t.view(torch.float16 if fp16 else torch.bfloat16)


def _f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def _with_out_bias(spec: LayerSpec, std: float = 0.25) -> LayerSpec:
    return dataclasses.replace(spec, out_bias_std=std)


def _pair(spec: LayerSpec, seed: int, layout: str):
    """The layer drawn with an output bias, as device layers with and without it."""
    vq = _vq()
    data = synth.make_layer(_with_out_bias(spec), seed)
    assert data.out_bias is not None
    with_b = vq.Layer.from_synth(data, layout=layout)
    without = dataclasses.replace(with_b, out_bias=None, _desc=None)
    return data, with_b, without


GEMV_CASES = [
    # (spec, layout, batch)
    (LayerSpec(700, 8 * 130 + 3, 8, (12, 8), (0.02, 0.005)), "rows", 1),
    (LayerSpec(700, 8 * 130 + 3, 8, (12, 8), (0.02, 0.005)), "rows", 5),
    (LayerSpec(96, 6 * 3000 + 2, 6, (12, 4), (0.02, 0.005)), "rows", 2),      # K splits
    (LayerSpec(513, 8 * 200, 8, (16,), (0.02,)), "rows", 1),
    (LayerSpec(64, 8 * 4000, 8, (16,), (0.02,)), "rows", 1),                 # K splits
    (LayerSpec(513, 8 * 200, 8, (16,), (0.02,)), "rows", 2),
    (LayerSpec(300, 8 * 3000, 8, (16,), (0.02,)), "rows", 16),               # TC, K splits
    (LayerSpec(200, 4 * 150 + 1, 4, (8, 4), (0.02, 0.005)), "rows", 3),       # split-K gather
    (LayerSpec(1000, 8 * 260, 8, (16,), (0.02,)), "tile4", 1),
    (LayerSpec(1000, 8 * 260, 8, (16,), (0.02,)), "tile4", 2),
    (LayerSpec(1000, 8 * 260, 8, (16,), (0.02,)), "tile4", 3),
    (LayerSpec(1000, 8 * 260 + 5, 8, (16,), (0.02,)), "tile4", 16),
    (LayerSpec(900, 6 * 400 + 4, 6, (12, 4), (0.02, 0.005)), "tile4", 1),
    (LayerSpec(900, 8 * 300, 8, (12, 8), (0.02, 0.005)), "tile4", 4),
    (LayerSpec(900, 8 * 300, 8, (12,), (0.02,)), "tile4", 12),
]


@pytest.mark.parametrize("i", range(len(GEMV_CASES)))
def test_gemv_output_bias(i):
    vq = _vq()
    spec, layout, batch = GEMV_CASES[i]
    data, with_b, without = _pair(spec, 500 + i, layout)
    x = synth.make_x(600 + i, batch, spec.in_features)
    ref_b = oracle.linear(data, x)
    ref_0 = oracle.linear(data, x, out_bias=np.zeros(spec.out_features, np.uint16))
    for od in ("float32", "bfloat16"):
        y_b = _f64(vq.gemv(with_b, _x_dev(x), out_dtype=_TORCH[od]))
        y_0 = _f64(vq.gemv(without, _x_dev(x), out_dtype=_TORCH[od]))
        assert_close(y_b, ref_b, od)
        assert_close(y_0, ref_0, od)
    # fp32 outputs: the bias is the whole difference between the two calls
    y_b = _f64(vq.gemv(with_b, _x_dev(x), out_dtype=torch.float32))
    y_0 = _f64(vq.gemv(without, _x_dev(x), out_dtype=torch.float32))
    bf = data.out_bias.view(np.float16).astype(np.float64)
    assert np.allclose(y_b - y_0, np.tile(bf, (batch, 1)), rtol=0,
                       atol=1e-5 * (np.abs(ref_0).max() + np.abs(bf).max()))


MULTI_SETS = [
    # (specs, layout): fused 2^16 set, fused 2^12 + 2^8 set, row-order fallback
    ([LayerSpec(1024, 8 * 256, 8, (16,), (0.02,)), LayerSpec(2048, 8 * 256, 8, (16,), (0.02,))], "tile4"),
    ([LayerSpec(1024, 8 * 256, 8, (12, 8), (0.02, 0.005)),
      LayerSpec(1024, 8 * 256, 8, (12, 8), (0.02, 0.005))], "tile4"),
    ([LayerSpec(333, 8 * 100 + 1, 8, (12, 8), (0.02, 0.005)), LayerSpec(77, 8 * 100 + 1, 8, (16,), (0.02,))],
     "rows"),
]


@pytest.mark.parametrize("i", range(len(MULTI_SETS)))
def test_gemv_multi_output_bias(i):
    vq = _vq()
    specs, layout = MULTI_SETS[i]
    pairs = [_pair(s, 700 + 10 * i + j, layout) for j, s in enumerate(specs)]
    # one layer of the set carries no output bias
    layers = [p[1] for p in pairs[:-1]] + [pairs[-1][2]]
    x = synth.make_x(800 + i, 1, specs[0].in_features)
    ys = vq.gemv_multi(layers, _x_dev(x), out_dtype=torch.float32)
    for j, ((data, _, _), y) in enumerate(zip(pairs, ys)):
        ob = None if j == len(pairs) - 1 else data.out_bias
        zero = np.zeros(data.spec.out_features, np.uint16)
        ref = oracle.linear(data, x, out_bias=zero if ob is None else ob)
        assert_close(_f64(y), ref, "float32")


GEMM_CASES = [
    # (spec, layout, m, fp16 x)
    (LayerSpec(300, 8 * 64 + 3, 8, (12, 8), (0.02, 0.005)), "rows", 200, False),
    (LayerSpec(300, 6 * 90, 6, (12, 4), (0.02, 0.005)), "rows", 130, True),
    (LayerSpec(520, 8 * 96, 8, (16,), (0.02,)), "tile4", 257, False),
    (LayerSpec(520, 8 * 96, 8, (16, 8), (0.02, 0.005)), "rows", 700, True),
]


@pytest.mark.parametrize("i", range(len(GEMM_CASES)))
def test_gemm_output_bias(i):
    vq = _vq()
    spec, layout, m, fp16 = GEMM_CASES[i]
    data, with_b, without = _pair(spec, 900 + i, layout)
    x = synth.make_x(950 + i, m, spec.in_features, as_fp16=fp16, ld=-(-spec.in_features // 8) * 8)
    rows = np.unique(np.linspace(0, m - 1, 24).astype(int))
    ref_b = oracle.linear(data, x[rows], x_is_fp16=fp16)
    ref_0 = oracle.linear(data, x[rows], x_is_fp16=fp16, out_bias=np.zeros(spec.out_features, np.uint16))
    for od in ("float32", "float16"):
        y_b = _f64(vq.gemm(with_b, _x_dev(x, fp16), out_dtype=_TORCH[od]))[rows]
        y_0 = _f64(vq.gemm(without, _x_dev(x, fp16), out_dtype=_TORCH[od]))[rows]
        assert_close(y_b, ref_b, od)
        assert_close(y_0, ref_0, od)


def _signs(n, seed):
    rng = np.random.default_rng(seed)
    bits = rng.integers(0, 2, size=n).astype(np.uint8)
    words = np.packbits(np.concatenate([bits, np.zeros((-n) % 32, np.uint8)]), bitorder="little")
    words = words.view(np.uint32)
    return words, torch.from_numpy(words.view(np.int32).copy()).cuda()


@pytest.mark.parametrize("layout", ["rows", "tile4"])
@pytest.mark.parametrize("batch", [1, 3])
def test_gemv_rht_output_bias_lands_on_y(layout, batch):
    """y = U^T (W~ (V x)) + b_out: the bias is not rotated (batch 1 in the
    tiled order builds x~ inside the table kernel)."""
    vq = _vq()
    spec = LayerSpec(1024, 8 * 128, 8, (16,), (0.02,))
    data, with_b, _ = _pair(spec, 990, layout)
    s_in, d_in = _signs(spec.in_features, 991)
    s_out, d_out = _signs(spec.out_features, 992)
    x = synth.make_x(993, batch, spec.in_features)
    w = oracle.f16_to_f32(oracle.dequant(data)).astype(np.float64)
    xt = oracle.rht(oracle.bf16_to_f32(x).astype(np.float64), s_in)
    ref = oracle.rht(xt @ w.T, s_out, inverse=True)
    ref = ref + data.out_bias.view(np.float16).astype(np.float64)[None, :]
    y = vq.gemv_rht(with_b, d_in, d_out, _x_dev(x), out_dtype=torch.float32)
    assert_close(_f64(y), ref, "float32")


def test_empty_input_rows_give_the_output_bias():
    """Kin = 0: every row of y is b_out exactly (gemv and gemm), and zeros
    without it."""
    vq = _vq()
    n = 37
    b_out = synth.to_f16_bits(np.linspace(-3, 3, n).astype(np.float32))
    books = [torch.zeros((256, 8), dtype=torch.float16, device="cuda")]
    idx = [torch.zeros((n, 4), dtype=torch.int32, device="cuda")]
    ob = torch.from_numpy(b_out.view(np.int16)).cuda().view(torch.float16)
    layer = vq.Layer(n, 0, 8, [8], idx, books, out_bias=ob)
    plain = vq.Layer(n, 0, 8, [8], idx, books)
    x = torch.zeros((4, 8), dtype=torch.bfloat16, device="cuda")
    want = np.tile(b_out.view(np.float16).astype(np.float64), (4, 1))
    for od in (torch.float32, torch.float16, torch.bfloat16):
        y = vq.gemv(layer, x, out_dtype=od)
        got = _f64(y)
        exp = want if od != torch.bfloat16 else _f64(torch.from_numpy(want).to(torch.bfloat16))
        assert np.array_equal(got, exp)
        assert np.array_equal(_f64(vq.gemm(layer, x, out_dtype=od)), exp)
        assert not _f64(vq.gemv(plain, x, out_dtype=od)).any()

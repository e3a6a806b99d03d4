"""GPU parity of the tensor-core batched decode (vq_gemv, batch >= 2, layers
with one 2^16-entry d = 8 book, row or tiled index order) against the fp64
oracle, through the C ABI.

Covered: N below, on and past the 128-row tile of a CTA; nvec below, on and
past the 8-vector step, with a partial last vector; every batch 2..16; both
index orders; bf16 and fp16 x; every output type; scale and bias present and
absent; tiny and huge activation magnitudes (the per-row power-of-two scaling
into fp16); layers narrow enough to split the input dimension across CTAs;
strided x and y; stale workspace contents; the 70B decode layers on sampled
rows at B = 4, 8 and 16; and a bounded wait that runs out."""
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


def _f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def _layer(data, layout):
    vq = _vq()
    layer = vq.Layer.from_synth(data)
    return vq.repack_tile4(layer) if layout == "tile4" else layer


def _status(ws: torch.Tensor) -> int:
    torch.cuda.synchronize()
    return int(ws[:4].cpu().numpy().view(np.int32)[0])


TC_SPECS = [
    LayerSpec(1, 8, 8, (16,), (0.02,)),
    LayerSpec(127, 8 * 8, 8, (16,), (0.02,)),
    LayerSpec(128, 8 * 9 + 3, 8, (16,), (0.02,)),
    LayerSpec(129, 8 * 64, 8, (16,), (0.02,), None, None),
    LayerSpec(1000, 1001, 8, (16,), (0.02,)),
    LayerSpec(3000, 8 * 300 + 5, 8, (16,), (0.02,), (0.5, 1.5), None),
    LayerSpec(300, 8 * 3000, 8, (16,), (0.02,), None, 1e-3),
]


@pytest.mark.parametrize("i", range(len(TC_SPECS)))
@pytest.mark.parametrize("layout", ["rows", "tile4"])
def test_tc_gemv(i, layout):
    vq = _vq()
    spec = TC_SPECS[i]
    data = synth.make_layer(spec, seed=5100 + i)
    layer = _layer(data, layout)
    for batch in (3, 16):
        nws = vq.gemv_workspace_size(layer, batch)
        ws = torch.full((nws,), 0x55, dtype=torch.uint8, device="cuda")     # stale contents are fine
        for fp16 in (False, True):
            x = synth.make_x(5150 + i, batch, spec.in_features, outlier_frac=0.01, as_fp16=fp16)
            ref = oracle.linear(data, x, x_is_fp16=fp16)
            for od in (torch.float32, torch.bfloat16, torch.float16):
                y = vq.gemv(layer, _x_dev(x, fp16), out_dtype=od, workspace=ws)
                assert_close(_f64(y), ref, str(od).split(".")[-1])
                assert _status(ws) == vq.VQ_OK


@pytest.mark.parametrize("batch", range(2, 17))
def test_tc_gemv_every_batch(batch):
    vq = _vq()
    spec = LayerSpec(700, 8 * 200 + 3, 8, (16,), (0.02,))
    data = synth.make_layer(spec, seed=5200)
    x = synth.make_x(5201, batch, spec.in_features, outlier_frac=0.01)
    ref = oracle.linear(data, x)
    for layout in ("rows", "tile4"):
        y = vq.gemv(_layer(data, layout), _x_dev(x), out_dtype=torch.float32)
        assert_close(_f64(y), ref, "float32")


@pytest.mark.parametrize("mag", [1e-30, 1e-3, 1.0, 1e3, 1e30])
def test_tc_gemv_activation_magnitudes(mag):
    """Each row of x is scaled by its own power of two into fp16: tiny and
    huge rows in one batch stay within the bar (checked row by row)."""
    vq = _vq()
    spec = LayerSpec(1500, 8 * 150, 8, (16,), (0.02,))
    data = synth.make_layer(spec, seed=5300)
    layer = _layer(data, "rows")
    x = oracle.bf16_to_f32(synth.make_x(5301, 4, spec.in_features, outlier_frac=0.01))
    x[1] *= np.float32(mag)                       # rows of very different size
    x[3] *= np.float32(1.0 / mag) if mag > 1e-20 else np.float32(1.0)
    xb = oracle.f32_to_bf16(x)
    ref = oracle.linear(data, xb)
    y = _f64(vq.gemv(layer, _x_dev(xb), out_dtype=torch.float32))
    for b in range(4):
        assert_close(y[b:b + 1], ref[b:b + 1], "float32")


def test_tc_gemv_strided_x_and_y():
    vq = _vq()
    spec = LayerSpec(600, 8 * 100, 8, (16,), (0.02,))
    data = synth.make_layer(spec, seed=5400)
    layer = _layer(data, "tile4")
    x = synth.make_x(5401, 5, spec.in_features, outlier_frac=0.01, ld=spec.in_features + 40)
    ref = oracle.linear(data, x[:, :spec.in_features])
    ybuf = torch.zeros((5, spec.out_features + 24), dtype=torch.float32, device="cuda")
    vq.gemv(layer, _x_dev(x)[:, :spec.in_features], out=ybuf[:, :spec.out_features])
    assert_close(_f64(ybuf[:, :spec.out_features]), ref, "float32")
    assert (ybuf[:, spec.out_features:] == 0).all()


@pytest.mark.parametrize("li", [0, 2])
@pytest.mark.parametrize("layout", ["rows", "tile4"])
def test_tc_gemv_70b_layers(li, layout):
    """The 2-bpw 70B gate_proj (28672 x 8192: 224 row tiles) and down_proj
    (8192 x 28672: the input dimension split across CTAs) at B = 4, 8, 16."""
    vq = _vq()
    w = WORKLOADS["llama3_70b_mlp"]
    spec, seed = w.layers[li]
    data = synth.make_layer(spec, seed)
    layer = _layer(data, layout)
    rows = sample_rows(spec.out_features, 192, seed + 7)
    rd = torch.from_numpy(rows).cuda()
    x = synth.make_x(w.x_seed + li, 16, spec.in_features, w.outlier_frac)
    ref = oracle.linear(data, x, rows)
    for b in (4, 8, 16):
        y = vq.gemv(layer, _x_dev(x)[:b], out_dtype=torch.bfloat16)
        assert_close(_f64(y[:, rd]), ref[:b], "bfloat16")


def test_tc_bounded_wait_gives_up_with_timeout_status(monkeypatch):
    """With a wait budget of 0 clocks, the first wait that finds its stage
    not yet complete gives up: the kernel records VQ_ERR_TIMEOUT in the
    workspace's status word, drains its copies and returns.  The next call
    with the normal budget is correct."""
    vq = _vq()
    spec = LayerSpec(2000, 8 * 2000, 8, (16,), (0.02,))
    data = synth.make_layer(spec, seed=5500)
    layer = _layer(data, "rows")
    x = synth.make_x(5501, 8, spec.in_features, outlier_frac=0.01)
    ws = torch.zeros(vq.gemv_workspace_size(layer, 8), dtype=torch.uint8, device="cuda")
    monkeypatch.setenv("VQ_WAIT_BUDGET", "0")
    vq.gemv(layer, _x_dev(x), out_dtype=torch.float32, workspace=ws)
    assert _status(ws) == vq.VQ_ERR_TIMEOUT
    monkeypatch.delenv("VQ_WAIT_BUDGET")
    y = vq.gemv(layer, _x_dev(x), out_dtype=torch.float32, workspace=ws)
    assert _status(ws) == vq.VQ_OK
    assert_close(_f64(y), oracle.linear(data, x), "float32")

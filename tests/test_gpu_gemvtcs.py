"""GPU parity of the tensor-core batched decode for layers whose books fit
shared memory (vq_gemv, batch 3..16: a main book of up to 2^12 entries, an
optional residual, d = 6 or 8, row or tiled index order) against the fp64
oracle, through the C ABI.

The table kernels are limited to batch 1 here (VQ_LUT_MAX_BATCH), so the
tiled order reaches this kernel too.  Covered: N below, on and past the
128-row tile; nvec below, on and past the 8-vector step with a partial last
vector (d = 6: vectors padded to 8 columns); field widths whose records
straddle 32-bit words (10 + 3 bits); one book and two; the largest staged
pair (2^12 + 2^12); scale and bias present and absent; bf16 and fp16 x;
every output type; every batch 2..16; narrow layers split along the input
dimension; the 8B up and 405B gate layers on sampled rows; a bounded wait
that runs out."""
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


@pytest.fixture(autouse=True)
def _tables_at_batch_one_only(monkeypatch):
    monkeypatch.setenv("VQ_LUT_MAX_BATCH", "1")


SPECS = [
    LayerSpec(1, 8, 8, (12, 8), (0.02, 0.005)),
    LayerSpec(127, 8 * 8, 8, (12, 8), (0.02, 0.005)),
    LayerSpec(128, 6 * 9 + 4, 6, (12, 4), (0.02, 0.005)),
    LayerSpec(129, 8 * 64, 8, (12,), (0.02,), None, None),
    LayerSpec(1000, 6 * 170 + 2, 6, (12, 4), (0.02, 0.005)),
    LayerSpec(300, 8 * 3000, 8, (12, 8), (0.02, 0.005), (0.5, 1.5), None),
    LayerSpec(260, 8 * 64 + 7, 8, (8, 8), (0.02, 0.005), None, 1e-3),
    LayerSpec(200, 8 * 64, 8, (12, 12), (0.02, 0.005)),
    LayerSpec(77, 6 * 33 + 1, 6, (10, 3), (0.02, 0.005)),
]


@pytest.mark.parametrize("i", range(len(SPECS)))
@pytest.mark.parametrize("layout", ["rows", "tile4"])
def test_tcs_gemv(i, layout):
    vq = _vq()
    spec = SPECS[i]
    data = synth.make_layer(spec, seed=6100 + i, pad_garbage=layout == "rows")
    layer = _layer(data, layout)
    for batch in (3, 16):
        nws = vq.gemv_workspace_size(layer, batch)
        ws = torch.full((nws,), 0x55, dtype=torch.uint8, device="cuda")     # stale contents are fine
        for fp16 in (False, True):
            x = synth.make_x(6150 + i, batch, spec.in_features, outlier_frac=0.01, as_fp16=fp16)
            ref = oracle.linear(data, x, x_is_fp16=fp16)
            for od in (torch.float32, torch.bfloat16, torch.float16):
                y = vq.gemv(layer, _x_dev(x, fp16), out_dtype=od, workspace=ws)
                assert_close(_f64(y), ref, str(od).split(".")[-1])
                assert _status(ws) == vq.VQ_OK


@pytest.mark.parametrize("batch", range(2, 17))
def test_tcs_gemv_every_batch(batch, monkeypatch):
    monkeypatch.setenv("VQ_TCS_MIN_BATCH", "2")
    vq = _vq()
    spec = LayerSpec(700, 6 * 200 + 3, 6, (12, 4), (0.02, 0.005))
    data = synth.make_layer(spec, seed=6200)
    x = synth.make_x(6201, batch, spec.in_features, outlier_frac=0.01)
    ref = oracle.linear(data, x)
    for layout in ("rows", "tile4"):
        y = vq.gemv(_layer(data, layout), _x_dev(x), out_dtype=torch.float32)
        assert_close(_f64(y), ref, "float32")


@pytest.mark.parametrize("name,li", [("llama3_8b_up", 0), ("llama31_405b", 4)])
@pytest.mark.parametrize("layout", ["rows", "tile4"])
def test_tcs_gemv_model_layers(name, li, layout):
    """The 8B up_proj (14336 x 4096, 2^12 + 2^8) and the 405B gate_proj
    (53248 x 16384, d = 6, 2^12 + 2^4) at B = 4, 8, 16 on sampled rows."""
    vq = _vq()
    w = WORKLOADS[name]
    spec, seed = w.layers[li]
    data = synth.make_layer(spec, seed)
    layer = _layer(data, layout)
    rows = sample_rows(spec.out_features, 160, seed + 7)
    rd = torch.from_numpy(rows).cuda()
    x = synth.make_x(w.x_seed + li, 16, spec.in_features, w.outlier_frac)
    ref = oracle.linear(data, x, rows)
    for b in (4, 8, 16):
        y = vq.gemv(layer, _x_dev(x)[:b], out_dtype=torch.bfloat16)
        assert_close(_f64(y[:, rd]), ref[:b], "bfloat16")


def test_tcs_bounded_wait_gives_up_with_timeout_status(monkeypatch):
    vq = _vq()
    spec = LayerSpec(2000, 8 * 1000, 8, (12, 8), (0.02, 0.005))
    data = synth.make_layer(spec, seed=6500)
    layer = _layer(data, "rows")
    x = synth.make_x(6501, 8, spec.in_features, outlier_frac=0.01)
    ws = torch.zeros(vq.gemv_workspace_size(layer, 8), dtype=torch.uint8, device="cuda")
    monkeypatch.setenv("VQ_WAIT_BUDGET", "0")
    vq.gemv(layer, _x_dev(x), out_dtype=torch.float32, workspace=ws)
    assert _status(ws) == vq.VQ_ERR_TIMEOUT
    monkeypatch.delenv("VQ_WAIT_BUDGET")
    y = vq.gemv(layer, _x_dev(x), out_dtype=torch.float32, workspace=ws)
    assert _status(ws) == vq.VQ_OK
    assert_close(_f64(y), oracle.linear(data, x), "float32")

"""GPU parity for vq_gemm (tcgen05 prefill GEMM) against the fp64 oracle.

Both sources of weight tiles are exercised -- fused (centroids gathered into
shared memory) and staged (W_hat dequantised once, tiles by TMA) -- on shapes
spanning several tiles with ragged M, N and K edges, the generic vector
lengths, and the full-size prefill workloads on sampled output columns.  The
first word of the workspace is the kernel's status word (0 = no device wait
ran out of budget)."""
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


def _x_dev(x_bits, fp16=False):
    t = torch.from_numpy(x_bits.view(np.int16)).cuda()
    return t.view(torch.float16 if fp16 else torch.bfloat16)


def _run(layer, xd, out_dtype, kin):
    vq = _vq()
    m = xd.shape[0]
    need = vq.gemm_workspace_size(layer, m, xd.dtype)
    ws = torch.full((max(need, 256),), 0x7F, dtype=torch.uint8, device="cuda")
    y = vq.gemm(layer, xd, out_dtype=out_dtype, workspace=ws)
    torch.cuda.synchronize()
    status = int(ws[:4].view(torch.int32).item())
    assert status == 0, f"device status word {status}"
    return y


SPECS = [
    (LayerSpec(256, 64, 8, (16,), (0.02,)), 128),
    (LayerSpec(300, 1000, 8, (12, 8), (0.02, 0.005)), 200),
    (LayerSpec(512, 800, 8, (16, 8), (0.02, 0.005)), 64),
    (LayerSpec(600, 2048, 8, (16,), (0.02,), None, None), 260),
    (LayerSpec(257, 6 * 100 + 4, 6, (12, 4), (0.02, 0.005)), 130),
    (LayerSpec(100, 5 * 40 + 3, 5, (7, 3), (0.02, 0.005)), 33),
    (LayerSpec(64, 512, 8, (8, 8), (0.02, 0.005), (0.5, 1.5), None), 1),
    (LayerSpec(1, 8, 8, (4,), (0.02,)), 1),
    (LayerSpec(384, 3 * 64, 4, (9, 2), (0.02, 0.005)), 129),
]


@pytest.mark.parametrize("mode", ["fused", "staged"])
@pytest.mark.parametrize("i", range(len(SPECS)))
def test_gemm_small(monkeypatch, mode, i):
    monkeypatch.setenv("VQ_GEMM_MODE", mode)
    spec, m = SPECS[i]
    data = synth.make_layer(spec, seed=700 + i)
    kin = spec.in_features
    ld = (kin + 7) // 8 * 8
    x = synth.make_x(60 + i, m, kin, outlier_frac=0.01, ld=ld)
    ref = oracle.linear(data, x[:, :kin])
    layer = _vq().Layer.from_synth(data)
    xd = _x_dev(x)[:, :kin]
    for od in (torch.float32, torch.bfloat16):
        y = _run(layer, xd, od, kin)
        assert_close(y.double().cpu().numpy(), ref, str(od).split(".")[-1])


@pytest.mark.parametrize("mode", ["fused", "staged"])
def test_gemm_fp16_input_and_fp16_output(monkeypatch, mode):
    monkeypatch.setenv("VQ_GEMM_MODE", mode)
    spec = LayerSpec(500, 1024, 8, (16, 8), (0.02, 0.005))
    data = synth.make_layer(spec, seed=81)
    x = synth.make_x(82, 300, 1024, as_fp16=True)
    ref = oracle.linear(data, x, x_is_fp16=True)
    y = _run(_vq().Layer.from_synth(data), _x_dev(x, fp16=True), torch.float16, 1024)
    assert_close(y.double().cpu().numpy(), ref, "float16")


def _prefill_cases():
    for li in range(len(WORKLOADS["prefill_8192"].layers)):
        for m in WORKLOADS["prefill_8192"].batches:
            yield "prefill_8192", li, m
    for li in range(len(WORKLOADS["llama31_405b"].layers)):
        yield "llama31_405b", li, 1024


@pytest.mark.parametrize("name,li,m", list(_prefill_cases()))
def test_gemm_workloads(name, li, m):
    w = WORKLOADS[name]
    spec, seed = w.layers[li]
    data = synth.make_layer(spec, seed)
    layer = _vq().Layer.from_synth(data)
    x = synth.make_x(w.x_seed + li, m, spec.in_features, w.outlier_frac)
    cols = sample_rows(spec.out_features, 48, seed + 2)
    ref = oracle.linear(data, x, cols)
    y = _run(layer, _x_dev(x), torch.bfloat16, spec.in_features)
    got = y[:, torch.from_numpy(cols).cuda()].double().cpu().numpy()
    assert_close(got, ref, "bfloat16")


def test_gemm_both_modes_on_prefill_shape(monkeypatch):
    """The fused and staged forms agree with the oracle on the full 8192 x 8192
    prefill layer (M = 512) for every output column of a sampled row set."""
    spec, seed = WORKLOADS["prefill_8192"].layers[0]
    data = synth.make_layer(spec, seed)
    layer = _vq().Layer.from_synth(data)
    x = synth.make_x(5, 512, spec.in_features)
    cols = sample_rows(spec.out_features, 64, 9)
    ref = oracle.linear(data, x, cols)
    for mode in ("fused", "staged"):
        monkeypatch.setenv("VQ_GEMM_MODE", mode)
        y = _run(layer, _x_dev(x), torch.float32, spec.in_features)
        assert_close(y[:, torch.from_numpy(cols).cuda()].double().cpu().numpy(), ref, "float32")


@pytest.mark.parametrize("spec,m,mode", [
    (LayerSpec(30000, 520, 8, (12, 8), (0.02, 0.005)), 700, "fused"),
    (LayerSpec(30000, 520, 8, (16,), (0.02,)), 1000, "staged"),
    (LayerSpec(30000, 6 * 90 + 4, 6, (12, 4), (0.02, 0.005)), 515, "staged"),
])
def test_gemm_two_subtile_blocks(monkeypatch, spec, m, mode):
    """Wide layers make each CTA cover 256 rows of x (two accumulators sharing
    every weight tile); ragged M and K on both weight-tile sources."""
    monkeypatch.setenv("VQ_GEMM_MODE", mode)
    data = synth.make_layer(spec, seed=m)
    kin = spec.in_features
    ld = (kin + 7) // 8 * 8
    x = synth.make_x(m + 1, m, kin, outlier_frac=0.01, ld=ld)
    cols = sample_rows(spec.out_features, 64, m + 2)
    ref = oracle.linear(data, x[:, :kin], cols)
    y = _run(_vq().Layer.from_synth(data), _x_dev(x)[:, :kin], torch.float32, kin)
    assert_close(y[:, torch.from_numpy(cols).cuda()].double().cpu().numpy(), ref, "float32")


def test_gemm_degenerate_and_errors():
    vq = _vq()
    spec = LayerSpec(40, 0, 8, (4,), (0.02,))
    layer = vq.Layer.from_synth(synth.make_layer(spec, seed=1))
    y = torch.full((3, 40), 5.0, device="cuda")
    vq.gemm(layer, torch.zeros((3, 8), dtype=torch.bfloat16, device="cuda"), out=y)
    assert (y == 0).all()
    spec = LayerSpec(40, 64, 8, (4,), (0.02,))
    layer = vq.Layer.from_synth(synth.make_layer(spec, seed=2))
    x = torch.zeros((4, 72), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(vq.VQError) as e:             # ldx not a multiple of 8
        vq.gemm(layer, x[:, 1:65])
    assert e.value.status == vq.VQ_ERR_ALIGNMENT
    big = vq.Layer.from_synth(synth.make_layer(LayerSpec(16, 64, 16, (4,), (0.02,)), seed=3))
    with pytest.raises(vq.VQError) as e:             # d > 8 has no tensor-core path
        vq.gemm(big, x[:, :64])
    assert e.value.status == vq.VQ_ERR_UNSUPPORTED


@pytest.mark.parametrize("mode", ["fused", "staged"])
def test_gemm_bf16_rows_beyond_fp16_range(monkeypatch, mode):
    """bf16 activations beyond fp16's range (|x| up to 1e30) and rows of tiny
    values (1e-30): each row is scaled into fp16 by its own power of two, so
    every row stays within the bar (checked row by row), with scale and bias."""
    monkeypatch.setenv("VQ_GEMM_MODE", mode)
    spec = LayerSpec(300, 512, 8, (16, 8), (0.02, 0.005))
    data = synth.make_layer(spec, seed=91)
    x = oracle.bf16_to_f32(synth.make_x(92, 130, 512, outlier_frac=0.01))
    x[0] *= np.float32(1e30)
    x[1] *= np.float32(1e5)          # past 65504
    x[2] *= np.float32(1e-30)
    x[3] = 0.0                       # an all-zero row
    xb = oracle.f32_to_bf16(x)
    ref = oracle.linear(data, xb)
    y = _run(_vq().Layer.from_synth(data), _x_dev(xb), torch.float32, 512).double().cpu().numpy()
    assert np.isfinite(y).all()
    for r in range(xb.shape[0]):
        assert_close(y[r:r + 1], ref[r:r + 1], "float32")


@pytest.mark.parametrize("mode", ["fused", "staged"])
def test_gemm_bounded_wait_gives_up_with_timeout_status(monkeypatch, mode):
    """With a wait budget of 0 clocks the pipeline's first wait that finds its
    stage not yet complete gives up: the call completes, the status word reads
    VQ_ERR_TIMEOUT, and the next call with the normal budget is correct."""
    vq = _vq()
    monkeypatch.setenv("VQ_GEMM_MODE", mode)
    spec = LayerSpec(1024, 2048, 8, (16,), (0.02,))
    data = synth.make_layer(spec, seed=95)
    layer = vq.Layer.from_synth(data)
    x = synth.make_x(96, 512, 2048, outlier_frac=0.01)
    xd = _x_dev(x)
    ws = torch.zeros(vq.gemm_workspace_size(layer, 512, xd.dtype), dtype=torch.uint8, device="cuda")
    monkeypatch.setenv("VQ_WAIT_BUDGET", "0")
    vq.gemm(layer, xd, out_dtype=torch.float32, workspace=ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == vq.VQ_ERR_TIMEOUT
    monkeypatch.delenv("VQ_WAIT_BUDGET")
    y = _run(layer, xd, torch.float32, 2048)
    assert_close(y.double().cpu().numpy(), oracle.linear(data, x), "float32")

"""GPU parity for the randomized Hadamard transform (vq_rht) and the decode
product of a layer stored in the rotated basis (vq_gemv_rht), against the
oracle's plain O(n b) transform: block sizes from 1 (odd n) to 2^15, ragged
row counts, every input and output type, forward, inverse and the round
trip; then y = U^T (W~ (V x)) for row-order and tiled layers at batch 1 and
4, within the decode bar."""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth import LayerSpec, WORKLOADS
from tests._util import assert_close, sample_rows

pytestmark = pytest.mark.gpu

_TORCH = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32}


def _vq():
    from bit_packed_index_b200 import vq
    return vq


def _signs(n, seed):
    rng = np.random.default_rng(seed)
    bits = rng.integers(0, 2, size=n).astype(np.uint8)
    words = np.packbits(np.concatenate([bits, np.zeros((-n) % 32, np.uint8)]), bitorder="little")
    words = words.view(np.uint32)
    return words, torch.from_numpy(words.view(np.int32).copy()).cuda()


def _rand(rows, n, dtype, seed):
    rng = np.random.default_rng(seed)
    x = torch.from_numpy(rng.standard_normal((rows, n), dtype=np.float32)).cuda().to(_TORCH[dtype])
    return x, x.double().cpu().numpy()


@pytest.mark.parametrize("n", [1, 6, 24, 96, 1000, 6144, 8192, 28672, 65536])
@pytest.mark.parametrize("dtype", ["bf16", "fp16", "fp32"])
def test_rht_matches_the_oracle(n, dtype):
    vq = _vq()
    rows = 3 if n < 32768 else 1
    x, xf = _rand(rows, n, dtype, 4000 + n)
    words, sd = _signs(n, 4100 + n)
    for inverse in (False, True):
        ref = oracle.rht(xf, words, inverse=inverse)
        y = vq.rht(x, sd, inverse=inverse, out_dtype=torch.float32)
        err = np.abs(y.double().cpu().numpy() - ref).max() / np.abs(ref).max()
        assert err < 1e-5, (inverse, err)
    # bf16 / fp16 outputs: the fp32 result rounded once
    for od in ("bf16", "fp16"):
        y = vq.rht(x, sd, out_dtype=_TORCH[od]).double().cpu().numpy()
        ref = oracle.rht(xf, words)
        u = 2.0 ** -8 if od == "bf16" else 2.0 ** -11
        assert (np.abs(y - ref) <= u * np.abs(ref) + 1e-5 * np.abs(ref).max()).all()


def test_rht_round_trip_and_strides():
    vq = _vq()
    n = 4096 + 2048
    gen = torch.Generator(device="cuda").manual_seed(4199)
    base = torch.randn((5, n + 64), device="cuda", dtype=torch.float32, generator=gen)
    x = base[:, :n]                                    # row stride n + 64
    _, sd = _signs(n, 4200)
    y = vq.rht(x, sd)
    z = vq.rht(y, sd, inverse=True)
    assert torch.allclose(z, x, atol=1e-5, rtol=1e-5)
    assert torch.allclose(y.norm(dim=1), x.norm(dim=1), rtol=1e-5)


def _rotated_ref(data, x_bits, s_in, s_out):
    """U^T (W~ (V x)) in fp64 with the oracle's transform and dequant."""
    w = oracle.f16_to_f32(oracle.dequant(data)).astype(np.float64)
    x = oracle.bf16_to_f32(x_bits).astype(np.float64)
    xt = oracle.rht(x, s_in)
    yt = xt @ w.T
    return oracle.rht(yt, s_out, inverse=True)


GEMV_RHT_SPECS = [
    LayerSpec(384, 1000, 8, (12, 8), (0.02, 0.005)),           # blocks of 8 / 128
    LayerSpec(300, 8 * 100 + 5, 8, (16,), (0.02,)),             # odd Kin: blocks of 1
    LayerSpec(3072, 2048, 8, (16,), (0.02,)),
]


@pytest.mark.parametrize("i", range(len(GEMV_RHT_SPECS)))
@pytest.mark.parametrize("layout", ["rows", "tile4"])
@pytest.mark.parametrize("batch", [1, 4])
def test_gemv_rht_matches_the_oracle(i, layout, batch):
    vq = _vq()
    spec = GEMV_RHT_SPECS[i]
    data = synth.make_layer(spec, seed=4300 + i)
    layer = vq.Layer.from_synth(data, layout=layout)
    s_in, d_in = _signs(spec.in_features, 4310 + i)
    s_out, d_out = _signs(spec.out_features, 4320 + i)
    x = synth.make_x(4330 + i, batch, spec.in_features, outlier_frac=0.01)
    xd = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    y = vq.gemv_rht(layer, d_in, d_out, xd, out_dtype=torch.float32)
    assert_close(y.double().cpu().numpy(), _rotated_ref(data, x, s_in, s_out), "float32")


def test_gemv_rht_70b_gate_tiled():
    """The 70B gate layer (blocks of 8192 in, 4096 out) in the tiled order."""
    vq = _vq()
    w = WORKLOADS["llama3_70b_mlp"]
    spec, seed = w.layers[0]
    data = synth.make_layer(spec, seed)
    layer = vq.Layer.from_synth(data, layout="tile4")
    s_in, d_in = _signs(spec.in_features, 4400)
    s_out, d_out = _signs(spec.out_features, 4401)
    x = synth.make_x(w.x_seed, 1, spec.in_features, w.outlier_frac)
    xd = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    y = vq.gemv_rht(layer, d_in, d_out, xd, out_dtype=torch.bfloat16)
    assert_close(y.double().cpu().numpy(), _rotated_ref(data, x, s_in, s_out), "bfloat16")

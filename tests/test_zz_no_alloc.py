"""vq_gemv_noalloc: the decode GEMV for callers that cannot allocate device
memory where they run the layer (it takes its split-K scratch from a fixed
array inside the library).  Its output must match vq_gemv's, which gets a
caller-allocated workspace, and the fp64 oracle, on two calls in a row (the
second call finds the first call's leftovers in the shared array).  This file is collected last so
that a run stopping at the first failure has already run every other test."""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth import LayerSpec
from tests._util import TOL, assert_close, normwise_err

pytestmark = pytest.mark.gpu


def _x_dev(x_bits):
    return torch.from_numpy(x_bits.view(np.int16)).cuda().view(torch.bfloat16)


@pytest.mark.parametrize("spec,batch", [
    (LayerSpec(512, 8 * 4000, 8, (16,), (0.02,)), 1),          # single-row kernel, K split
    (LayerSpec(1024, 6 * 2731, 6, (12, 4), (0.02, 0.005)), 4),  # batched kernel, K split
    (LayerSpec(2048, 4096, 8, (12, 8), (0.02, 0.005)), 16),
])
def test_noalloc_matches_workspace_version_twice(spec, batch):
    from bit_packed_index_b200 import vq
    data = synth.make_layer(spec, seed=4242)
    layer = vq.Layer.from_synth(data)
    need = vq.gemv_workspace_size(layer, batch)
    assert 0 < need <= vq.NOALLOC_SCRATCH_BYTES        # the scratch is really used
    xb = synth.make_x(4243, batch, spec.in_features)
    x = _x_dev(xb)
    exact = oracle.linear(data, xb)                      # the fp64 definition
    ref = vq.gemv(layer, x, out_dtype=torch.float32).double().cpu().numpy()
    for _ in range(2):
        out = torch.full((batch, spec.out_features), float("nan"), device="cuda")
        vq.gemv_noalloc(layer, x, out=out)
        got = out.double().cpu().numpy()
        assert np.isfinite(got).all()
        assert normwise_err(got, ref) <= TOL
        assert_close(got, exact, "float32")


def test_noalloc_rejects_layers_beyond_the_scratch():
    from bit_packed_index_b200 import vq
    # a tiled layer with a 2^16 book and a residual book runs only the split-K
    # kernel at batch 16, whose partial sums take ~10.5 MB
    spec = LayerSpec(28672, 8192, 8, (16, 8), (0.02, 0.005))
    data = synth.make_layer(spec, seed=4244)
    layer = vq.repack_tile4(vq.Layer.from_synth(data))
    assert vq.gemv_workspace_size(layer, 16) > vq.NOALLOC_SCRATCH_BYTES
    x = _x_dev(synth.make_x(4245, 16, spec.in_features))
    with pytest.raises(vq.VQError) as e:
        vq.gemv_noalloc(layer, x)
    assert e.value.status == vq.VQ_ERR_WORKSPACE

"""GPU parity for the Hessian of a layer's inputs (vq_hessian: h = 2 X^T X / n
+ 0.01 mean(diag) I, X^T X on the tcgen05 tensor cores) against the oracle's
fp64 definition.  Bar: fp32 accumulation of n exact products is off by at
most about n * 2^-24 of sum_t |x_ti x_tj| <= max_i h_ii (Cauchy-Schwarz), so
max |h - ref| <= (n * 2^-24 + 1e-6) * max |ref| (normwise)."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


def _vq():
    from bit_packed_index_b200 import vq
    return vq


def _bits(n, d, seed, fp16, outliers=0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, d), dtype=np.float32)
    if outliers:
        x[:, rng.choice(d, outliers, replace=False)] *= 20.0
    return oracle.f32_to_f16(x) if fp16 else oracle.f32_to_bf16(x)


def _dev(bits, fp16):
    return torch.from_numpy(bits.view(np.int16)).cuda().view(torch.float16 if fp16 else torch.bfloat16)


def _bar(n):
    return n * 2.0 ** -24 + 1e-6


@pytest.mark.parametrize("n,d", [(40, 8), (300, 48), (1000, 200), (4096, 130), (777, 1000), (1, 3)])
@pytest.mark.parametrize("fp16", [False, True])
def test_hessian_matches_the_oracle(n, d, fp16):
    vq = _vq()
    xb = _bits(n, d, 5000 + n + d, fp16, outliers=min(2, d // 8))
    h = vq.hessian(_dev(xb, fp16)).double().cpu().numpy()
    ref = oracle.hessian(xb, x_is_fp16=fp16)
    err = np.abs(h - ref).max() / np.abs(ref).max()
    assert err <= _bar(n), err


def test_hessian_strided_input_and_output():
    vq = _vq()
    n, d = 500, 96
    xb = _bits(n, d + 40, 5100, False)
    x = _dev(xb, False)[:, :d]                        # row stride d + 40
    out = torch.full((d, d + 8), float("nan"), dtype=torch.float32, device="cuda")[:, :d]
    h = vq.hessian(x, out=out).double().cpu().numpy()
    ref = oracle.hessian(np.ascontiguousarray(xb[:, :d]))
    assert np.abs(h - ref).max() / np.abs(ref).max() <= _bar(n)


def test_hessian_large_sampled_columns():
    """4096 tokens x 8192 features; the off-diagonal block of 64 sampled
    features against the oracle on those columns (damping touches only the
    diagonal, which the small cases check)."""
    vq = _vq()
    n, d = 4096, 8192
    xb = _bits(n, d, 5200, False, outliers=8)
    h = vq.hessian(_dev(xb, False))
    cols = np.sort(np.random.default_rng(5201).choice(d, 64, replace=False))
    sub = h[torch.from_numpy(cols).cuda()][:, torch.from_numpy(cols).cuda()].double().cpu().numpy()
    ref = oracle.hessian(np.ascontiguousarray(xb[:, cols]))
    off = ~np.eye(64, dtype=bool)
    scale = np.abs(ref).max()
    assert np.abs(sub - ref)[off].max() / scale <= _bar(n)

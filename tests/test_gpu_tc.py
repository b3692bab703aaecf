"""GPU: the tensor-core GEMMs in isolation against float64 products of the same
bf16 values (the oracle's matmul is numpy's), K-major and MN-major operands,
ragged tails in every dimension."""
import numpy as np
import pytest
import torch

from learnable_channel_permutation_b200 import binding as b
from learnable_channel_permutation_b200 import synth

import gpu_helpers as H

pytestmark = pytest.mark.gpu


def _bf(shape, seed, scale=1.0):
    x = np.random.default_rng(seed).standard_normal(shape).astype(np.float32) * np.float32(scale)
    return synth.bf16_round(x)


@pytest.mark.parametrize("T,cout,cin", [(200, 392, 256), (128, 256, 64), (1, 8, 8), (333, 520, 4104),
                                        (2048, 4096, 4096)])
def test_calib_gemm_dense_and_sparse_outputs(gpu_lib, T, cout, cin):
    X, W, At = _bf((T, cin), 1), _bf((cout, cin), 2, 0.02), _bf((cout, cin), 3, 0.02)
    dev = lambda a: torch.from_numpy(a).cuda().to(torch.bfloat16)
    Yd = torch.full((T, cout), float("nan"), device="cuda")
    Ys = torch.full((T, cout), float("nan"), device="cuda")
    b.calib_gemm(dev(X), dev(W), dev(At), Yd, Ys)
    torch.cuda.synchronize()
    assert b.device_error() == 0
    ref_d = X.astype(np.float64) @ W.astype(np.float64).T
    ref_s = X.astype(np.float64) @ At.astype(np.float64).T
    assert H.relerr(Yd.cpu().numpy(), ref_d) <= 1e-5
    assert H.relerr(Ys.cpu().numpy(), ref_s) <= 1e-5


@pytest.mark.parametrize("T,cout,cin", [(200, 392, 256), (64, 128, 256), (1, 8, 8), (333, 520, 264),
                                        (2048, 4096, 4096)])
def test_grad_gemm_mn_major_operands(gpu_lib, T, cout, cin):
    G, X = _bf((T, cout), 4, 1e-3), _bf((T, cin), 5)
    dAt = torch.full((cout, cin), float("nan"), device="cuda", dtype=torch.bfloat16)
    b.grad_gemm(torch.from_numpy(G).cuda().to(torch.bfloat16), torch.from_numpy(X).cuda().to(torch.bfloat16), dAt)
    torch.cuda.synchronize()
    assert b.device_error() == 0
    ref = G.astype(np.float64).T @ X.astype(np.float64)
    got = dAt.float().cpu().numpy()
    # float32 accumulation, one bf16 rounding of the result (2^-9 relative)
    assert H.relerr(got, ref) <= 4e-3
    assert np.max(np.abs(got - ref)) <= 2 ** -8 * np.max(np.abs(ref)) + 1e-30

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


@pytest.mark.parametrize("T,cout,cin", [(200, 392, 256), (128, 256, 64), (1, 8, 8), (333, 520, 4104),
                                        (300, 4160, 192), (2048, 4096, 4096)])
def test_calib_gemm_loss_epilogue(gpu_lib, T, cout, cin):
    """The loss epilogue: D = Y_d - Y_s and Y_s in bf16 (one rounding of the
    float32 accumulations) and the per-token partials of every 64-channel slot."""
    X, W, At = _bf((T, cin), 1), _bf((cout, cin), 2, 0.02), _bf((cout, cin), 3, 0.02)
    dev = lambda a: torch.from_numpy(a).cuda().to(torch.bfloat16)
    nsl = (cout + 63) // 64
    D = torch.full((T, cout), float("nan"), device="cuda", dtype=torch.bfloat16)
    Ys = torch.full((T, cout), float("nan"), device="cuda", dtype=torch.bfloat16)
    part = torch.full((T, nsl, 4), float("nan"), device="cuda")
    b.calib_gemm_loss(dev(X), dev(W), dev(At), D, Ys, part)
    torch.cuda.synchronize()
    assert b.device_error() == 0
    yd = X.astype(np.float64) @ W.astype(np.float64).T
    ys = X.astype(np.float64) @ At.astype(np.float64).T
    got_d, got_s = D.float().cpu().numpy(), Ys.float().cpu().numpy()
    assert H.relerr(got_d, yd - ys) <= 4e-3
    assert H.relerr(got_s, ys) <= 4e-3
    assert np.max(np.abs(got_s - ys)) <= 2 ** -8 * np.max(np.abs(ys)) + 1e-30
    p = part.cpu().numpy()
    ref = np.zeros((T, nsl, 3))
    for s in range(nsl):
        c = slice(64 * s, min(64 * s + 64, cout))
        ref[:, s, 0] = np.sum(yd[:, c] * ys[:, c], axis=1)
        ref[:, s, 1] = np.sum(yd[:, c] ** 2, axis=1)
        ref[:, s, 2] = np.sum(ys[:, c] ** 2, axis=1)
    for k in range(3):
        assert H.relerr(p[:, :, k], ref[:, :, k]) <= 1e-5, k
    assert np.all(p[:, :, 3] == 0)


def _pair_inputs(T, cout, seed, zero_token=None):
    rng = np.random.default_rng(seed)
    yd = rng.standard_normal((T, cout))
    ys = 0.7 * yd + 0.5 * rng.standard_normal((T, cout))
    if zero_token is not None:
        ys[zero_token] = 0.0
    nsl = (cout + 63) // 64
    part = np.zeros((T, nsl, 4), np.float32)
    for s in range(nsl):
        c = slice(64 * s, min(64 * s + 64, cout))
        part[:, s, 0] = np.sum(yd[:, c] * ys[:, c], axis=1)
        part[:, s, 1] = np.sum(yd[:, c] ** 2, axis=1)
        part[:, s, 2] = np.sum(ys[:, c] ** 2, axis=1)
    Dq = synth.bf16_round((yd - ys).astype(np.float32))
    Sq = synth.bf16_round(ys.astype(np.float32))
    return yd, ys, Dq, Sq, part


@pytest.mark.parametrize("T,cout,zero", [(1, 8, None), (37, 264, 5), (300, 4096, None), (64, 11008, 0),
                                         (40, 13824, None)])
def test_loss_pair_against_the_oracle(gpu_lib, T, cout, zero):
    from oracle import lcp_oracle as O
    counter = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call in range(2):       # the kernel leaves its counter at zero for the next call
        yd, ys, Dq, Sq, part = _pair_inputs(T, cout, 40 + call, zero)
        loss = torch.full((1,), float("nan"), device="cuda")
        stats = torch.empty(T, 4, device="cuda")
        G = torch.full((T, cout), float("nan"), device="cuda", dtype=torch.bfloat16)
        to = lambda a: torch.from_numpy(a).cuda().to(torch.bfloat16)
        b.loss_pair(to(Dq), to(Sq), torch.from_numpy(part).cuda(), loss, stats, G, counter)
        torch.cuda.synchronize()
        assert int(counter[0]) == 0
        ref, cos = O.cosine_loss(yd.T, ys.T)
        assert abs(float(loss[0]) - ref) <= 1e-5 * abs(ref)
        assert H.relerr(stats.cpu().numpy()[:, 3], cos) <= 1e-5
        # G from the bf16 pair (y_d = D + Ys) with the exact statistics, then one bf16 rounding
        g = G.float().cpu().numpy()
        ydq, ysq = Dq.astype(np.float64) + Sq, Sq.astype(np.float64)
        dot, nd, ns = np.sum(yd * ys, 1), np.linalg.norm(yd, axis=1), np.linalg.norm(ys, axis=1)
        den = nd * ns
        ok = den > O.COS_EPS
        c = np.where(ok, dot / np.where(ok, den, 1), 0)
        ca = np.where(ok, -1 / (T * np.where(ok, den, 1)), -1 / (T * O.COS_EPS))
        cb = np.where(ok, c / (T * np.where(ok, ns * ns, 1)), 0)
        g_pair = ca[:, None] * ydq + cb[:, None] * ysq
        assert H.relerr(g, g_pair) <= 4e-3
        # and against the oracle's gradient on the exact outputs: the pair's bf16 rounding on top
        assert H.relerr(g, O.cosine_loss_grad(yd.T, ys.T).T) <= 1e-2

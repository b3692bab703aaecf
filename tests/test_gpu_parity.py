"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Every comparison uses seeded inputs from ``synth``; the oracle never sees a
value that came from the GPU except where stated: the mask-conditioned
gradient check gives the oracle the GPU's mask, and the mask bit-exactness
check gives the oracle the GPU's W' (the two are defined that way: the mask
is only unique given identical W').
"""
import numpy as np
import pytest
import torch

from learnable_channel_permutation_b200 import binding as b
from learnable_channel_permutation_b200 import synth
from oracle import lcp_oracle as O

import gpu_helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu(gpu_lib):
    yield


# ------------------------------------------------------------- Sinkhorn ----

@pytest.mark.parametrize("B", [32, 64, 128, 256])
@pytest.mark.parametrize("iters,tau,scale", [(5, 0.5, 1e-3), (1, 1.0, 1.0), (20, 0.1, 0.05), (5, 1.0, 3.0)])
def test_sinkhorn_fwd_matches_oracle(B, iters, tau, scale):
    nb = 3
    L = (np.random.default_rng(B + iters).standard_normal((nb, B, B)) * scale).astype(np.float32)
    Ld = torch.from_numpy(L).cuda()
    P = torch.empty_like(Ld)
    ck = torch.empty(nb, iters, 2, B, device="cuda")
    b.sinkhorn_fwd(Ld, P, ck, tau, iters)
    torch.cuda.synchronize()
    Pref, _ = O.sinkhorn(L, tau, iters)
    assert H.relerr(P.cpu().numpy(), Pref) <= H.TOL_P
    assert np.max(np.abs(P.cpu().numpy().sum(axis=1) - 1)) < 1e-5


def test_sinkhorn_model_scale_kernels_match_oracle():
    """B = 64 launches of at least 1024 blocks run the forward pass one warp a block and the
    reverse pass two warps a block: 1100 blocks, every fifth one peaked enough (range of Z_0
    above 64) for the log-domain fallback, the rest in the linear domain; reverse with two
    dP partials."""
    nb, B, iters, tau, splits = 1100, 64, 5, 0.1, 2
    rng = np.random.default_rng(64064)
    scale = np.where(np.arange(nb) % 5 == 0, 1.5, 0.01)[:, None, None]
    L = (rng.standard_normal((nb, B, B)) * scale).astype(np.float32)
    dP = rng.standard_normal((splits, nb, B, B)).astype(np.float32)
    Ld = torch.from_numpy(L).cuda()
    P = torch.empty_like(Ld)
    ck = torch.empty(nb, iters, 2, B, device="cuda")
    dL = torch.empty_like(Ld)
    b.sinkhorn_fwd(Ld, P, ck, tau, iters)
    b.sinkhorn_bwd(Ld, ck, torch.from_numpy(dP).cuda(), dL, tau, iters)
    torch.cuda.synchronize()
    Pref, tr = O.sinkhorn(L, tau, iters)
    ref = O.sinkhorn_backward(tr, Pref, dP.astype(np.float64).sum(axis=0), tau)
    Pg, dLg = P.cpu().numpy(), dL.cpu().numpy()
    z = L / tau
    peaked = (z.max(axis=(1, 2)) - z.min(axis=(1, 2))) > 64
    assert 0 < peaked.sum() < nb                      # both arithmetics are exercised
    for sel in (peaked, ~peaked):
        assert H.relerr(Pg[sel], Pref[sel]) <= H.TOL_P
        assert H.relerr(dLg[sel], ref[sel]) <= 1e-5
    assert np.max(np.abs(Pg.sum(axis=1) - 1)) < 1e-5


@pytest.mark.parametrize("B", [32, 64, 128, 256])
@pytest.mark.parametrize("splits", [1, 3])
def test_sinkhorn_bwd_matches_oracle(B, splits):
    nb, iters, tau = 2, 5, 0.5
    rng = np.random.default_rng(100 + B)
    L = (rng.standard_normal((nb, B, B)) * 0.5).astype(np.float32)
    dP = rng.standard_normal((splits, nb, B, B)).astype(np.float32)
    Ld = torch.from_numpy(L).cuda()
    P = torch.empty_like(Ld)
    ck = torch.empty(nb, iters, 2, B, device="cuda")
    dL = torch.empty_like(Ld)
    b.sinkhorn_fwd(Ld, P, ck, tau, iters)
    b.sinkhorn_bwd(Ld, ck, torch.from_numpy(dP).cuda(), dL, tau, iters)
    torch.cuda.synchronize()
    Pref, tr = O.sinkhorn(L, tau, iters)
    ref = O.sinkhorn_backward(tr, Pref, dP.astype(np.float64).sum(axis=0), tau)
    assert H.relerr(dL.cpu().numpy(), ref) <= 1e-5
    # row-shift invariance of the forward makes every row of dL sum to zero
    assert np.max(np.abs(dL.cpu().numpy().sum(axis=2))) <= 1e-5 * np.max(np.abs(ref)) * B


# ---------------------------------------------------------------- mask -----

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("n,m", [(2, 4), (4, 8), (1, 4), (3, 4), (1, 8), (7, 8), (4, 4)])
def test_nm_mask_bit_exact(dtype, n, m):
    rng = np.random.default_rng(7 * n + m)
    rows, cols = 37, 320
    W = (np.round(rng.standard_normal((rows, cols)) * 4) / 4).astype(np.float32)   # many ties
    W[0, :8] = [0.0, -0.0, 0.0, -0.0, 1.0, -1.0, 1.0, -1.0]
    W[1] = rng.standard_normal(cols).astype(np.float32)
    if dtype == "bf16":
        W = synth.bf16_round(W)
    Wt = torch.from_numpy(W).cuda()
    if dtype == "bf16":
        Wt = Wt.to(torch.bfloat16)
    bits = torch.empty(rows, cols // 32, dtype=torch.int32, device="cuda")
    b.nm_mask(Wt, bits, n, m)
    torch.cuda.synchronize()
    ref = O.pack_mask_bits(O.nm_mask(W, n, m))
    assert np.array_equal(bits.cpu().numpy().view(np.uint32), ref)


def test_nm_mask_large_ragged_rows():
    rng = np.random.default_rng(5)
    W = rng.standard_normal((4099, 4096)).astype(np.float32)
    bits = torch.empty(4099, 128, dtype=torch.int32, device="cuda")
    b.nm_mask(torch.from_numpy(W).cuda(), bits, 2, 4)
    torch.cuda.synchronize()
    assert np.array_equal(bits.cpu().numpy().view(np.uint32), O.pack_mask_bits(O.nm_mask(W, 2, 4)))


# ------------------------------------------------------------- permute -----

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_permute_weight_matches_oracle(dtype):
    rng = np.random.default_rng(9)
    B, nb, cout = 64, 3, 200
    W = (rng.standard_normal((cout, nb * B)) * 0.02).astype(np.float32)
    if dtype == "bf16":
        W = synth.bf16_round(W)
    P, _ = O.sinkhorn(rng.standard_normal((nb, B, B)), 0.5, 5)
    P32 = P.astype(np.float32)
    Wt = torch.from_numpy(W).cuda()
    if dtype == "bf16":
        Wt = Wt.to(torch.bfloat16)
    Wp = torch.empty(cout, nb * B, device="cuda")
    b.permute_weight(Wt, torch.from_numpy(P32).cuda(), Wp)
    torch.cuda.synchronize()
    assert H.relerr(Wp.cpu().numpy(), O.permute_weight(W.astype(np.float64), P32.astype(np.float64))) <= 1e-6


# ---------------------------------------------------------------- loss -----

@pytest.mark.parametrize("T,cout", [(1, 8), (37, 264), (300, 4096)])
def test_loss_fwd_bwd_match_oracle(T, cout):
    rng = np.random.default_rng(T)
    Yd = rng.standard_normal((T, cout)).astype(np.float32)
    Ys = (Yd * 0.7 + rng.standard_normal((T, cout)) * 0.5).astype(np.float32)
    Ydd, Ysd = torch.from_numpy(Yd).cuda(), torch.from_numpy(Ys).cuda()
    loss = torch.empty(1, device="cuda")
    stats = torch.empty(T, 4, device="cuda")
    G = torch.empty(T, cout, device="cuda")
    b.loss_fwd(Ydd, Ysd, loss, stats)
    b.loss_bwd(Ydd, Ysd, stats, G)
    torch.cuda.synchronize()
    ref, _ = O.cosine_loss(Yd.T.astype(np.float64), Ys.T.astype(np.float64))
    Gref = O.cosine_loss_grad(Yd.T.astype(np.float64), Ys.T.astype(np.float64)).T
    assert abs(float(loss[0]) - ref) / ref <= 1e-5
    assert H.relerr(G.cpu().numpy(), Gref) <= 1e-5


# --------------------------------------------------------- whole step ------

def _step_case(wl, flags=0, tol_loss=None, tol_dl=None, cos=None, L_override=None):
    inputs = synth.make_inputs(wl)
    out, s = H.run_gpu(wl, inputs, flags=flags, L_override=L_override)
    f32 = wl.dtype == "f32"
    errs = []
    for li, g in zip(inputs, out):
        td, tc = H.dl_bounds(li.spec, wl.dtype)
        errs.append(H.check_layer(li, wl, g, tol_loss or (H.TOL_LOSS_F32 if f32 else H.TOL_LOSS_BF16),
                                  tol_dl or td, cos if cos is not None else tc))
    return errs


def test_step_toy_fp32_layer():
    errs = _step_case(synth.toy_256())
    assert errs[0]["mask_agree"] > 0.99


@pytest.mark.parametrize("flags", [0, b.FLAG_SIMT])
def test_step_bf16_ragged_with_outliers(flags):
    wl = synth.custom(392, 256, 200, 64, 2, 4, 0.5, 5, "bf16", seed=1, outliers=True)
    _step_case(wl, flags=flags)


@pytest.mark.parametrize("flags", [0, b.FLAG_SIMT])
@pytest.mark.parametrize("B,n,m,iters,tau", [(32, 2, 4, 5, 1.0), (128, 4, 8, 20, 0.1), (256, 2, 4, 5, 0.5),
                                             (64, 4, 8, 5, 1.0)])
def test_step_bf16_block_sizes(flags, B, n, m, iters, tau):
    wl = synth.custom(136, 512, 72, B, n, m, tau, iters, "bf16", seed=B + n)
    _step_case(wl, flags=flags)


def test_step_fp32_block_sizes_and_4of8():
    for B, n, m in ((32, 2, 4), (128, 4, 8), (256, 2, 4)):
        wl = synth.custom(48, 512, 40, B, n, m, 0.5, 5, "f32", seed=3)
        _step_case(wl)


@pytest.mark.parametrize("flags", [0, b.FLAG_SIMT])
def test_step_multi_layer_shared_x(flags):
    wl = synth.Workload("mini_mlp", [
        synth.LayerSpec("gate", 264, 256, 96, "x256"),
        synth.LayerSpec("up", 264, 256, 96, "x256"),
        synth.LayerSpec("down", 256, 256, 96, "x256b", x_kind="halfnormal"),
    ], block=64, n=2, m=4, tau=0.5, iters=5, dtype="bf16")
    _step_case(wl, flags=flags)


@pytest.mark.parametrize("flags", [0, b.FLAG_SIMT])
def test_step_single_token_and_minimum_rows(flags):
    wl = synth.custom(8, 64, 1, 64, 2, 4, 0.5, 5, "bf16", seed=4)
    _step_case(wl, flags=flags)


def test_step_identity_logits_collapse_to_plain_pruning():
    # L = c I with c / tau large gives P = I exactly in float32: W' = W and the
    # mask is plain N:M magnitude pruning of W, bit for bit.
    wl = synth.custom(128, 256, 64, 64, 2, 4, 0.5, 5, "bf16", seed=6)
    inputs = synth.make_inputs(wl)
    L = np.broadcast_to(np.eye(64, dtype=np.float32) * 200.0, (4, 64, 64)).copy()
    out, _ = H.run_gpu(wl, inputs, L_override=[L])
    g = out[0]
    assert np.array_equal(g["P"], np.broadcast_to(np.eye(64, dtype=np.float32), g["P"].shape))
    assert np.array_equal(g["mask_words"], O.pack_mask_bits(O.nm_mask(inputs[0].W, 2, 4)))


def test_step_zero_logits_keep_the_first_n_of_each_group():
    # L = 0: P = 1/B, every column of a block of W' is the block mean, and the
    # tie rule keeps indices 0..N-1 of each group -- provided the GPU's W'
    # columns of a block are bitwise equal, which this checks as well.
    wl = synth.custom(64, 128, 32, 32, 2, 4, 1.0, 5, "bf16", seed=8)
    inputs = synth.make_inputs(wl)
    out, _ = H.run_gpu(wl, inputs, L_override=[np.zeros((4, 32, 32), np.float32)])
    g = out[0]
    Wp = g["Wp"].reshape(64, 4, 32)
    assert np.all(Wp == Wp[:, :, :1])
    mk = g["mask"].reshape(64, -1, 4)
    assert np.all(mk[:, :, :2]) and not np.any(mk[:, :, 2:])


def test_step_peaked_permutation_recovered():
    wl = synth.custom(96, 128, 48, 32, 2, 4, 0.5, 5, "bf16", seed=9)
    inputs = synth.make_inputs(wl)
    rng = np.random.default_rng(9)
    sig = [rng.permutation(32) for _ in range(4)]
    L = np.zeros((4, 32, 32), np.float32)
    for k in range(4):
        L[k, np.arange(32), sig[k]] = 100.0
    out, _ = H.run_gpu(wl, inputs, L_override=[L])
    g = out[0]
    for k in range(4):
        assert np.array_equal(np.argmax(g["P"][k], axis=1), sig[k])
    W = inputs[0].W
    for k in range(4):
        for i in range(32):
            assert np.array_equal(g["Wp"][:, 32 * k + sig[k][i]], W[:, 32 * k + i])


def test_empty_call_is_a_noop():
    import ctypes
    hp = b.hparams(64, 2, 4, 5, 0.5, b.BF16)
    assert b.lib().lcp_step(None, 0, ctypes.byref(hp), None, 0, None) == 0


def test_workload_q_proj_full_size():
    """The headline layer (4096 x 4096, T = 2048, B = 64, 2:4) in the launch
    configuration the benchmark times, against the float64 oracle."""
    wl = synth.q_proj_4096()
    errs = _step_case(wl)
    assert errs[0]["mask_agree"] > 0.9

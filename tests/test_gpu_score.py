"""Importance-score masks ([PermLLM] integration with existing pruning methods):
the score kernels against the oracle, and steps with LCP_FLAG_SCORE whose mask
is taken from S_hat = S P_B."""
import numpy as np
import pytest
import torch

from learnable_channel_permutation_b200 import binding as b
from learnable_channel_permutation_b200 import synth
from oracle import lcp_oracle as O

import gpu_helpers as H

pytestmark = pytest.mark.gpu

KINDS = {"magnitude": b.SCORE_MAGNITUDE, "wanda": b.SCORE_WANDA, "ria": b.SCORE_RIA}


@pytest.mark.parametrize("kind", list(KINDS))
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_score_matches_oracle(gpu_lib, kind, dtype):
    wl = synth.custom(200, 320, 96, 64, 2, 4, 1.0, 5, dtype, seed=60, outliers=True)
    li = synth.make_inputs(wl)[0]
    W, X, _ = H.to_dev(li, dtype)
    S = b.score(W, X, KINDS[kind])
    torch.cuda.synchronize()
    ref = O.importance(W.double().cpu().numpy(), X.double().cpu().numpy(), kind)
    tol = 1e-5 if dtype == "f32" else 4e-3      # S is stored in the weights' type
    assert H.relerr(S.float().cpu().numpy(), ref) <= tol


@pytest.mark.parametrize("dtype,flags,B,kind", [
    ("bf16", 0, 64, "wanda"), ("bf16", 0, 32, "ria"), ("bf16", 0, 64, "magnitude"),
    ("bf16", b.FLAG_SIMT, 128, "wanda"), ("f32", 0, 64, "ria"),
])
def test_step_with_scores_matches_the_oracle(gpu_lib, dtype, flags, B, kind):
    wl = synth.custom(264, 512, 160, B, 2, 4, 0.5, 5, dtype, seed=61 + B, outliers=True)
    li = synth.make_inputs(wl)[0]
    W, X, L = H.to_dev(li, dtype)
    d = b.alloc_outputs(W, X, L, with_mask=True, with_wp=True)
    d["S"] = b.score(W, X, KINDS[kind])
    s = b.Step([d], wl.block, wl.n, wl.m, wl.iters, wl.tau, flags=flags | b.FLAG_SCORE | b.FLAG_WRITE_WPRIME)
    s.run()
    torch.cuda.synchronize()
    assert b.device_error() == 0
    Shat = d["Wp"].cpu().numpy()                      # the matrix the mask ranks
    mask_words = d["mask"].cpu().numpy().view(np.uint32)
    mask = O.unpack_mask_bits(mask_words, li.spec.cin)
    Lh = d["L"].cpu().numpy()
    S_stored = d["S"].double().cpu().numpy()
    P_ref, _ = O.sinkhorn(Lh, wl.tau, wl.iters)
    assert H.relerr(d["P"].cpu().numpy(), P_ref) <= H.TOL_P
    Shat_ref = O.permute_weight(S_stored, P_ref)
    assert H.relerr(Shat, Shat_ref) <= 1e-5
    assert np.array_equal(O.pack_mask_bits(O.nm_mask(Shat.astype(np.float32), wl.n, wl.m)), mask_words)
    ref = O.step(li.W, li.X, Lh, wl.tau, wl.iters, wl.n, wl.m, mask=mask)
    tl = H.TOL_LOSS_F32 if dtype == "f32" else H.TOL_LOSS_BF16
    td = H.TOL_DL_F32 if dtype == "f32" else H.TOL_DL_BF16
    assert abs(float(d["loss"][0].cpu()) - ref["loss"]) / ref["loss"] <= tl
    assert H.relerr(d["dL"].cpu().numpy(), ref["dL"]) <= td
    own = O.forward(li.W, li.X, Lh, wl.tau, wl.iters, wl.n, wl.m, score=S_stored)["mask"]
    assert np.mean(own == mask) >= 0.99                # near-ties may flip against float64

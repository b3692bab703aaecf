"""Hardening ([PermLLM] "Method" 2): the GPU's per-block assignment against the
oracle, and whole steps with LCP_FLAG_HARD against the oracle's hardened step.

Where several permutations attain the maximum of Tr(P^T P_hat), any of them is
correct: the tests check that the GPU's permutation is valid and reaches the
oracle's maximum (exactly when the maximum is unique by a wide margin), then
evaluate the oracle's hardened step at the GPU's permutation.
"""
import numpy as np
import pytest
import torch

from learnable_channel_permutation_b200 import binding as b
from learnable_channel_permutation_b200 import synth
from oracle import lcp_oracle as O

import gpu_helpers as H

pytestmark = pytest.mark.gpu


def _gpu_harden(P):
    Pt = torch.from_numpy(np.ascontiguousarray(P, np.float32)).cuda()
    nb, B, _ = P.shape
    perm = torch.empty(nb, B, dtype=torch.int32, device="cuda")
    Ph = torch.empty_like(Pt)
    b.harden(Pt, perm, Ph)
    torch.cuda.synchronize()
    assert b.device_error() == 0
    return perm.cpu().numpy().astype(np.int64), Ph.cpu().numpy()


def _check_valid(perm, Ph):
    nb, B = perm.shape
    for k in range(nb):
        assert sorted(perm[k]) == list(range(B))
    assert np.array_equal(Ph, O.perm_matrix(perm))


@pytest.mark.parametrize("B", [32, 64, 128, 256])
@pytest.mark.parametrize("kind", ["spread", "init_scale", "peaked", "few_large"])
def test_harden_reaches_the_maximum(gpu_lib, B, kind):
    rng = np.random.default_rng(B + len(kind))
    nb = 6
    if kind == "few_large":
        # a wide range (0 .. 0.6) but a maximum near 2, set by many near-tied small entries
        P = rng.uniform(0, 1e-3, (nb, B, B))
        for k in range(nb):
            P[k].flat[rng.choice(B * B, size=4, replace=False)] = rng.uniform(0.3, 0.6, 4)
        P = P.astype(np.float32)
    elif kind == "peaked":
        pis = np.stack([rng.permutation(B) for _ in range(nb)])
        P = (0.7 * O.perm_matrix(pis) + 0.3 / B + rng.uniform(0, 1e-4, (nb, B, B))).astype(np.float32)
    else:
        sd = 1.0 if kind == "spread" else 1e-3
        Lt = torch.from_numpy(rng.normal(0, sd, (nb, B, B)).astype(np.float32)).cuda()
        Pt = torch.empty_like(Lt)
        b.sinkhorn_fwd(Lt, Pt, None, 0.5, 5)
        P = Pt.cpu().numpy()
    perm, Ph = _gpu_harden(P)
    _check_valid(perm, Ph)
    P64 = P.astype(np.float64)
    best = O.assignment_value(P64, O.harden(P64))
    got = O.assignment_value(P64, perm)
    assert np.all(got >= best - 1e-5 * np.maximum(1.0, np.abs(best))), (got, best)
    if kind == "peaked":
        assert np.array_equal(perm, pis)


def test_harden_all_ties_gives_a_permutation(gpu_lib):
    P = np.full((3, 64, 64), 1.0 / 64, np.float32)
    perm, Ph = _gpu_harden(P)
    _check_valid(perm, Ph)


def _run_hard(wl, flags=0):
    li = synth.make_inputs(wl)[0]
    W, X, L = H.to_dev(li, wl.dtype)
    d = b.alloc_outputs(W, X, L, with_mask=True, with_wp=True)
    nb = li.spec.cin // wl.block
    d["perm"] = torch.full((nb, wl.block), -1, dtype=torch.int32, device="cuda")
    s = b.Step([d], wl.block, wl.n, wl.m, wl.iters, wl.tau, flags=flags | b.FLAG_HARD | b.FLAG_WRITE_WPRIME)
    s.run()
    torch.cuda.synchronize()
    assert b.device_error() == 0
    g = dict(P=d["P"].cpu().numpy(), dL=d["dL"].cpu().numpy(), loss=float(d["loss"][0].cpu()),
             mask_words=d["mask"].cpu().numpy().view(np.uint32), Wp=d["Wp"].cpu().numpy(),
             perm=d["perm"].cpu().numpy().astype(np.int64), L=d["L"].cpu().numpy())
    g["mask"] = O.unpack_mask_bits(g["mask_words"], li.spec.cin)
    return li, g


@pytest.mark.parametrize("dtype,flags,B,n,m", [
    ("bf16", 0, 64, 2, 4), ("bf16", 0, 32, 2, 4), ("bf16", 0, 128, 4, 8), ("bf16", 0, 256, 2, 4),
    ("bf16", b.FLAG_SIMT, 64, 2, 4), ("f32", 0, 64, 2, 4),
])
def test_step_hard_matches_the_oracle(gpu_lib, dtype, flags, B, n, m):
    wl = synth.custom(264, 512, 160, B, n, m, 0.5, 5, dtype, seed=21 + B, outliers=True)
    li, g = _run_hard(wl, flags)
    L = g["L"]
    P_ref, _ = O.sinkhorn(L, wl.tau, wl.iters)
    assert H.relerr(g["P"], P_ref) <= H.TOL_P                       # layer.P is the soft P_hat
    perm = g["perm"]
    _check_valid(perm, O.perm_matrix(perm))
    best = O.assignment_value(P_ref, O.harden(P_ref))
    assert np.all(O.assignment_value(P_ref, perm) >= best - 1e-5)
    ref = O.step_hard(li.W, li.X, L, wl.tau, wl.iters, wl.n, wl.m, perm=perm)
    # a hard permutation makes W' an exact column gather, so W' and the mask are exact
    assert np.array_equal(g["Wp"].astype(np.float64), ref["Wp"])
    assert np.array_equal(g["mask"], ref["mask"])
    tl = H.TOL_LOSS_F32 if dtype == "f32" else H.TOL_LOSS_BF16
    td = H.TOL_DL_F32 if dtype == "f32" else H.TOL_DL_BF16
    assert abs(g["loss"] - ref["loss"]) / abs(ref["loss"]) <= tl
    assert H.relerr(g["dL"], ref["dL"]) <= td
    if dtype == "bf16":
        assert H.cosine(g["dL"], ref["dL"]) >= H.COS_DL_BF16

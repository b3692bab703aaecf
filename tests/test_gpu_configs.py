"""GPU parity on every workload configuration at its full size, in the launch
configuration the benchmark uses: the MLP of a 7B layer (gate/up 11008 x 4096,
down 4096 x 11008 with ReLU-like input, T = 2048), points of the block-size /
iteration / temperature / N:M sweep on 4096 x 4096 (T = 2048), and the seven
projections of a 13B layer in one lcp_step call (T = 4096).

Every layer is compared with the float64 oracle: P; the mask bit-exactly
against the oracle's mask of the GPU's own W' (sampled rows); the loss and the
mask-conditioned dL (the oracle is given the GPU's mask) under the bounds of
tests/tolerances.py; and exact invariants (every row of dL_b sums to zero, N
kept per group).  The whole 1024 x 1024 sweep grid runs against the oracle too.
"""
import numpy as np
import pytest

from learnable_channel_permutation_b200 import synth
from oracle import lcp_oracle as O

import gpu_helpers as H

pytestmark = pytest.mark.gpu


def _check_full_size(wl, inputs, out, rng, sample_rows=128):
    errs = []
    for li, g in zip(inputs, out):
        P_ref, _ = O.sinkhorn(g["L"], wl.tau, wl.iters)
        assert H.relerr(g["P"], P_ref) <= H.TOL_P
        cout, cin = li.W.shape
        rows = np.sort(rng.choice(cout, size=min(sample_rows, cout), replace=False))
        Wp = g["Wp"][rows].astype(np.float32)
        assert np.array_equal(O.pack_mask_bits(O.nm_mask(Wp, wl.n, wl.m)), g["mask_words"][rows])
        assert H.relerr(Wp, O.permute_weight(li.W[rows].astype(np.float64), P_ref)) <= 1e-5
        assert np.all(g["mask"].reshape(cout, -1, wl.m).sum(axis=2) == wl.n)
        dL = g["dL"]
        assert np.max(np.abs(dL.sum(axis=2))) <= 1e-4 * max(np.max(np.abs(dL)), 1e-30) * wl.block
        assert np.isfinite(dL).all()
        # the full float64 oracle, conditioned on the GPU's mask
        ref = O.step(li.W, li.X, g["L"], wl.tau, wl.iters, wl.n, wl.m, mask=g["mask"])
        tol_dl, cos_dl = H.dl_bounds(li.spec)
        e = dict(layer=li.spec.name, loss=abs(g["loss"] - ref["loss"]) / abs(ref["loss"]),
                 dL=H.relerr(dL, ref["dL"]), dL_cos=H.cosine(dL, ref["dL"]))
        assert e["loss"] <= H.TOL_LOSS_BF16, e
        assert e["dL"] <= tol_dl, e
        assert e["dL_cos"] >= cos_dl, e
        errs.append(e)
        del ref
    return errs


def _run_full(wl, seed, sample_rows=128):
    inputs = synth.make_inputs(wl)
    out, _ = H.run_gpu(wl, inputs)
    errs = _check_full_size(wl, inputs, out, np.random.default_rng(seed), sample_rows)
    print(wl.name, errs)


@pytest.mark.slow
def test_mlp_7b_full_size_against_the_oracle(gpu_lib):
    _run_full(synth.mlp_7b(), 3)


@pytest.mark.slow
def test_block_13b_full_size_against_the_oracle(gpu_lib):
    """Seven layers in one lcp_step call; T = 4096 is the gradient GEMM's longest K."""
    _run_full(synth.block_13b(), 5, sample_rows=64)


@pytest.mark.slow
@pytest.mark.parametrize("B,iters,tau,nm", [(32, 5, 1.0, (2, 4)), (128, 5, 1.0, (2, 4)), (256, 5, 1.0, (2, 4)),
                                            (64, 20, 0.1, (4, 8)), (256, 20, 0.1, (2, 4)), (32, 20, 0.1, (4, 8))])
def test_sweep_point_full_size_against_the_oracle(gpu_lib, B, iters, tau, nm):
    """Points of the sweep on its 4096 x 4096, T = 2048 layer (the headline
    point B = 64, 5 iterations, tau 0.5, 2:4 is test_gpu_parity's)."""
    _run_full(synth.sweep_4096(B, iters, tau, nm[0], nm[1]), B + iters)


@pytest.mark.parametrize("B", [32, 64, 128, 256])
@pytest.mark.parametrize("iters", [5, 20])
@pytest.mark.parametrize("tau", [1.0, 0.1])
@pytest.mark.parametrize("nm", [(2, 4), (4, 8)])
def test_sweep_point_reduced(gpu_lib, B, iters, tau, nm):
    """Every point of the block-size / iteration / temperature / N:M sweep on a
    1024 x 1024 layer with 192 tokens, against the float64 oracle."""
    n, m = nm
    wl = synth.custom(1024, 1024, 192, B, n, m, tau, iters, "bf16", seed=B + iters)
    inputs = synth.make_inputs(wl)
    out, _ = H.run_gpu(wl, inputs)
    for li, g in zip(inputs, out):
        H.check_layer(li, wl, g, H.TOL_LOSS_BF16, H.TOL_DL_BF16, H.COS_DL_BF16)

"""GPU parity on every workload configuration: the MLP pair of a 7B layer, the
block-size / iteration / temperature / N:M sweep, and the 7 projections of a
13B layer in one lcp_step call.

Full-size runs (the launch configuration the benchmark uses) are checked on
what the oracle can afford at that size: P (it does not depend on X), the mask
bit-exactly against the oracle's mask of the GPU's own W' on sampled rows,
exact invariants (every row of dL_b sums to zero, N kept per group, the loss
in [0, 2]).  The same layers with the token count cut to a few hundred are
then compared with the full float64 oracle (loss and mask-conditioned dL).
"""
import numpy as np
import pytest

from learnable_channel_permutation_b200 import synth
from oracle import lcp_oracle as O

import gpu_helpers as H

pytestmark = pytest.mark.gpu


def _check_full_size(wl, inputs, out, rng, sample_rows=64):
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
        assert 0.0 <= g["loss"] <= 2.0 and np.isfinite(dL).all()


def _reduced(wl, tokens):
    layers = [synth.LayerSpec(s.name, s.cout, s.cin, tokens, s.x_key, s.w_outliers, s.x_outliers, s.x_kind)
              for s in wl.layers]
    return synth.Workload(wl.name + f"_T{tokens}", layers, wl.block, wl.n, wl.m, wl.tau, wl.iters, wl.dtype,
                          wl.seed)


def _check_reduced(wl):
    inputs = synth.make_inputs(wl)
    out, _ = H.run_gpu(wl, inputs)
    for li, g in zip(inputs, out):
        H.check_layer(li, wl, g, H.TOL_LOSS_BF16, H.TOL_DL_BF16, H.COS_DL_BF16,
                      agreement=li.W.size <= 4096 * 4096)


@pytest.mark.slow
def test_mlp_7b_full_size_and_reduced_tokens(gpu_lib):
    wl = synth.mlp_7b()
    inputs = synth.make_inputs(wl)
    out, _ = H.run_gpu(wl, inputs)
    _check_full_size(wl, inputs, out, np.random.default_rng(3))
    _check_reduced(_reduced(wl, 256))


@pytest.mark.slow
def test_block_13b_full_size_and_reduced_tokens(gpu_lib):
    wl = synth.block_13b()
    inputs = synth.make_inputs(wl)
    out, _ = H.run_gpu(wl, inputs)
    _check_full_size(wl, inputs, out, np.random.default_rng(5), sample_rows=32)
    _check_reduced(_reduced(wl, 128))


@pytest.mark.parametrize("B", [32, 64, 128, 256])
@pytest.mark.parametrize("iters", [5, 20])
@pytest.mark.parametrize("tau", [1.0, 0.1])
@pytest.mark.parametrize("nm", [(2, 4), (4, 8)])
def test_sweep_point_reduced(gpu_lib, B, iters, tau, nm):
    """Every point of the block-size / iteration / temperature / N:M sweep on a
    1024 x 1024 layer with 192 tokens, against the float64 oracle."""
    n, m = nm
    wl = synth.custom(1024, 1024, 192, B, n, m, tau, iters, "bf16", seed=B + iters)
    _check_reduced(wl)


@pytest.mark.parametrize("B", [32, 128, 256])
def test_sweep_block_sizes_full_size(gpu_lib, B):
    """The sweep's 4096 x 4096, T = 2048 layer at the other block sizes, full size."""
    wl = synth.sweep_4096(B, 5, 1.0, 2, 4)
    inputs = synth.make_inputs(wl)
    out, _ = H.run_gpu(wl, inputs)
    _check_full_size(wl, inputs, out, np.random.default_rng(B))

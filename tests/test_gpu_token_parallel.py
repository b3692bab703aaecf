"""GPU: the token-parallel split of one layer on one GPU.  Two token shards run
through lcp_step_shard (mean over the global token count, stopping before the
Sinkhorn reverse pass); their dP and losses are summed and lcp_sinkhorn_bwd
finishes the step.  The result is compared with the whole batch's oracle and
with lcp_step on the whole batch."""
import numpy as np
import pytest
import torch

from learnable_channel_permutation_b200 import binding as b
from learnable_channel_permutation_b200 import parallel, synth
from oracle import lcp_oracle as O

import gpu_helpers as H

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,flags", [("bf16", 0), ("bf16", b.FLAG_SIMT), ("f32", 0)])
def test_two_token_shards_sum_to_the_whole_batch(gpu_lib, dtype, flags):
    T = 203
    wl = synth.custom(136, 256, T, 64, 2, 4, 0.5, 5, dtype, seed=21, outliers=True)
    (li,) = synth.make_inputs(wl)
    W, X, L = H.to_dev(li, dtype)
    whole = b.alloc_outputs(W, X, L)
    b.Step([whole], wl.block, wl.n, wl.m, wl.iters, wl.tau, flags=flags).run()
    dPs, cks, losses, masks = [], [], [], []
    for r in range(2):
        sl = parallel.token_shard(T, r, 2)
        d = b.alloc_outputs(W, X[sl].contiguous(), L)
        st = b.Step([d], wl.block, wl.n, wl.m, wl.iters, wl.tau, flags=flags)
        dP, ck = torch.empty_like(L), torch.empty(L.shape[0], wl.iters, 2, wl.block, device="cuda")
        b.step_shard(st, T, [dP], [ck])
        dPs.append(dP); cks.append(ck); losses.append(d["loss"][:1]); masks.append(d["mask"])
    dL = torch.empty_like(L)
    b.sinkhorn_bwd(L, cks[0], dPs[0] + dPs[1], dL, wl.tau, wl.iters)
    torch.cuda.synchronize()
    assert b.device_error() == 0
    assert torch.equal(cks[0], cks[1]) and torch.equal(masks[0], masks[1]) and torch.equal(masks[0], whole["mask"])
    loss = float(losses[0] + losses[1])
    assert abs(loss - float(whole["loss"][0])) <= 1e-5 * abs(float(whole["loss"][0]))
    mask = O.unpack_mask_bits(whole["mask"].cpu().numpy().view(np.uint32), li.spec.cin)
    ref = O.step(li.W, li.X, li.L, wl.tau, wl.iters, wl.n, wl.m, mask=mask)
    tol_dl, cos_dl = H.dl_bounds(li.spec, dtype)
    got = dL.cpu().numpy()
    assert abs(loss - ref["loss"]) <= (H.TOL_LOSS_F32 if dtype == "f32" else H.TOL_LOSS_BF16) * abs(ref["loss"])
    assert H.relerr(got, ref["dL"]) <= tol_dl
    if cos_dl is not None:
        assert H.cosine(got, ref["dL"]) >= cos_dl
    # the whole-batch step of the same path: equal up to the rounding of the two shards' products
    assert H.relerr(got, whole["dL"].cpu().numpy()) <= (1e-5 if dtype == "f32" else 1e-2)

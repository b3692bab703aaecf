"""AdamW on the logits and the training loop with the linear temperature
schedule ([PermLLM] "Implementation details"), GPU against the oracle."""
import numpy as np
import pytest
import torch

from learnable_channel_permutation_b200 import binding as b
from learnable_channel_permutation_b200 import synth
from oracle import lcp_oracle as O

import gpu_helpers as H

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("t", [1, 2, 50])
def test_adamw_matches_oracle(gpu_lib, t):
    rng = np.random.default_rng(40 + t)
    shape = (8, 64, 64)
    L0 = rng.normal(0, 1e-2, shape).astype(np.float32)
    g = rng.normal(0, 1e-3, shape).astype(np.float32)
    m0 = (rng.normal(0, 1e-4, shape) if t > 1 else np.zeros(shape)).astype(np.float32)
    v0 = (np.abs(rng.normal(0, 1e-7, shape)) if t > 1 else np.zeros(shape)).astype(np.float32)
    L, dL, m, v = (torch.from_numpy(a.copy()).cuda() for a in (L0, g, m0, v0))
    opt = b.adamw_params(lr=5e-3, weight_decay=0.01)
    b.adamw(L, dL, m, v, opt, t)
    torch.cuda.synchronize()
    Lr, mr, vr = O.adamw_update(L0, g, m0, v0, t, lr=5e-3, weight_decay=0.01)
    assert H.relerr(m.cpu().numpy(), mr) <= 1e-6
    assert H.relerr(v.cpu().numpy(), vr) <= 1e-6
    assert H.relerr(L.cpu().numpy() - L0, Lr - L0) <= 1e-5     # the update itself, not just L


def _trainer(wl, total, lr, flags=0):
    li = synth.make_inputs(wl)[0]
    W, X, L = H.to_dev(li, wl.dtype)
    d = b.alloc_outputs(W, X, L)
    s = b.Step([d], wl.block, wl.n, wl.m, wl.iters, 1.0, flags=flags)
    return li, d, b.Trainer(s, b.adamw_params(lr=lr), total)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_train_steps_follow_the_schedule_and_adamw(gpu_lib, dtype):
    """Steps one call at a time: each step's loss is the oracle's step at the
    scheduled temperature and the current logits, and each update is AdamW of
    that step's dL (the GPU's own: comparing whole Adam trajectories would
    amplify last-bit dL differences through the normalisation m / sqrt(v))."""
    wl = synth.toy_256() if dtype == "f32" else synth.custom(256, 512, 160, 64, 2, 4, 1.0, 5, "bf16", seed=6,
                                                              outliers=True)
    total, lr = 5, 5e-3
    li, d, tr = _trainer(wl, total, lr)
    L = d["L"].cpu().numpy().astype(np.float64)
    m = np.zeros_like(L)
    v = np.zeros_like(L)
    tl = H.TOL_LOSS_F32 if dtype == "f32" else H.TOL_LOSS_BF16
    for s_ in range(total):
        tr.run(s_, 1)
        torch.cuda.synchronize()
        tau = O.tau_schedule(s_, total)
        ref = O.step(li.W, li.X, L, tau, wl.iters, wl.n, wl.m)
        assert abs(float(d["loss"][0].cpu()) - ref["loss"]) / ref["loss"] <= tl, s_
        g = d["dL"].cpu().numpy().astype(np.float64)
        L_next, m, v = O.adamw_update(L, g, m, v, s_ + 1, lr=lr)
        got = d["L"].cpu().numpy().astype(np.float64)
        assert H.relerr(got - L, L_next - L) <= 1e-5, s_
        L = got
    assert b.device_error() == 0


def test_train_split_into_calls_equals_one_call(gpu_lib):
    """run(0, 2) + run(2, 2) enqueues exactly what run(0, 4) does."""
    wl = synth.custom(256, 512, 192, 64, 2, 4, 1.0, 5, "bf16", seed=3, outliers=True)
    _, d1, tr1 = _trainer(wl, 4, 1e-3)
    _, d2, tr2 = _trainer(wl, 4, 1e-3)
    tr1.run(0, 4)
    tr2.run(0, 2)
    tr2.run(2, 2)
    torch.cuda.synchronize()
    for k in ("L", "dL", "P"):
        assert torch.equal(d1[k], d2[k]), k


def test_train_bf16_lowers_the_loss(gpu_lib):
    """Twenty bf16 steps on a layer with outlier channels: the loss goes down and
    the first step is the plain step at tau = 1."""
    wl = synth.custom(512, 1024, 256, 64, 2, 4, 1.0, 5, "bf16", seed=4, outliers=True)
    li, d, tr = _trainer(wl, 20, 5e-3)
    L0 = d["L"].cpu().numpy().copy()
    tr.run(0, 1)
    torch.cuda.synchronize()
    first = float(d["loss"][0].cpu())
    ref = O.step(li.W, li.X, L0, 1.0, wl.iters, wl.n, wl.m)
    assert abs(first - ref["loss"]) / ref["loss"] <= H.TOL_LOSS_BF16
    tr.run(1, 19)
    torch.cuda.synchronize()
    assert b.device_error() == 0
    assert float(d["loss"][0].cpu()) < first

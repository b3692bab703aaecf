"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
on seeded inputs and compare with the CPU oracle."""
import numpy as np
import torch

from learnable_channel_permutation_b200 import binding as b
from oracle import lcp_oracle as O

from tolerances import (TOL_P, TOL_LOSS_F32, TOL_LOSS_BF16, TOL_DL_F32, TOL_DL_BF16, COS_DL_BF16,  # noqa: F401
                        TOL_DL_BF16_RELU, COS_DL_BF16_RELU, dl_bounds)


def relerr(a, b_):
    a = np.asarray(a, np.float64)
    b_ = np.asarray(b_, np.float64)
    return float(np.linalg.norm(a - b_) / max(np.linalg.norm(b_), 1e-300))


def cosine(a, b_):
    a = np.asarray(a, np.float64).ravel()
    b_ = np.asarray(b_, np.float64).ravel()
    return float(a @ b_ / (np.linalg.norm(a) * np.linalg.norm(b_)))


def to_dev(li, dtype):
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    W = torch.from_numpy(li.W).to("cuda").to(tdt).contiguous()
    X = torch.from_numpy(li.X).to("cuda").to(tdt).contiguous()
    L = torch.from_numpy(li.L).to("cuda").contiguous()
    return W, X, L


def run_gpu(wl, inputs, flags=0, with_wp=True, L_override=None):
    """One lcp_step over every layer of ``wl``; returns per-layer numpy outputs."""
    dev = []
    xcache = {}
    for i, li in enumerate(inputs):
        key = li.spec.x_key
        W, X, L = to_dev(li, wl.dtype)
        if key in xcache:
            X = xcache[key]          # layers that share X share one device buffer
        xcache[key] = X
        if L_override is not None:
            L = torch.from_numpy(np.ascontiguousarray(L_override[i], np.float32)).cuda()
        d = b.alloc_outputs(W, X, L, with_mask=True, with_wp=with_wp)
        dev.append(d)
    f = flags | (b.FLAG_WRITE_WPRIME if with_wp else 0)
    s = b.Step(dev, wl.block, wl.n, wl.m, wl.iters, wl.tau, flags=f)
    s.run()
    torch.cuda.synchronize()
    assert b.device_error() == 0, "a bounded wait inside a tensor-core kernel expired"
    out = []
    for d in dev:
        cout, cin = d["W"].shape
        r = dict(P=d["P"].cpu().numpy(), dL=d["dL"].cpu().numpy(), loss=float(d["loss"][0].cpu()),
                 mask_words=d["mask"].cpu().numpy().view(np.uint32),
                 L=d["L"].cpu().numpy())
        r["mask"] = O.unpack_mask_bits(r["mask_words"], cin)
        if with_wp:
            r["Wp"] = d["Wp"].cpu().numpy()
        out.append(r)
    return out, s


def check_layer(li, wl, g, tol_loss, tol_dl, cos_dl=None, check_wp=True, agreement=True):
    """Compare one GPU layer result ``g`` with the oracle; returns a dict of errors."""
    L = g["L"]
    # P (Sinkhorn) against the oracle
    P_ref, _ = O.sinkhorn(L, wl.tau, wl.iters)
    e = dict(P=relerr(g["P"], P_ref))
    assert e["P"] <= TOL_P, e
    # mask: bit-exact against the oracle's mask of the GPU's own W'
    if check_wp and "Wp" in g:
        Wp = g["Wp"].astype(np.float32)
        assert np.array_equal(O.pack_mask_bits(O.nm_mask(Wp, wl.n, wl.m)), g["mask_words"])
        Wp_ref = O.permute_weight(li.W.astype(np.float64), P_ref)
        e["Wp"] = relerr(Wp, Wp_ref)
        assert e["Wp"] <= 1e-5, e
    # loss and dL: mask-conditioned oracle (the GPU's mask injected)
    ref = O.step(li.W, li.X, L, wl.tau, wl.iters, wl.n, wl.m, mask=g["mask"])
    e["loss"] = abs(g["loss"] - ref["loss"]) / abs(ref["loss"])
    e["dL"] = relerr(g["dL"], ref["dL"])
    e["dL_cos"] = cosine(g["dL"], ref["dL"])
    assert e["loss"] <= tol_loss, e
    assert e["dL"] <= tol_dl, e
    if cos_dl is not None:
        assert e["dL_cos"] >= cos_dl, e
    # unconditioned: agreement of the GPU mask with the float64 oracle's mask
    if agreement:
        e["mask_agree"] = float(np.mean(O.nm_mask(O.permute_weight(li.W.astype(np.float64), P_ref), wl.n, wl.m)
                                        == g["mask"]))
    return e

"""Writes the stored expected values under tests/golden/ from the CPU oracle only.

Run from the repository root:  python tests/golden/make_golden.py
Every value written here comes from ``oracle.lcp_oracle`` applied to inputs of
``learnable_channel_permutation_b200.synth``; nothing comes from the CUDA path.
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import lcp_oracle as O  # noqa: E402
from learnable_channel_permutation_b200 import synth  # noqa: E402


def toy_case():
    wl = synth.custom(cout=16, cin=64, tokens=24, block=32, n=2, m=4, tau=0.5, iters=5,
                      dtype="f32", seed=7, name="golden_toy")
    (li,) = synth.make_inputs(wl)
    # widen the logits so that P is far from uniform and the gradient informative
    L = (li.L.astype(np.float64) * 300.0).astype(np.float32)
    out = O.step(li.W, li.X, L, wl.tau, wl.iters, wl.n, wl.m)
    return dict(
        source="oracle.lcp_oracle.step on synth.custom(16x64, T=24, B=32, 2:4, tau=0.5, 5 iters, f32, seed 7),"
               " logits scaled by 300",
        cout=16, cin=64, tokens=24, block=32, n=2, m=4, tau=0.5, iters=5, seed=7, logit_scale=300.0,
        loss=repr(float(out["loss"])),
        P=[repr(float(v)) for v in out["P"].ravel()],
        dL=[repr(float(v)) for v in out["dL"].ravel()],
        mask_words=[int(v) for v in O.pack_mask_bits(out["mask"]).ravel()],
    )


if __name__ == "__main__":
    with open(os.path.join(HERE, "toy_step.json"), "w") as f:
        json.dump(toy_case(), f, indent=0)
    print("wrote", os.path.join(HERE, "toy_step.json"))

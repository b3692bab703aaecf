"""The stored toy fixture, and the named workloads' settings.

The toy fixture (tests/golden/toy_step.json, written by make_golden.py from the
oracle) is checked two ways: the oracle replays it bit for bit, which guards
against regressions only; and an independent float64 restatement of the pages'
forward equations differentiated by torch autograd (tests/autograd_reference.py)
reproduces its loss, P, mask and dL within rounding, which pins the stored
values, the oracle's hand-written reverse pass included, to something other
than the oracle.
"""
import json
import os

import numpy as np

from oracle import lcp_oracle as O
from learnable_channel_permutation_b200 import synth

import autograd_reference as AR

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _toy():
    g = json.load(open(os.path.join(HERE, "toy_step.json")))
    wl = synth.custom(cout=g["cout"], cin=g["cin"], tokens=g["tokens"], block=g["block"], n=g["n"],
                      m=g["m"], tau=g["tau"], iters=g["iters"], dtype="f32", seed=g["seed"])
    (li,) = synth.make_inputs(wl)
    L = (li.L.astype(np.float64) * g["logit_scale"]).astype(np.float32)
    return g, wl, li, L


def test_toy_fixture_matches_an_autograd_restatement():
    g, wl, li, L = _toy()
    ref = AR.autograd_step(li.W, li.X, L, wl.tau, wl.iters, wl.n, wl.m)
    assert ref["gap"] > 1e-9          # the two W' agree to ~1e-16: rounding cannot flip the mask
    P = np.array([float(v) for v in g["P"]]).reshape(ref["P"].shape)
    dL = np.array([float(v) for v in g["dL"]]).reshape(ref["dL"].shape)
    assert abs(float(g["loss"]) - ref["loss"]) <= 1e-12 * abs(ref["loss"])
    assert np.max(np.abs(P - ref["P"])) <= 1e-13
    assert O.pack_mask_bits(ref["mask"]).ravel().tolist() == g["mask_words"]
    assert np.linalg.norm(dL - ref["dL"]) <= 1e-12 * np.linalg.norm(ref["dL"])


def test_oracle_replays_toy_fixture_bit_for_bit():
    g, wl, li, L = _toy()
    out = O.step(li.W, li.X, L, wl.tau, wl.iters, wl.n, wl.m)
    assert float(out["loss"]) == float(g["loss"])
    assert np.array_equal(out["P"].ravel(), np.array([float(v) for v in g["P"]]))
    assert np.array_equal(out["dL"].ravel(), np.array([float(v) for v in g["dL"]]))
    assert O.pack_mask_bits(out["mask"]).ravel().tolist() == g["mask_words"]


def test_headline_workload_uses_the_papers_settings():
    h = json.load(open(os.path.join(HERE, "pages_hparams.json")))
    wl = synth.q_proj_4096()
    assert wl.block == h["block_size_paper"] and wl.iters == h["sinkhorn_iterations_paper"]
    assert (wl.n, wl.m) == (2, 4)
    assert h["temperature_schedule"][1] <= wl.tau <= h["temperature_schedule"][0]


def test_synth_is_deterministic_and_bf16_exact():
    wl = synth.custom(64, 128, 40, 32, 2, 4, 0.5, 5, "bf16", seed=3, outliers=True)
    a, b = synth.make_inputs(wl)[0], synth.make_inputs(wl)[0]
    assert np.array_equal(a.W, b.W) and np.array_equal(a.X, b.X) and np.array_equal(a.L, b.L)
    synth.bf16_bits(a.W)
    synth.bf16_bits(a.X)
    assert a.outlier_channels.size == 1
    c = a.outlier_channels[0]
    assert np.std(a.W[:, c]) > 4 * np.std(np.delete(a.W, c, axis=1))


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2**-8, 1.0 + 3 * 2**-8, 1.0 + 2**-9, -2.5, 0.0], np.float32)
    r = synth.bf16_round(x)
    assert r.tolist() == [1.0, 1.0, 1.0 + 2**-6, 1.0, -2.5, 0.0]

"""Seeded synthetic inputs shared by the CUDA path, the oracle and the benchmark.

This module draws random numbers and rounds them to the storage precision of
the workload; it holds none of the arithmetic of the learnable channel
permutation itself (no Sinkhorn, no permutation, no mask, no loss).  Both the
GPU path and the CPU oracle consume exactly the arrays produced here.

Recipe (every workload):

* ``numpy.random.Generator(PCG64)`` seeded with ``SeedSequence([seed, layer,
  stream])``; stream 0 draws W, 1 draws X, 2 draws the logits L, 3 chooses
  the outlier input channels.  Layers that share an activation matrix (the
  gate/up pair, or every attention projection of one block) share the X
  stream of the first layer that uses it.
* W ~ N(0, 0.02), X ~ N(0, 1) (or max(0, N(0, 1)) for the input of a down
  projection where the workload says "ReLU-like"), L ~ N(0, 1e-3) with 1e-3
  read as a standard deviation (the PermLLM blog page, section 6, advises
  std 1e-3 for the permutation initialisation).
* Outlier channels: round(0.01 * C_in) input channels, chosen without
  replacement; W[:, c] is scaled by 10 and X[:, c] by 5 before rounding.
* For bf16 workloads the float32 draws are rounded to bf16 with
  round-to-nearest-even; the arrays returned hold those exactly
  representable values in float32, and ``bf16_bits`` gives the raw bits.
* X is stored as [T, C_in] row-major (token-major activations); W as
  [C_out, C_in]; L as [C_in / B, B, B].

The calibration set of the paper (128 C4 samples of 1024 tokens, PermLLM
summary, "Experimental setup") and the LLaMA weights are not available; these
draws stand in for them with the projection shapes of LLaMA-7B/13B.
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional

import numpy as np

STREAM_W, STREAM_X, STREAM_L, STREAM_OUTLIER = 0, 1, 2, 3


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even), kept as float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    nan = np.isnan(x)
    out = r.astype(np.uint32).view(np.float32).copy()
    out[nan] = np.float32("nan")
    return out


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Raw bf16 bit patterns (uint16) of float32 values that are already bf16-exact."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    if np.any(u & 0xFFFF):
        raise ValueError("bf16_bits: values are not bf16-representable; call bf16_round first")
    return (u >> 16).astype(np.uint16)


def _rng(seed: int, layer: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, layer, stream])))


@dataclass
class LayerSpec:
    """One linear layer of a workload: W is [cout, cin]; X is [tokens, cin]."""

    name: str
    cout: int
    cin: int
    tokens: int
    x_key: str                 # layers with the same key share one X
    w_outliers: bool = False
    x_outliers: bool = False
    x_kind: str = "normal"     # "normal" or "halfnormal"


@dataclass
class Workload:
    name: str
    layers: List[LayerSpec]
    block: int
    n: int
    m: int
    tau: float
    iters: int
    dtype: str                 # "f32" or "bf16"
    seed: int = 0
    note: str = ""


@dataclass
class LayerInputs:
    spec: LayerSpec
    W: np.ndarray              # float32 [cout, cin] (bf16-exact for bf16 workloads)
    X: np.ndarray              # float32 [tokens, cin]
    L: np.ndarray              # float32 [cin/B, B, B]
    outlier_channels: np.ndarray = field(default_factory=lambda: np.zeros(0, np.int64))


def _draw_layer(wl: Workload, li: int, spec: LayerSpec, x_cache: Dict[str, np.ndarray]) -> LayerInputs:
    seed = wl.seed
    rw = _rng(seed, li, STREAM_W)
    W = rw.standard_normal((spec.cout, spec.cin), dtype=np.float32) * np.float32(0.02)
    rl = _rng(seed, li, STREAM_L)
    L = rl.standard_normal((spec.cin // wl.block, wl.block, wl.block), dtype=np.float32) * np.float32(1e-3)
    chans = np.zeros(0, np.int64)
    if spec.w_outliers or spec.x_outliers:
        k = int(round(0.01 * spec.cin))
        chans = np.sort(_rng(seed, li, STREAM_OUTLIER).choice(spec.cin, size=k, replace=False))
    if spec.w_outliers and chans.size:
        W[:, chans] *= np.float32(10.0)
    if spec.x_key in x_cache:
        X = x_cache[spec.x_key]
    else:
        rx = _rng(seed, li, STREAM_X)
        X = rx.standard_normal((spec.tokens, spec.cin), dtype=np.float32)
        if spec.x_kind == "halfnormal":
            np.maximum(X, 0, out=X)
        elif spec.x_kind != "normal":
            raise ValueError(spec.x_kind)
        if spec.x_outliers and chans.size:
            X[:, chans] *= np.float32(5.0)
        if wl.dtype == "bf16":
            X = bf16_round(X)
        x_cache[spec.x_key] = X
    if wl.dtype == "bf16":
        W = bf16_round(W)
    return LayerInputs(spec, np.ascontiguousarray(W), np.ascontiguousarray(X), np.ascontiguousarray(L), chans)


def make_inputs(wl: Workload) -> List[LayerInputs]:
    """Draw every layer of a workload (deterministic in ``wl.seed``)."""
    cache: Dict[str, np.ndarray] = {}
    return [_draw_layer(wl, i, s, cache) for i, s in enumerate(wl.layers)]


# --------------------------------------------------------------------------
# Named workloads (shapes of LLaMA-7B / 13B projections, plus a toy layer).
# --------------------------------------------------------------------------

def toy_256() -> Workload:
    """Toy fp32 layer: W 256x256, X with 128 tokens, B=64, tau 1, 5 iterations, 2:4."""
    return Workload("toy_256", [LayerSpec("toy", 256, 256, 128, "x")], block=64, n=2, m=4,
                    tau=1.0, iters=5, dtype="f32")


def q_proj_4096(tokens: int = 2048) -> Workload:
    """LLaMA-7B q_proj shape: W 4096x4096 bf16 with 1% outlier input channels, T=2048."""
    return Workload("q_proj_4096", [LayerSpec("q_proj", 4096, 4096, tokens, "x", True, True)],
                    block=64, n=2, m=4, tau=0.5, iters=5, dtype="bf16")


def mlp_7b(tokens: int = 2048) -> Workload:
    """LLaMA-7B MLP: gate/up 11008x4096 share X; down 4096x11008 with a half-normal input."""
    return Workload("mlp_7b", [
        LayerSpec("gate_proj", 11008, 4096, tokens, "x4096"),
        LayerSpec("up_proj", 11008, 4096, tokens, "x4096"),
        LayerSpec("down_proj", 4096, 11008, tokens, "x11008", x_kind="halfnormal"),
    ], block=64, n=2, m=4, tau=0.5, iters=5, dtype="bf16")


def sweep_4096(block: int, iters: int, tau: float, n: int, m: int, tokens: int = 2048) -> Workload:
    """Block-size / iteration sweep point on W 4096x4096 (no outliers)."""
    return Workload(f"sweep_4096_B{block}_it{iters}_tau{tau:g}_{n}of{m}",
                    [LayerSpec("w", 4096, 4096, tokens, "x")],
                    block=block, n=n, m=m, tau=tau, iters=iters, dtype="bf16")


def block_13b(tokens: int = 4096) -> Workload:
    """LLaMA-13B block: q/k/v/o 5120^2, gate/up 13824x5120, down 5120x13824, T=4096, W outliers."""
    L = [LayerSpec(nm, 5120, 5120, tokens, "x5120", True) for nm in ("q_proj", "k_proj", "v_proj", "o_proj")]
    L += [LayerSpec(nm, 13824, 5120, tokens, "x5120", True) for nm in ("gate_proj", "up_proj")]
    L += [LayerSpec("down_proj", 5120, 13824, tokens, "x13824", True)]
    return Workload("block_13b", L, block=64, n=2, m=4, tau=0.5, iters=5, dtype="bf16")


def custom(cout: int, cin: int, tokens: int, block: int, n: int, m: int, tau: float, iters: int,
           dtype: str, seed: int = 0, outliers: bool = False, name: Optional[str] = None) -> Workload:
    """A single layer of arbitrary shape, used for parity cases with ragged tails."""
    nm = name or f"custom_{cout}x{cin}_T{tokens}_B{block}_{n}of{m}_{dtype}"
    return Workload(nm, [LayerSpec("w", cout, cin, tokens, "x", outliers, outliers)], block=block,
                    n=n, m=m, tau=tau, iters=iters, dtype=dtype, seed=seed)


def sweep_points() -> List[Workload]:
    out = []
    for B in (32, 64, 128, 256):
        for it in (5, 20):
            for tau in (1.0, 0.1):
                for (n, m) in ((2, 4), (4, 8)):
                    out.append(sweep_4096(B, it, tau, n, m))
    return out

"""A CPU model of where the bf16 tensor-core step rounds, used to derive the
tolerance of the bf16 dL comparison (test infrastructure, like the oracle).

Every quantity is computed in float64 from the oracle's exact pieces, except
that it is rounded to bf16 (or float32) exactly where the tensor-core path
stores or feeds a value in that precision:

* P is float32; for W' it is split into two bf16 parts, W' = W P_hi + W P_lo
  (about 2^-17 relative), and W' is float32 (the mask compares float32 W');
* A = M (.) W' is rounded to bf16 before At = A P_hi^T, and At is stored in
  bf16 (the operand of the bf16 calibration GEMM);
* Y_d = X W^T and Y_s = X At^T are float32 accumulations of bf16 operands
  (modelled exactly: their rounding is far below the bf16 roundings);
* G is stored in bf16.  ``g_from_pair`` models the variant in which the
  calibration GEMM stores D = Y_d - Y_s and Y_s in bf16 and G is formed from
  them with the exact per-token statistics;
* dAt = G^T X is stored in bf16;
* the block backward multiplies bf16 operands: dA = dAt P_hi, dW' = M (.) dA
  rounded to bf16, A = M (.) W' in bf16, dP_b = dAt_b^T A_b + W_b^T dW'_b
  (for B = 128 and 256 its W' is W P_hi alone: those kernels have no room for P_lo);
* the Sinkhorn passes are float32 (modelled exactly).

The model returns the mask it took (from its own float32 W'), so the oracle
can be run mask-conditioned on it, exactly as the GPU tests do.
"""

import numpy as np

from learnable_channel_permutation_b200.synth import bf16_round
from oracle import lcp_oracle as O


def bf(x):
    return bf16_round(np.asarray(x, np.float32)).astype(np.float64)


def f32(x):
    return np.asarray(x, np.float32).astype(np.float64)


def block_right(M, P):
    """M P_B for a [rows, nb*B] matrix and blocks P [nb, B, B]."""
    nb, B, _ = P.shape
    out = np.empty_like(M)
    for b in range(nb):
        out[:, b * B:(b + 1) * B] = M[:, b * B:(b + 1) * B] @ P[b]
    return out


def modelled_step(W, X_tokens, L, tau, iters, n, m, g_from_pair=False):
    W = np.asarray(W, np.float64)
    X = np.asarray(X_tokens, np.float64)                      # [T, C_in], bf16-exact
    T = X.shape[0]
    P, trace = O.sinkhorn(L, tau, iters)
    P32 = f32(P)
    P_hi = bf(P32)
    P_lo = bf(P32 - P_hi)
    Wp = f32(block_right(W, P_hi) + block_right(W, P_lo))
    mask = O.nm_mask(Wp.astype(np.float32), n, m)
    A = bf(np.where(mask, Wp, 0.0))
    At = bf(block_right(A, np.transpose(P_hi, (0, 2, 1))))
    Yd = X @ W.T                                              # [T, C_out]
    Ys = X @ At.T
    loss, _ = O.cosine_loss(Yd.T, Ys.T)
    if g_from_pair:
        Dq, Ysq = bf(Yd - Ys), bf(Ys)
        dot = np.sum(Yd * Ys, axis=1, keepdims=True)
        nd = np.sqrt(np.sum(Yd * Yd, axis=1, keepdims=True))
        ns = np.sqrt(np.sum(Ys * Ys, axis=1, keepdims=True))
        c = dot / np.maximum(nd * ns, O.COS_EPS)
        G = -((Dq + Ysq) / np.maximum(nd * ns, O.COS_EPS) - c * Ysq / np.maximum(ns * ns, 1e-300)) / T
    else:
        G = O.cosine_loss_grad(Yd.T, Ys.T).T
    G = bf(G)
    dAt = bf(G.T @ X)                                         # [C_out, C_in]
    dWp = bf(np.where(mask, block_right(dAt, P_hi), 0.0))
    nb, B, _ = P.shape
    Ab = bf(np.where(mask, f32(block_right(W, P_hi)), 0.0)) if B >= 128 else A
    dP = np.empty_like(P)
    for b in range(nb):
        s = slice(b * B, (b + 1) * B)
        dP[b] = dAt[:, s].T @ Ab[:, s] + W[:, s].T @ dWp[:, s]
    dL = O.sinkhorn_backward(trace, P, dP, tau)
    return dict(loss=loss, dL=dL, mask=mask, P=P)


def predicted_errors(W, X_tokens, L, tau, iters, n, m, g_from_pair=False):
    """Normwise dL error, dL cosine and loss error of the modelled bf16 path
    against the float64 oracle run on the model's own mask."""
    mod = modelled_step(W, X_tokens, L, tau, iters, n, m, g_from_pair)
    ref = O.step(W, X_tokens, L, tau, iters, n, m, mask=mod["mask"])
    a, r = mod["dL"].ravel(), ref["dL"].ravel()
    return dict(dL=float(np.linalg.norm(a - r) / np.linalg.norm(r)),
                dL_cos=float(a @ r / (np.linalg.norm(a) * np.linalg.norm(r))),
                loss=abs(mod["loss"] - ref["loss"]) / abs(ref["loss"]))

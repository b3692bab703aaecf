"""Plain CPU oracle of the learnable-channel-permutation (LCP) hot path, in float64.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import or run this module.
It shares no code with the CUDA path: no kernels, no helpers, no tables.

Sources (the web pages the method is taken from):

* [PermLLM]  "PermLLM: Learnable Channel Permutation for N:M Sparse Large
  Language Models" (summary page of arXiv 2510.10136): section "Method",
  subsections 1 (soft permutation relaxation: S_0(X) = exp(X),
  S_i(X) = T_c(T_r(S_{i-1}(X))), P_hat = S_L(W_P / tau)), 3 (block-wise
  permutation: P_B = diag(P_1, ..., P_NB), W_hat_B = W P_B), "optimization
  objective" (L_cos(y, y~) = 1 - y.y~ / (|y| |y~|)) and "integration with
  existing pruning methods" (the mask keeps the best N of every group of M
  consecutive columns, straight-through estimator in the backward pass).
* [Blog]  "PermLLM: dynamic channel permutation for N:M sparse LLMs"
  (intelliparadigm.com): section 2.1 (plain N:M pruning: groups of M, keep the
  N largest |w|, zero the rest) and section 2.2 (Sinkhorn in the log domain,
  row normalisation first, then column normalisation, then exp).

* [PermLLM] "Method", subsection 2 (hardening and gradient approximation):
  in the forward pass the soft P_hat is hardened to the permutation
  P = argmax over permutation matrices of Tr(P^T P_hat) (the Hungarian
  algorithm), and the backward pass takes dP/dP_hat = 1 (straight-through).

* [PermLLM] "Effect on inference acceleration": the deployed layer applies
  the channel permutation to its input at run time (a custom CUDA kernel,
  compared there with PyTorch) and multiplies by the 2:4 sparse weight.

* [PermLLM] "Implementation details": the logits are trained with AdamW
  (learning rate 1e-3 or 5e-3), 5 Sinkhorn iterations, the temperature
  decreasing linearly from 1 to 0.1, block size 64.

Readings where the pages are silent or garbled (each is restated where used):

1. The default forward pass uses the soft P; ``step_hard`` is the hardened
   variant (per block, since P_B is block-diagonal the trace splits by block).
2. The mask score is |W'| with W' = W P_B.
3. The mask is a constant in the backward pass (straight-through).
4. One iteration = a row normalisation followed by a column normalisation.
5. Z_0 = L / tau.
6. Equal magnitudes: the lower channel index is kept first (+0 and -0 tie).
7. Groups are M consecutive input channels of W' (permuted order).
8. Cosine denominator max(|y_d| |y_s|, 1e-8).
9. The loss is the mean over the T tokens (columns of Y).
11. Importance scores (the pages name Wanda and RIA as the pruning metrics S
    of "integration with existing pruning methods" without defining them):
    the published definitions, Wanda S_ij = |W_ij| ||X_j||_2 and RIA
    S_ij = (|W_ij| / sum_k |W_kj| + |W_ij| / sum_k |W_ik|) ||X_j||_2^0.5,
    with X_j the j-th input channel over the calibration tokens.
12. Inference format (the pages give none): the deployed weight is
    A = M (.) (W P_B) for the hard P_B, in permuted column order, kept as the
    two kept entries of every group of four columns (in column order) and
    their positions 0..3 in the group; the positions are packed as 4-bit
    fields (first position in the low two bits) of 32-bit words, eight
    groups a word, group g at bits 4 (g % 8) of word g // 8.  The input side
    is x_pi = P_B^T x, i.e. x_pi[bB + pi_b(i)] = x[bB + i].
10. AdamW is Loshchilov and Hutter's (decoupled weight decay, bias-corrected
    moments) with the usual defaults beta = (0.9, 0.999), eps = 1e-8, decay
    0.01 (the pages give only the learning rate); the linear temperature
    schedule puts 1 at the first step and 0.1 at the last.

Notation follows the pages: W is C_out x C_in, X is the C_in x T matrix of
calibration activations (the callers store it token-major, [T, C_in]; this
module transposes it once at entry), L are the learnable logits of the
C_in / B diagonal blocks of the permutation, each B x B, P_b[i, j] moving
source channel bB+i to permuted slot bB+j.
"""

from __future__ import annotations

from typing import Dict, List, Optional, Tuple

import numpy as np

COS_EPS = 1e-8


# ---------------------------------------------------------------------------
# Sinkhorn normalisation  ([PermLLM] Method 1; [Blog] 2.2)
# ---------------------------------------------------------------------------

def logsumexp(z: np.ndarray, axis: int) -> np.ndarray:
    """log(sum(exp(z))) along ``axis`` with the maximum shifted out (kept dims)."""
    mx = np.max(z, axis=axis, keepdims=True)
    return mx + np.log(np.sum(np.exp(z - mx), axis=axis, keepdims=True))


def sinkhorn(logits: np.ndarray, tau: float, n_iters: int) -> Tuple[np.ndarray, List[np.ndarray]]:
    """Soft block permutations P_b = S_L(L_b / tau) for every block b.

    ``logits`` has shape [nb, B, B].  In the log domain S_0 = exp is applied
    last: starting from Z = L / tau, each of the ``n_iters`` iterations first
    subtracts every row's log-sum-exp (T_r: rows sum to one) and then every
    column's (T_c: columns sum to one); P = exp(Z).

    Returns P and the trace [Z_0, Z after T_r of iteration 1, Z after T_c of
    iteration 1, ...] (2 * n_iters + 1 arrays) that the backward pass replays.
    """
    Z = np.asarray(logits, dtype=np.float64) / float(tau)
    trace = [Z]
    for _ in range(n_iters):
        Z = Z - logsumexp(Z, axis=2)      # T_r: normalise each row i over j
        trace.append(Z)
        Z = Z - logsumexp(Z, axis=1)      # T_c: normalise each column j over i
        trace.append(Z)
    return np.exp(Z), trace


def sinkhorn_backward(trace: List[np.ndarray], P: np.ndarray, dP: np.ndarray, tau: float) -> np.ndarray:
    """Gradient of a scalar loss w.r.t. the logits, given dloss/dP.

    Reverse-mode through P = exp(Z_final) and each normalisation:
    a column step Z' = Z - lse_col(Z) has Jacobian delta_ik - exp(Z'_kj), so
    dZ = dZ' - exp(Z') * colsum(dZ'); a row step likewise with row sums.
    Finally Z_0 = L / tau gives dL = dZ_0 / tau.
    """
    dZ = np.asarray(dP, np.float64) * P
    for s in range(len(trace) - 1, 0, -1):
        Z_after = trace[s]
        if s % 2 == 0:   # column normalisation (T_c)
            dZ = dZ - np.exp(Z_after) * np.sum(dZ, axis=1, keepdims=True)
        else:            # row normalisation (T_r)
            dZ = dZ - np.exp(Z_after) * np.sum(dZ, axis=2, keepdims=True)
    return dZ / float(tau)


# ---------------------------------------------------------------------------
# Block-diagonal permutation  ([PermLLM] Method 3)
# ---------------------------------------------------------------------------

def block_diag(P: np.ndarray) -> np.ndarray:
    """The dense C_in x C_in matrix P_B = diag(P_1, ..., P_NB)."""
    nb, B, _ = P.shape
    out = np.zeros((nb * B, nb * B), dtype=np.float64)
    for b in range(nb):
        out[b * B:(b + 1) * B, b * B:(b + 1) * B] = P[b]
    return out


def permute_weight(W: np.ndarray, P: np.ndarray) -> np.ndarray:
    """W' = W P_B, one block of columns at a time (P_B is zero off the diagonal)."""
    W = np.asarray(W, np.float64)
    nb, B, _ = P.shape
    Wp = np.empty_like(W)
    for b in range(nb):
        Wp[:, b * B:(b + 1) * B] = W[:, b * B:(b + 1) * B] @ P[b]
    return Wp


def permute_inputs(P: np.ndarray, Xc: np.ndarray) -> np.ndarray:
    """Xp = P_B^T X for X given as C_in x T: permuted channel bB+k mixes sources bB+i by P_b[i, k]."""
    nb, B, _ = P.shape
    Xp = np.empty_like(Xc)
    for b in range(nb):
        Xp[b * B:(b + 1) * B, :] = P[b].T @ Xc[b * B:(b + 1) * B, :]
    return Xp


# ---------------------------------------------------------------------------
# N:M magnitude mask  ([Blog] 2.1; [PermLLM] integration with pruning methods)
# ---------------------------------------------------------------------------

def nm_mask(Wp: np.ndarray, n: int, m: int) -> np.ndarray:
    """Boolean mask keeping, in every row, the n largest |W'| of each group of m
    consecutive columns.  Equal magnitudes keep the lower column first.

    The comparison is made in the precision of the array passed in (a float32
    W' is compared as float32).
    """
    rows, cols = Wp.shape
    if cols % m:
        raise ValueError("columns must be a multiple of m")
    mag = np.abs(Wp).reshape(rows, cols // m, m)
    # stable sort of -|w|: largest first, equal keys in index order
    order = np.argsort(-mag, axis=2, kind="stable")
    keep = np.zeros(mag.shape, dtype=bool)
    np.put_along_axis(keep, order[:, :, :n], True, axis=2)
    return keep.reshape(rows, cols)


def pack_mask_bits(mask: np.ndarray) -> np.ndarray:
    """Pack a [rows, cols] boolean mask into uint32 words: bit (j % 32) of word j // 32."""
    rows, cols = mask.shape
    if cols % 32:
        raise ValueError("columns must be a multiple of 32")
    bits = mask.reshape(rows, cols // 32, 32).astype(np.uint64)
    weights = (np.uint64(1) << np.arange(32, dtype=np.uint64))
    return (bits * weights).sum(axis=2).astype(np.uint32)


def unpack_mask_bits(words: np.ndarray, cols: int) -> np.ndarray:
    words = np.asarray(words, np.uint32)
    rows = words.shape[0]
    shifts = np.arange(32, dtype=np.uint32)
    bits = (words[:, :, None] >> shifts) & np.uint32(1)
    return bits.reshape(rows, -1)[:, :cols].astype(bool)


# ---------------------------------------------------------------------------
# Cosine objective  ([PermLLM] optimization objective)
# ---------------------------------------------------------------------------

def cosine_loss(Yd: np.ndarray, Ys: np.ndarray) -> Tuple[float, np.ndarray]:
    """Mean over tokens (columns) of 1 - cos(y_d, y_s); returns (loss, cos per token)."""
    dot = np.sum(Yd * Ys, axis=0)
    nd = np.sqrt(np.sum(Yd * Yd, axis=0))
    ns = np.sqrt(np.sum(Ys * Ys, axis=0))
    cos = dot / np.maximum(nd * ns, COS_EPS)
    return float(np.mean(1.0 - cos)), cos


def cosine_loss_grad(Yd: np.ndarray, Ys: np.ndarray) -> np.ndarray:
    """d loss / d Ys for the token-averaged cosine loss (same shape as Ys)."""
    T = Ys.shape[1]
    dot = np.sum(Yd * Ys, axis=0)
    nd = np.sqrt(np.sum(Yd * Yd, axis=0))
    ns = np.sqrt(np.sum(Ys * Ys, axis=0))
    den = nd * ns
    G = np.empty_like(Ys)
    ok = den > COS_EPS
    c = np.where(ok, dot / np.where(ok, den, 1.0), 0.0)
    with np.errstate(divide="ignore", invalid="ignore"):
        g_ok = -(Yd / np.where(ok, den, 1.0) - c * Ys / np.where(ok, ns * ns, 1.0)) / T
    g_clamped = -(Yd / COS_EPS) / T
    G[:, ok] = g_ok[:, ok]
    G[:, ~ok] = g_clamped[:, ~ok]
    return G


# ---------------------------------------------------------------------------
# Hardening  ([PermLLM] Method 2)
# ---------------------------------------------------------------------------

def harden(P: np.ndarray) -> np.ndarray:
    """Per block, the permutation maximising Tr(P_b^T P_hat_b) = sum_i P_hat_b[i, pi(i)].

    Returns pi as an int array [nb, B] (row i of block b goes to column pi[b, i]).
    The maximisation is a linear assignment problem; scipy's solver is the step
    used here (the pins check it against enumeration of all permutations).
    When several permutations reach the maximum any of them is a correct result.
    """
    from scipy.optimize import linear_sum_assignment
    P = np.asarray(P, np.float64)
    nb, B, _ = P.shape
    perm = np.empty((nb, B), np.int64)
    for b in range(nb):
        rows, cols = linear_sum_assignment(P[b], maximize=True)
        perm[b, rows] = cols
    return perm


def perm_matrix(perm: np.ndarray) -> np.ndarray:
    """The 0/1 matrices of per-block permutations pi: P[b, i, pi[b, i]] = 1."""
    nb, B = perm.shape
    P = np.zeros((nb, B, B))
    for b in range(nb):
        P[b, np.arange(B), perm[b]] = 1.0
    return P


def assignment_value(P: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """Per block, sum_i P[b, i, pi[b, i]] (the objective the hardening maximises)."""
    nb, B = perm.shape
    return np.array([np.sum(np.asarray(P[b], np.float64)[np.arange(B), perm[b]]) for b in range(nb)])


# ---------------------------------------------------------------------------
# One forward + backward step of one layer
# ---------------------------------------------------------------------------

def importance(W: np.ndarray, X_tokens: np.ndarray, kind: str) -> np.ndarray:
    """Pruning metric S ([PermLLM] integration with pruning methods; reading 11):
    "magnitude" |W|, "wanda" |W_ij| ||X_j||, "ria" (|W_ij| / col sum + |W_ij| / row sum) ||X_j||^0.5."""
    A = np.abs(np.asarray(W, np.float64))
    xn = np.sqrt(np.sum(np.asarray(X_tokens, np.float64) ** 2, axis=0))      # ||X_j|| over the tokens
    if kind == "magnitude":
        return A
    if kind == "wanda":
        return A * xn[None, :]
    if kind == "ria":
        col = A.sum(axis=0, keepdims=True)       # sum over output rows of column j
        row = A.sum(axis=1, keepdims=True)       # sum over input columns of row i
        return (A / col + A / row) * np.sqrt(xn)[None, :]
    raise ValueError(kind)


def forward(W: np.ndarray, X_tokens: np.ndarray, logits: np.ndarray, tau: float, n_iters: int,
            n: int, m: int, mask: Optional[np.ndarray] = None, Wp: Optional[np.ndarray] = None,
            P: Optional[np.ndarray] = None, score: Optional[np.ndarray] = None) -> Dict[str, object]:
    """Forward pass in the pages' order.

    ``X_tokens`` is [T, C_in]; internally X = X_tokens^T (C_in x T).
    ``mask`` / ``Wp`` / ``P`` inject a given mask, permuted weight or soft
    permutation in place of the computed one (used to compare with another
    implementation on identical intermediate values).  ``score`` is an
    importance matrix S [C_out, C_in]: the mask is then taken from
    S_hat = S P_B instead of |W'| ([PermLLM] integration with pruning methods).
    """
    W = np.asarray(W, np.float64)
    Xc = np.asarray(X_tokens, np.float64).T
    trace = None
    if P is None:
        P, trace = sinkhorn(logits, tau, n_iters)
    else:
        P = np.asarray(P, np.float64)
    Wp_used = permute_weight(W, P) if Wp is None else np.asarray(Wp)
    Shat = None if score is None else permute_weight(np.asarray(score, np.float64), P)
    if mask is not None:
        M = np.asarray(mask, bool)
    else:
        M = nm_mask(Wp_used if Shat is None else Shat, n, m)
    Wp64 = np.asarray(Wp_used, np.float64)
    A = np.where(M, Wp64, 0.0)
    Xp = permute_inputs(P, Xc)
    Ys = A @ Xp
    Yd = W @ Xc
    loss, cos = cosine_loss(Yd, Ys)
    return dict(P=P, trace=trace, Wp=Wp64, mask=M, A=A, Xc=Xc, Xp=Xp, Yd=Yd, Ys=Ys,
                loss=loss, cos=cos, W=W, Shat=Shat)


def backward(fw: Dict[str, object], tau: float) -> Dict[str, np.ndarray]:
    """Hand-written reverse pass to the logits, mask held constant (straight-through).

    Ys = A Xp        ->  dA = G Xp^T,  dXp = A^T G
    Xp = P_B^T X     ->  dP_b += X_b dXp_b^T
    A = M * W'       ->  dW' = M * dA
    W' = W P_B       ->  dP_b += W_b^T dW'_b
    then back through the Sinkhorn normalisations.
    """
    P = fw["P"]
    nb, B, _ = P.shape
    G = cosine_loss_grad(fw["Yd"], fw["Ys"])
    dA = G @ fw["Xp"].T
    dXp = fw["A"].T @ G
    dWp = np.where(fw["mask"], dA, 0.0)
    W, Xc = fw["W"], fw["Xc"]
    dP = np.empty_like(P)
    for b in range(nb):
        s = slice(b * B, (b + 1) * B)
        dP[b] = Xc[s, :] @ dXp[s, :].T + W[:, s].T @ dWp[:, s]
    out = dict(G=G, dA=dA, dWp=dWp, dP=dP)
    if fw["trace"] is not None:
        out["dL"] = sinkhorn_backward(fw["trace"], P, dP, tau)
    return out


def step(W: np.ndarray, X_tokens: np.ndarray, logits: np.ndarray, tau: float, n_iters: int,
         n: int, m: int, mask: Optional[np.ndarray] = None, score: Optional[np.ndarray] = None) -> Dict[str, object]:
    """Forward and backward of one layer; returns the forward dict plus G, dP, dL."""
    fw = forward(W, X_tokens, logits, tau, n_iters, n, m, mask=mask, score=score)
    fw.update(backward(fw, tau))
    return fw


def step_hard(W: np.ndarray, X_tokens: np.ndarray, logits: np.ndarray, tau: float, n_iters: int,
              n: int, m: int, perm: Optional[np.ndarray] = None,
              mask: Optional[np.ndarray] = None, score: Optional[np.ndarray] = None) -> Dict[str, object]:
    """Forward with the hardened permutation, backward straight through it.

    P_hat = Sinkhorn(L / tau); P = harden(P_hat) (or the given ``perm``, to
    compare with another implementation's choice among tied maxima); the
    forward pass uses P; the reverse pass computes dP for P exactly as in
    ``backward`` and hands it to the Sinkhorn reverse pass as dP_hat
    (dP/dP_hat = 1).
    """
    P_soft, trace = sinkhorn(logits, tau, n_iters)
    if perm is None:
        perm = harden(P_soft)
    P_hard = perm_matrix(np.asarray(perm))
    fw = forward(W, X_tokens, logits, tau, n_iters, n, m, mask=mask, P=P_hard, score=score)
    fw.update(backward(fw, tau))
    fw["dL"] = sinkhorn_backward(trace, P_soft, fw["dP"], tau)
    fw["P_soft"], fw["perm"], fw["trace"] = P_soft, np.asarray(perm), trace
    return fw


def loss_of_logits(W, X_tokens, logits, tau, n_iters, n, m, mask=None) -> float:
    return forward(W, X_tokens, logits, tau, n_iters, n, m, mask=mask)["loss"]


# ---------------------------------------------------------------------------
# Training loop  ([PermLLM] "Implementation details")
# ---------------------------------------------------------------------------

def adamw_update(L, g, m, v, t, lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01):
    """One AdamW step (decoupled decay, bias-corrected moments); returns new (L, m, v)."""
    L, g, m, v = (np.asarray(a, np.float64) for a in (L, g, m, v))
    m = beta1 * m + (1.0 - beta1) * g
    v = beta2 * v + (1.0 - beta2) * g * g
    m_hat = m / (1.0 - beta1 ** t)
    v_hat = v / (1.0 - beta2 ** t)
    L = L * (1.0 - lr * weight_decay) - lr * m_hat / (np.sqrt(v_hat) + eps)
    return L, m, v


def tau_schedule(s: int, total: int, tau_start: float = 1.0, tau_end: float = 0.1) -> float:
    """Temperature of step s of a total-step run, linear from tau_start to tau_end."""
    if total <= 1:
        return float(tau_start)
    return float(tau_start + (tau_end - tau_start) * s / (total - 1))


def train(W, X_tokens, logits, n_iters, n, m, total, steps=None, lr=1e-3, tau_start=1.0, tau_end=0.1,
          hard=False, **adam):
    """``steps`` (default all) training steps: forward + backward at tau_s, then
    AdamW on L.  Returns the logits after the last step, the per-step losses and
    the last step's dL."""
    L = np.asarray(logits, np.float64).copy()
    mom = np.zeros_like(L)
    vel = np.zeros_like(L)
    losses, dL = [], None
    for s in range(total if steps is None else steps):
        tau = tau_schedule(s, total, tau_start, tau_end)
        fw = (step_hard if hard else step)(W, X_tokens, L, tau, n_iters, n, m)
        losses.append(fw["loss"])
        dL = fw["dL"]
        L, mom, vel = adamw_update(L, dL, mom, vel, s + 1, lr=lr, **adam)
    return L, losses, dL


# ---------------------------------------------------------------------------
# Inference side  ([PermLLM] "Effect on inference acceleration")
# ---------------------------------------------------------------------------
# The deployed layer computes y = A x_pi with A = M (.) (W P_B) (hard P_B, 2:4
# mask) and x_pi = P_B^T x.  The functions below restate that product on the
# compressed form of A (reading 12): gather the inputs, then for every kept
# entry multiply by the input at its position.

def gather_channels(X_tokens: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """x_pi = P_B^T x for every token: X_pi[t, bB + perm[b, i]] = X[t, bB + i].

    ``perm`` [nb, B] is the hardening's permutation (row i of block b goes to
    column perm[b, i]), so the source channel i of block b lands in slot perm[b, i].
    """
    X = np.asarray(X_tokens)
    perm = np.asarray(perm)
    nb, B = perm.shape
    out = np.empty_like(X)
    for b in range(nb):
        out[:, b * B + perm[b]] = X[:, b * B:(b + 1) * B]
    return out


def pack_24(A: np.ndarray, mask: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Compressed 2:4 form of A under ``mask`` (exactly two kept of every four
    consecutive columns): values[:, 2g + k] is the k-th kept entry of group g in
    column order and idx[:, 2g + k] its position 0..3 in the group."""
    A = np.asarray(A)
    M = np.asarray(mask, bool)
    rows, cols = A.shape
    if cols % 4:
        raise ValueError("columns must be a multiple of 4")
    G = M.reshape(rows, cols // 4, 4)
    if not np.all(G.sum(axis=2) == 2):
        raise ValueError("every group of four must keep exactly two entries")
    # positions of the kept entries, ascending: a stable sort puts kept (key 0) first
    pos = np.argsort(np.where(G, 0, 1), axis=2, kind="stable")[:, :, :2]
    vals = np.take_along_axis(A.reshape(rows, cols // 4, 4), pos, axis=2)
    return vals.reshape(rows, cols // 2), pos.reshape(rows, cols // 2).astype(np.int64)


def meta_words(idx: np.ndarray) -> np.ndarray:
    """Positions -> 32-bit metadata words (reading 12): group g's field at bits
    4 (g % 8) of word g // 8, first position in the low two bits."""
    idx = np.asarray(idx, np.uint64)
    rows, half = idx.shape
    if half % 16:
        raise ValueError("columns must be a multiple of 32")
    field = idx[:, 0::2] | (idx[:, 1::2] << np.uint64(2))          # [rows, groups]
    field = field.reshape(rows, half // 16, 8)
    shifts = (np.uint64(4) * np.arange(8, dtype=np.uint64))
    return (field << shifts).sum(axis=2).astype(np.uint32)


def unpack_24(vals: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """The dense matrix of a compressed form (zeros where nothing is kept)."""
    vals = np.asarray(vals, np.float64)
    rows, half = vals.shape
    cols = 4 * (np.arange(half) // 2)[None, :] + np.asarray(idx)
    A = np.zeros((rows, 2 * half))
    A[np.arange(rows)[:, None], cols] = vals
    return A


def sparse24_mm(vals: np.ndarray, idx: np.ndarray, X_tokens: np.ndarray,
                perm: Optional[np.ndarray] = None) -> np.ndarray:
    """Y[t, o] = sum over the kept entries k of row o of vals[o, k] * x_pi[t, slot(o, k)],
    slot(o, k) = 4 (k // 2) + idx[o, k]; x_pi = gather_channels(X, perm) (``perm``
    None: X is already in permuted order).  Returns Y as [T, rows]."""
    Xp = np.asarray(X_tokens, np.float64)
    if perm is not None:
        Xp = gather_channels(Xp, perm)
    vals = np.asarray(vals, np.float64)
    rows, half = vals.shape
    slot = 4 * (np.arange(half) // 2)[None, :] + np.asarray(idx)
    Y = np.empty((Xp.shape[0], rows))
    for r0 in range(0, rows, 128):
        r1 = min(rows, r0 + 128)
        Y[:, r0:r1] = np.einsum("ok,tok->to", vals[r0:r1], Xp[:, slot[r0:r1]])
    return Y


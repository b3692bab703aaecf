"""Pins of the CPU oracle to facts fixed by the pages and by mathematics.

Each test checks the oracle against something other than itself: a closed
form, an invariant, a textbook special case written independently, brute force
over every permutation of a toy layer, or finite differences.  A plausible
slip in the oracle (rows and columns swapped, iteration order reversed, tau
dropped, P used where P^T belongs, a backward term dropped, the tie rule
reversed) fails at least one of them.
"""

import itertools
import math

import numpy as np
import pytest

from oracle import lcp_oracle as O

import autograd_reference as AR


def rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


# ---------------------------------------------------------------- Sinkhorn --

def test_sinkhorn_zero_logits_give_uniform():
    for B in (4, 32, 64):
        P, _ = O.sinkhorn(np.zeros((3, B, B)), 0.5, 5)
        assert np.allclose(P, 1.0 / B, rtol=0, atol=1e-15)


def test_sinkhorn_additive_logits_give_uniform_after_one_iteration():
    # L_ij = a_i + b_j: the row step removes a_i, the column step removes b_j.
    B = 16
    a, b = rand((B, 1), 1), rand((1, B), 2)
    L = (a + b)[None]
    for iters in (1, 2, 5):
        P, _ = O.sinkhorn(L, 0.7, iters)
        assert np.allclose(P, 1.0 / B, rtol=0, atol=1e-14)


def test_sinkhorn_columns_sum_to_one_after_any_iteration_count():
    L = rand((4, 32, 32), 3, 2.0)
    for iters in (1, 2, 3, 5):
        P, _ = O.sinkhorn(L, 0.5, iters)
        assert np.allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-12)


def test_sinkhorn_doubly_stochastic_at_init_scale():
    # logits ~ N(0, 1e-3) (initialisation std of the blog page, section 6)
    L = rand((64, 64, 64), 4, 1e-3)
    P, _ = O.sinkhorn(L, 0.5, 5)
    assert np.max(np.abs(P.sum(axis=1) - 1)) < 1e-12
    assert np.max(np.abs(P.sum(axis=2) - 1)) < 1e-5


def test_sinkhorn_peaked_logits_converge_to_doubly_stochastic():
    rng = np.random.default_rng(5)
    L = np.stack([np.eye(32)[rng.permutation(32)] * 3.0 + rng.standard_normal((32, 32)) * 0.5
                  for _ in range(3)])
    P, _ = O.sinkhorn(L, 1.0, 200)
    assert np.max(np.abs(P.sum(axis=1) - 1)) < 1e-12
    assert np.max(np.abs(P.sum(axis=2) - 1)) < 1e-5


def test_sinkhorn_equals_linear_domain_sinkhorn_knopp_row_first():
    # Textbook Sinkhorn-Knopp in the linear domain, in the order the pages fix:
    # S_i = T_c(T_r(S_{i-1})), i.e. rows normalised before columns.
    rng = np.random.default_rng(6)
    L = rng.standard_normal((2, 8, 8)) * 1.5
    tau = 0.6
    for iters in (1, 2, 3, 7):
        K = np.exp(L / tau)
        for _ in range(iters):
            for b in range(K.shape[0]):
                for i in range(8):
                    K[b, i, :] = K[b, i, :] / sum(K[b, i, :])
                for j in range(8):
                    K[b, :, j] = K[b, :, j] / sum(K[b, :, j])
        P, _ = O.sinkhorn(L, tau, iters)
        assert np.allclose(P, K, rtol=1e-12, atol=0)


def test_sinkhorn_order_matters_so_the_previous_test_bites():
    rng = np.random.default_rng(7)
    L = rng.standard_normal((1, 8, 8))
    P, _ = O.sinkhorn(L, 1.0, 1)
    K = np.exp(L[0])
    K = K / K.sum(axis=0, keepdims=True)
    K = K / K.sum(axis=1, keepdims=True)          # column first: the wrong order
    assert not np.allclose(P[0], K, rtol=1e-6, atol=0)


def test_sinkhorn_2x2_limit_closed_form_with_temperature():
    # A positive 2x2 matrix scaled to doubly stochastic form is [[p,1-p],[1-p,p]]
    # and diagonal scaling keeps the cross ratio: p^2/(1-p)^2 = K00 K11 / (K01 K10),
    # so p = sigmoid((Z00 + Z11 - Z01 - Z10) / 2) with Z = L / tau.
    rng = np.random.default_rng(8)
    for _ in range(20):
        L = rng.standard_normal((1, 2, 2))
        tau = float(rng.uniform(0.5, 2.0))
        d = (L[0, 0, 0] + L[0, 1, 1] - L[0, 0, 1] - L[0, 1, 0]) / tau
        p = 1.0 / (1.0 + math.exp(-d / 2))
        P, _ = O.sinkhorn(L, tau, 3000)
        assert np.allclose(P[0], [[p, 1 - p], [1 - p, p]], rtol=0, atol=1e-10)


def test_sinkhorn_row_shift_invariance():
    L = rand((3, 16, 16), 9)
    shift = rand((3, 16, 1), 10, 5.0)
    P1, _ = O.sinkhorn(L, 0.5, 4)
    P2, _ = O.sinkhorn(L + shift, 0.5, 4)
    assert np.allclose(P1, P2, rtol=1e-12, atol=1e-15)


def test_sinkhorn_peaked_permutation_is_recovered_exactly():
    rng = np.random.default_rng(11)
    B, nb = 32, 3
    sig = [rng.permutation(B) for _ in range(nb)]
    L = np.zeros((nb, B, B))
    for b in range(nb):
        L[b, np.arange(B), sig[b]] = 60.0       # P_b[i, sigma(i)] = 1
    P, _ = O.sinkhorn(L, 0.5, 5)
    for b in range(nb):
        Pi = np.zeros((B, B))
        Pi[np.arange(B), sig[b]] = 1.0
        assert np.array_equal(P[b], Pi) or np.max(np.abs(P[b] - Pi)) < 1e-40
        assert np.array_equal(np.argmax(P[b], axis=1), sig[b])


# ------------------------------------------------------- block permutation --

def test_block_products_equal_dense_block_diagonal_products():
    rng = np.random.default_rng(12)
    W = rng.standard_normal((10, 24))
    X = rng.standard_normal((24, 7))
    P, _ = O.sinkhorn(rng.standard_normal((3, 8, 8)), 0.5, 3)
    PB = O.block_diag(P)
    assert np.allclose(O.permute_weight(W, P), W @ PB, rtol=1e-13, atol=1e-15)
    assert np.allclose(O.permute_inputs(P, X), PB.T @ X, rtol=1e-13, atol=1e-15)
    # block-diagonal structure
    assert np.count_nonzero(PB) == 3 * 64


def test_peaked_permutation_makes_wprime_an_exact_gather():
    rng = np.random.default_rng(13)
    B, nb = 8, 4
    W = rng.standard_normal((5, nb * B))
    L = np.zeros((nb, B, B))
    sig = [rng.permutation(B) for _ in range(nb)]
    for b in range(nb):
        L[b, np.arange(B), sig[b]] = 80.0
    P, _ = O.sinkhorn(L, 0.5, 5)
    Wp = O.permute_weight(W, P)
    for b in range(nb):
        for i in range(B):   # source channel bB+i lands in slot bB+sigma(i)
            assert np.array_equal(Wp[:, b * B + sig[b][i]], W[:, b * B + i])


# ------------------------------------------------------------------ N:M mask --

def _textbook_nm(W, n, m):
    """Plain N:M magnitude pruning written with explicit loops and an explicit tie key."""
    rows, cols = W.shape
    keep = np.zeros((rows, cols), bool)
    for r in range(rows):
        for g in range(cols // m):
            idx = list(range(g * m, (g + 1) * m))
            best = sorted(idx, key=lambda j: (-abs(float(W[r, j])), j))[:n]
            for j in best:
                keep[r, j] = True
    return keep


@pytest.mark.parametrize("n,m", [(2, 4), (4, 8), (1, 4), (3, 4), (1, 8), (7, 8)])
def test_mask_equals_textbook_pruning_with_ties(n, m):
    rng = np.random.default_rng(14)
    # quantised values give many exact ties, including +0 / -0
    W = np.round(rng.standard_normal((12, 64)) * 2) / 2
    W[0, :8] = [0.0, -0.0, 0.0, -0.0, 1.0, -1.0, 1.0, -1.0]
    assert np.array_equal(O.nm_mask(W, n, m), _textbook_nm(W, n, m))


def test_mask_characterisation_invariants():
    rng = np.random.default_rng(15)
    for (n, m) in ((2, 4), (4, 8)):
        W = np.round(rng.standard_normal((40, 128)) * 3) / 3
        M = O.nm_mask(W, n, m)
        g = M.reshape(40, -1, m)
        assert np.all(g.sum(axis=2) == n)
        mag = np.abs(W).reshape(40, -1, m)
        for r in range(40):
            for k in range(g.shape[1]):
                kept = [j for j in range(m) if g[r, k, j]]
                drop = [j for j in range(m) if not g[r, k, j]]
                for a in kept:
                    for b in drop:
                        assert mag[r, k, a] >= mag[r, k, b]
                        if mag[r, k, a] == mag[r, k, b]:
                            assert a < b


def test_identity_logits_collapse_to_plain_nm_pruning():
    rng = np.random.default_rng(16)
    B, nb = 16, 4
    W = rng.standard_normal((20, nb * B))
    # exp(-800) underflows to 0 in float64, so P is exactly the identity
    L = np.broadcast_to(np.eye(B) * 400.0, (nb, B, B)).copy()
    P, _ = O.sinkhorn(L, 0.5, 5)
    assert np.array_equal(P, np.broadcast_to(np.eye(B), P.shape))
    Wp = O.permute_weight(W, P)
    assert np.array_equal(Wp, W)
    assert np.array_equal(O.nm_mask(Wp, 2, 4), _textbook_nm(W, 2, 4))


def test_zero_logits_make_block_columns_equal_and_keep_the_first_n():
    rng = np.random.default_rng(17)
    B = 8
    W = rng.standard_normal((6, 4 * B))
    P, _ = O.sinkhorn(np.zeros((4, B, B)), 1.0, 5)
    Wp = O.permute_weight(W, P)
    # P = 1/B exactly, so every column of a block is the same block mean; the
    # summation order can differ between columns only by rounding, so compare
    # the mask on the exact block means instead.
    means = np.repeat(W.reshape(6, 4, B).mean(axis=2), B, axis=1)
    M = O.nm_mask(means, 2, 4)
    assert np.all(M.reshape(6, -1, 4)[:, :, :2]) and not np.any(M.reshape(6, -1, 4)[:, :, 2:])
    assert np.allclose(Wp, means, rtol=1e-14, atol=1e-16)


def test_mask_bit_packing():
    M = np.zeros((2, 64), bool)
    M[0, 0::2] = True          # 0x55555555 in both words
    M[1, 31] = True            # top bit of word 0
    M[1, 32] = True            # bottom bit of word 1
    words = O.pack_mask_bits(M)
    assert words.dtype == np.uint32
    assert words.tolist() == [[0x55555555, 0x55555555], [0x80000000, 0x00000001]]
    assert np.array_equal(O.unpack_mask_bits(words, 64), M)


# ------------------------------------------------------------------- loss --

def test_cosine_loss_special_values():
    rng = np.random.default_rng(18)
    Yd = rng.standard_normal((9, 5))
    assert abs(O.cosine_loss(Yd, Yd)[0]) < 1e-15
    assert abs(O.cosine_loss(Yd, -Yd)[0] - 2.0) < 1e-15
    assert abs(O.cosine_loss(Yd, 3.5 * Yd)[0]) < 1e-15
    a = np.array([[1.0, 0.0], [0.0, 2.0]])
    b = np.array([[0.0, 3.0], [1.0, 0.0]])
    assert abs(O.cosine_loss(a, b)[0] - 1.0) < 1e-15
    # one token at 45 degrees: 1 - 1/sqrt(2)
    u = np.array([[1.0], [0.0]])
    v = np.array([[1.0], [1.0]])
    assert abs(O.cosine_loss(u, v)[0] - (1 - 1 / math.sqrt(2))) < 1e-15


def test_cosine_loss_per_token_scale_invariance():
    rng = np.random.default_rng(19)
    Yd, Ys = rng.standard_normal((2, 11, 6))
    s = rng.uniform(0.1, 10.0, size=6)
    assert abs(O.cosine_loss(Yd * s, Ys * s)[0] - O.cosine_loss(Yd, Ys)[0]) < 1e-14


def test_cosine_loss_gradient_by_finite_differences():
    rng = np.random.default_rng(20)
    Yd, Ys = rng.standard_normal((2, 7, 4))
    G = O.cosine_loss_grad(Yd, Ys)
    eps = 1e-6
    num = np.zeros_like(Ys)
    for idx in np.ndindex(Ys.shape):
        e = np.zeros_like(Ys)
        e[idx] = eps
        num[idx] = (O.cosine_loss(Yd, Ys + e)[0] - O.cosine_loss(Yd, Ys - e)[0]) / (2 * eps)
    assert np.linalg.norm(G - num) / np.linalg.norm(num) < 1e-8
    # the gradient is orthogonal to y_s token by token (scale invariance)
    assert np.max(np.abs(np.sum(G * Ys, axis=0))) < 1e-14


def test_cosine_loss_gradient_in_the_clamped_region_by_finite_differences():
    """Reading: the cosine denominator is max(|y_d| |y_s|, 1e-8).  Where the clamp
    binds (here a token whose sparse output is exactly zero) the token's loss is
    1 - <y_d, y_s> / 1e-8, linear in y_s, so its gradient is -y_d / (1e-8 T).
    Both points of every central difference stay inside the clamp region
    (|y_d| h < 1e-8), where the difference is exact for a linear function."""
    rng = np.random.default_rng(22)
    Yd, Ys = rng.standard_normal((2, 6, 3))
    Ys[:, 1] = 0.0                      # token 1: zero-norm sparse output, the clamp binds
    G = O.cosine_loss_grad(Yd, Ys)
    T = Ys.shape[1]
    h = 1e-2 * O.COS_EPS / np.linalg.norm(Yd[:, 1])
    num = np.zeros(Ys.shape[0])
    for k in range(Ys.shape[0]):
        e = np.zeros_like(Ys)
        e[k, 1] = h
        num[k] = (O.cosine_loss(Yd, Ys + e)[0] - O.cosine_loss(Yd, Ys - e)[0]) / (2 * h)
    assert np.allclose(G[:, 1], num, rtol=1e-6, atol=0)
    assert np.allclose(G[:, 1], -Yd[:, 1] / (O.COS_EPS * T), rtol=1e-15, atol=0)
    # the token's loss is 1 there (cosine 0 at y_s = 0), and the other tokens are unaffected
    _, cos = O.cosine_loss(Yd, Ys)
    assert cos[1] == 0.0
    G_ref = O.cosine_loss_grad(Yd[:, [0, 2]], Ys[:, [0, 2]]) * 2 / 3
    assert np.allclose(G[:, [0, 2]], G_ref, rtol=1e-14, atol=0)


# -------------------------------------------------------- brute force over 8! --

def _hard_loss_independent(W, X_tokens, sigma, n, m):
    """Loss of a hard permutation computed in original channel order.

    Source channel i sits at permuted slot sigma[i].  Each group of m
    consecutive slots is a set of source channels; in every row the n largest
    |W| of that set survive (equal magnitudes: lower slot first).  The sparse
    output is the pruned W applied to the unpermuted X.
    """
    rows, cols = W.shape
    inv = np.argsort(sigma)                       # slot -> source channel
    Ws = np.zeros_like(W)
    for r in range(rows):
        for g in range(cols // m):
            slots = list(range(g * m, (g + 1) * m))
            best = sorted(slots, key=lambda j: (-abs(W[r, inv[j]]), j))[:n]
            for j in best:
                Ws[r, inv[j]] = W[r, inv[j]]
    X = X_tokens.T
    yd, ys = W @ X, Ws @ X
    c = np.sum(yd * ys, 0) / (np.linalg.norm(yd, axis=0) * np.linalg.norm(ys, axis=0))
    return float(np.mean(1 - c))


@pytest.mark.slow
def test_brute_force_all_permutations_of_an_8_channel_toy():
    rng = np.random.default_rng(21)
    Cout, Cin, T, n, m = 16, 8, 32, 2, 4
    W = rng.standard_normal((Cout, Cin)) * 0.02
    X = rng.standard_normal((T, Cin))
    perms = list(itertools.permutations(range(Cin)))
    assert len(perms) == 40320
    ind = np.array([_hard_loss_independent(W, X, np.array(s), n, m) for s in perms])
    # only the partition of the 8 channels into two groups of 4 matters: 35 values
    assert len(np.unique(np.round(ind, 12))) <= 35
    # oracle forward with the hard permutation injected as P reproduces every loss
    Pall = np.zeros((len(perms), 1, Cin, Cin))
    for k, s in enumerate(perms):
        Pall[k, 0, np.arange(Cin), np.array(s)] = 1.0
    orc = np.array([O.forward(W, X, None, 1.0, 0, n, m, P=Pall[k])["loss"] for k in range(len(perms))])
    assert np.max(np.abs(orc - ind)) < 1e-12
    # ... and so do peaked logits through the Sinkhorn path (a sample of them)
    for k in rng.choice(len(perms), 300, replace=False):
        L = Pall[k] * 80.0
        assert abs(O.forward(W, X, L, 0.5, 5, n, m)["loss"] - ind[k]) < 1e-12
    best = np.argmin(ind)
    assert ind[best] < ind[0] or best == 0


def test_no_pruning_and_hard_permutation_gives_zero_loss():
    rng = np.random.default_rng(22)
    W = rng.standard_normal((6, 16))
    X = rng.standard_normal((9, 16))
    P = np.zeros((2, 8, 8))
    for b in range(2):
        P[b, np.arange(8), rng.permutation(8)] = 1.0
    assert abs(O.forward(W, X, None, 1.0, 0, 4, 4, P=P)["loss"]) < 1e-14
    # soft P: W P P^T != W, so the loss is positive even with nothing pruned
    Ps, _ = O.sinkhorn(rng.standard_normal((2, 8, 8)), 1.0, 5)
    assert O.forward(W, X, None, 1.0, 0, 4, 4, P=Ps)["loss"] > 1e-6


def test_loss_invariant_to_weight_scale_and_token_scale():
    rng = np.random.default_rng(23)
    W = rng.standard_normal((12, 16)) * 0.02
    X = rng.standard_normal((10, 16))
    L = rng.standard_normal((2, 8, 8)) * 0.3
    base = O.forward(W, X, L, 0.5, 5, 2, 4)["loss"]
    assert abs(O.forward(3.0 * W, X, L, 0.5, 5, 2, 4)["loss"] - base) < 1e-13
    s = rng.uniform(0.2, 5, size=(10, 1))
    assert abs(O.forward(W, X * s, L, 0.5, 5, 2, 4)["loss"] - base) < 1e-13


# ------------------------------------------------------------ gradient dL --

def _fd_check(W, X, L, tau, iters, n, m, entries, eps=1e-6):
    out = O.step(W, X, L, tau, iters, n, m)
    dL = out["dL"]
    num, ana = [], []
    for idx in entries:
        Lp, Lm = L.copy(), L.copy()
        Lp[idx] += eps
        Lm[idx] -= eps
        fp = O.forward(W, X, Lp, tau, iters, n, m)
        fm = O.forward(W, X, Lm, tau, iters, n, m)
        if not (np.array_equal(fp["mask"], out["mask"]) and np.array_equal(fm["mask"], out["mask"])):
            continue
        num.append((fp["loss"] - fm["loss"]) / (2 * eps))
        ana.append(dL[idx])
    num, ana = np.array(num), np.array(ana)
    assert len(num) >= 0.5 * len(entries)
    return np.linalg.norm(num - ana) / np.linalg.norm(num)


@pytest.mark.parametrize("iters,tau", [(1, 1.0), (3, 0.5), (5, 0.5)])
def test_dL_matches_central_finite_differences(iters, tau):
    rng = np.random.default_rng(24 + iters)
    Cout, Cin, T, B = 24, 16, 20, 8
    W = rng.standard_normal((Cout, Cin)) * 0.02
    X = rng.standard_normal((T, Cin))
    L = rng.standard_normal((Cin // B, B, B)) * 0.5
    entries = [idx for idx in np.ndindex(L.shape)]
    assert _fd_check(W, X, L, tau, iters, 2, 4, entries) < 1e-6


def test_dL_finite_differences_4of8_with_outliers():
    rng = np.random.default_rng(30)
    Cout, Cin, T, B = 16, 32, 12, 16
    W = rng.standard_normal((Cout, Cin)) * 0.02
    W[:, 5] *= 10
    X = rng.standard_normal((T, Cin))
    X[:, 5] *= 5
    L = rng.standard_normal((Cin // B, B, B)) * 0.5
    entries = [tuple(int(v) for v in rng.integers(0, [2, B, B])) for _ in range(64)]
    assert _fd_check(W, X, L, 0.5, 5, 4, 8, entries) < 1e-6


def test_dL_rows_sum_to_zero():
    rng = np.random.default_rng(31)
    W = rng.standard_normal((20, 32)) * 0.02
    X = rng.standard_normal((15, 32))
    L = rng.standard_normal((4, 8, 8))
    dL = O.step(W, X, L, 0.5, 5, 2, 4)["dL"]
    assert np.max(np.abs(dL.sum(axis=2))) < 1e-12 * np.max(np.abs(dL)) * 64


def test_token_shards_sum_to_the_full_gradient():
    # loss is a token mean, so per-shard gradients weighted by shard size add up
    rng = np.random.default_rng(32)
    W = rng.standard_normal((20, 32)) * 0.02
    X = rng.standard_normal((30, 32))
    L = rng.standard_normal((4, 8, 8)) * 0.2
    full = O.step(W, X, L, 0.5, 5, 2, 4)
    a = O.step(W, X[:12], L, 0.5, 5, 2, 4)
    b = O.step(W, X[12:], L, 0.5, 5, 2, 4)
    assert abs((12 * a["loss"] + 18 * b["loss"]) / 30 - full["loss"]) < 1e-14
    assert np.allclose((12 * a["dL"] + 18 * b["dL"]) / 30, full["dL"], rtol=1e-10, atol=1e-16)


# --------------------------------------------------------------- hardening ---

def _all_perm_values(Pb):
    B = Pb.shape[0]
    return {pi: float(sum(Pb[i, pi[i]] for i in range(B))) for pi in itertools.permutations(range(B))}


@pytest.mark.parametrize("B", [2, 3, 5, 7])
def test_harden_attains_the_brute_force_maximum(B):
    """Tr(P^T P_hat) at the hardened P equals the maximum over all B! permutations."""
    rng = np.random.default_rng(100 + B)
    L = rng.normal(0, 1.0, (4, B, B))
    P, _ = O.sinkhorn(L, 0.7, 5)
    perm = O.harden(P)
    vals = O.assignment_value(P, perm)
    for b in range(4):
        allv = _all_perm_values(P[b])
        assert np.isclose(vals[b], max(allv.values()), rtol=0, atol=1e-12)
        assert sorted(perm[b]) == list(range(B))


def test_harden_recovers_a_dominant_permutation():
    """P_hat = 0.7 Pi + 0.3 / B (doubly stochastic) hardens to Pi itself."""
    rng = np.random.default_rng(5)
    B = 16
    pis = np.stack([rng.permutation(B) for _ in range(3)])
    P = 0.7 * O.perm_matrix(pis) + 0.3 / B
    assert np.array_equal(O.harden(P), pis)


def test_harden_ties_give_a_valid_permutation_with_the_maximum():
    """Uniform P_hat: every permutation is optimal; the result is a permutation of value 1."""
    P = np.full((2, 8, 8), 1.0 / 8)
    perm = O.harden(P)
    for b in range(2):
        assert sorted(perm[b]) == list(range(8))
    assert np.allclose(O.assignment_value(P, perm), 1.0)


def test_step_hard_forward_equals_the_soft_path_at_the_hard_matrix():
    """The hardened forward is the plain forward evaluated at P = perm_matrix(pi)."""
    rng = np.random.default_rng(8)
    W = rng.normal(0, 0.02, (16, 32))
    X = rng.normal(0, 1, (24, 32))
    L = rng.normal(0, 0.3, (2, 16, 16))
    fw = O.step_hard(W, X, L, 0.5, 5, 2, 4)
    ref = O.forward(W, X, L, 0.5, 5, 2, 4, P=O.perm_matrix(fw["perm"]))
    assert fw["loss"] == ref["loss"]
    assert np.array_equal(fw["mask"], ref["mask"])
    # a hard permutation makes W' an exact column gather
    Wp = np.concatenate([W[:, b * 16:(b + 1) * 16][:, np.argsort(fw["perm"][b])] for b in range(2)], axis=1)
    assert np.array_equal(fw["Wp"], Wp)


def test_step_hard_straight_through_gradient():
    """dL is the Sinkhorn reverse pass of the hard-P gradient (dP_hat = dP), and it
    differs from the soft-path dL (the estimator is not the true derivative)."""
    rng = np.random.default_rng(9)
    W = rng.normal(0, 0.02, (16, 32))
    X = rng.normal(0, 1, (24, 32))
    L = rng.normal(0, 0.3, (2, 16, 16))
    fw = O.step_hard(W, X, L, 0.5, 5, 2, 4)
    P_soft, trace = O.sinkhorn(L, 0.5, 5)
    assert np.array_equal(P_soft, fw["P_soft"])
    dP = fw["dP"]
    assert np.allclose(fw["dL"], O.sinkhorn_backward(trace, P_soft, dP, 0.5), rtol=0, atol=0)
    # dP of the hard path by finite differences in P at the hard matrix (mask held)
    P_hard = O.perm_matrix(fw["perm"])
    eps = 1e-6
    for (b, i, j) in [(0, 1, 2), (1, 5, 7), (0, 15, 0)]:
        Pp, Pm = P_hard.copy(), P_hard.copy()
        Pp[b, i, j] += eps
        Pm[b, i, j] -= eps
        lp = O.forward(W, X, L, 0.5, 5, 2, 4, P=Pp, mask=fw["mask"])["loss"]
        lm = O.forward(W, X, L, 0.5, 5, 2, 4, P=Pm, mask=fw["mask"])["loss"]
        assert np.isclose((lp - lm) / (2 * eps), dP[b, i, j], rtol=1e-5, atol=1e-9)
    soft = O.step(W, X, L, 0.5, 5, 2, 4)
    assert not np.allclose(soft["dL"], fw["dL"])


# --------------------------------------------------------- training loop ---

def test_adamw_first_step_closed_form():
    """t = 1 from zero moments: m_hat = g and v_hat = g^2, so the step is
    L (1 - lr wd) - lr g / (|g| + eps)."""
    rng = np.random.default_rng(30)
    L = rng.normal(size=50)
    g = rng.normal(size=50)
    out, m, v = O.adamw_update(L, g, np.zeros(50), np.zeros(50), 1, lr=5e-3, weight_decay=0.01)
    assert np.allclose(out, L * (1 - 5e-5) - 5e-3 * g / (np.abs(g) + 1e-8), rtol=1e-14, atol=0)
    assert np.allclose(m, 0.1 * g) and np.allclose(v, 0.001 * g * g)


def test_adamw_constant_gradient_and_pure_decay():
    """A constant gradient keeps m_hat = g, v_hat = g^2 at every t (bias correction
    exact): k steps move L by k lr g / (|g| + eps) without decay; a zero gradient
    only decays, L (1 - lr wd)^k."""
    g = np.array([0.3, -2.0, 1e-3])
    L = np.array([1.0, -1.0, 0.5])
    m = v = np.zeros(3)
    x = L.copy()
    for t in range(1, 8):
        x, m, v = O.adamw_update(x, g, m, v, t, lr=1e-3, weight_decay=0.0)
    assert np.allclose(x, L - 7 * 1e-3 * g / (np.abs(g) + 1e-8), rtol=1e-12, atol=1e-15)
    x, m, v = L.copy(), np.zeros(3), np.zeros(3)
    for t in range(1, 6):
        x, m, v = O.adamw_update(x, np.zeros(3), m, v, t, lr=1e-2, weight_decay=0.1)
    assert np.allclose(x, L * (1 - 1e-3) ** 5, rtol=1e-14, atol=0)


def test_adamw_matches_torch_adamw():
    """Five steps on random gradients agree with torch.optim.AdamW (float64, CPU)."""
    import torch
    rng = np.random.default_rng(31)
    L0 = rng.normal(size=(3, 4, 4))
    grads = [rng.normal(size=(3, 4, 4)) for _ in range(5)]
    p = torch.nn.Parameter(torch.from_numpy(L0.copy()))
    opt = torch.optim.AdamW([p], lr=5e-3, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.01)
    x, m, v = L0.copy(), np.zeros_like(L0), np.zeros_like(L0)
    for t, gr in enumerate(grads, start=1):
        p.grad = torch.from_numpy(gr.copy())
        opt.step()
        x, m, v = O.adamw_update(x, gr, m, v, t, lr=5e-3)
    assert np.allclose(x, p.detach().numpy(), rtol=1e-12, atol=1e-14)


def test_tau_schedule_endpoints_and_linearity():
    assert O.tau_schedule(0, 11) == 1.0
    assert np.isclose(O.tau_schedule(10, 11), 0.1)
    assert np.allclose(np.diff([O.tau_schedule(s, 11) for s in range(11)]), -0.09)
    assert O.tau_schedule(0, 1) == 1.0


def test_train_loop_lowers_the_loss_and_uses_the_schedule():
    """Twenty steps on a toy layer with outlier channels lower the loss, and the
    first step is the plain step at tau = 1."""
    rng = np.random.default_rng(32)
    W = rng.normal(0, 0.02, (32, 64))
    W[:, [3, 40]] *= 10
    X = rng.normal(0, 1, (96, 64))
    X[:, [3, 40]] *= 5
    L0 = rng.normal(0, 1e-3, (2, 32, 32))
    L, losses, _ = O.train(W, X, L0, 5, 2, 4, total=20, lr=5e-3)
    assert losses[0] == O.step(W, X, L0, 1.0, 5, 2, 4)["loss"]
    assert losses[-1] < losses[0]
    assert not np.allclose(L, L0)


# ------------------------------------------------------ importance scores ---

def test_importance_scores_by_explicit_loops():
    rng = np.random.default_rng(50)
    W = rng.normal(size=(5, 8))
    X = rng.normal(size=(7, 8))
    S_w = O.importance(W, X, "wanda")
    S_r = O.importance(W, X, "ria")
    for i in range(5):
        for j in range(8):
            xn = math.sqrt(sum(X[t, j] ** 2 for t in range(7)))
            col = sum(abs(W[k, j]) for k in range(5))
            row = sum(abs(W[i, k]) for k in range(8))
            assert math.isclose(S_w[i, j], abs(W[i, j]) * xn, rel_tol=1e-12)
            assert math.isclose(S_r[i, j], (abs(W[i, j]) / col + abs(W[i, j]) / row) * math.sqrt(xn), rel_tol=1e-12)


def test_score_mask_maximises_each_group_sum():
    """The mask keeps, in every group of M, the N-subset with the largest sum of S_hat
    (argmax over masks of sum (M . S_hat) for each group), checked by enumeration."""
    rng = np.random.default_rng(51)
    W = rng.normal(size=(6, 16))
    X = rng.normal(size=(9, 16))
    L = rng.normal(0, 0.5, (2, 8, 8))
    S = O.importance(W, X, "wanda")
    fw = O.forward(W, X, L, 0.7, 5, 2, 4, score=S)
    Sh = fw["Shat"]
    for i in range(6):
        for g in range(4):
            vals = Sh[i, 4 * g:4 * g + 4]
            best = max(sum(vals[list(c)]) for c in itertools.combinations(range(4), 2))
            assert np.isclose(vals[fw["mask"][i, 4 * g:4 * g + 4]].sum(), best)


def test_magnitude_score_with_a_hard_permutation_is_the_plain_mask():
    """S = |W| and P a permutation: S_hat = |W P| = |W'|, so the masks agree (the
    two scores differ only for soft P)."""
    rng = np.random.default_rng(52)
    W = rng.normal(size=(12, 32))
    X = rng.normal(size=(10, 32))
    pis = np.stack([rng.permutation(16) for _ in range(2)])
    P = O.perm_matrix(pis)
    S = O.importance(W, X, "magnitude")
    a = O.forward(W, X, None, 1.0, 5, 2, 4, P=P, score=S)["mask"]
    b_ = O.forward(W, X, None, 1.0, 5, 2, 4, P=P)["mask"]
    assert np.array_equal(a, b_)


def test_wanda_with_equal_channel_norms_is_magnitude():
    rng = np.random.default_rng(53)
    W = rng.normal(size=(8, 16))
    X = np.ones((4, 16)) * np.array([1, -1, 1, -1])[:, None]     # every ||X_j|| = 2
    assert np.allclose(O.importance(W, X, "wanda"), 2 * np.abs(W))


# --------------------------------------------------------- inference side ---

def test_pack_24_worked_example():
    """One row by hand: groups (1, -5, 3, 2) and (0.5, 4, -4, 1) keep (-5, 3) at
    positions 1, 2 and (4, -4) at 1, 2 (|4| = |-4|: both are the two largest);
    every field is 1 | 2 << 2 = 9.  With x = 1..8: -5*2 + 3*3 + 4*6 - 4*7 = -5."""
    W = np.array([[1.0, -5.0, 3.0, 2.0, 0.5, 4.0, -4.0, 1.0]])
    M = O.nm_mask(W, 2, 4)
    vals, idx = O.pack_24(W, M)
    assert vals.tolist() == [[-5.0, 3.0, 4.0, -4.0]]
    assert idx.tolist() == [[1, 2, 1, 2]]
    assert int(O.meta_words(np.tile(idx, (1, 8)))[0, 0]) == 0x99999999
    Y = O.sparse24_mm(vals, idx, np.arange(1.0, 9.0)[None, :])
    assert Y.tolist() == [[-5.0]]


def test_meta_words_field_by_field():
    rng = np.random.default_rng(60)
    first = rng.integers(0, 3, (3, 16))
    second = first + 1 + rng.integers(0, 3 - first)      # first < second <= 3
    idx = np.stack([first, second], axis=2).reshape(3, 32)
    words = O.meta_words(idx)
    for r in range(3):
        for g in range(16):
            field = (int(words[r, g // 8]) >> (4 * (g % 8))) & 0xF
            assert field & 3 == first[r, g] and field >> 2 == second[r, g]


def test_pack_24_round_trip_and_positions():
    rng = np.random.default_rng(61)
    A = rng.normal(size=(6, 64))
    M = O.nm_mask(rng.normal(size=(6, 64)), 2, 4)
    vals, idx = O.pack_24(A, M)
    assert np.array_equal(O.unpack_24(vals, idx), np.where(M, A, 0.0))
    assert np.all(idx[:, 0::2] < idx[:, 1::2])
    with pytest.raises(ValueError):
        O.pack_24(A, O.nm_mask(A, 1, 4))


def test_gather_is_the_block_permutation_of_the_inputs():
    """x_pi = P_B^T x: as token rows, X_pi = X P_B with P_B from perm_matrix."""
    rng = np.random.default_rng(62)
    pis = np.stack([rng.permutation(8) for _ in range(3)])
    X = rng.normal(size=(5, 24))
    assert np.array_equal(O.gather_channels(X, pis), X @ O.block_diag(O.perm_matrix(pis)))
    ident = np.tile(np.arange(8), (3, 1))
    assert np.array_equal(O.gather_channels(X, ident), X)


def test_sparse24_mm_is_the_hardened_sparse_output():
    """The deployed product on the compressed weight equals the training
    forward's sparse output Y_s = A P_B^T X for the same hard permutation and
    mask (a different route: dense block-diagonal matrices)."""
    rng = np.random.default_rng(63)
    W = rng.normal(size=(10, 32))
    X = rng.normal(size=(7, 32))
    pis = np.stack([rng.permutation(16) for _ in range(2)])
    fw = O.forward(W, X, None, 1.0, 5, 2, 4, P=O.perm_matrix(pis))
    vals, idx = O.pack_24(fw["A"], fw["mask"])
    Y = O.sparse24_mm(vals, idx, X, pis)
    assert np.allclose(Y.T, fw["Ys"], rtol=1e-12, atol=1e-12)


def test_sparse24_mm_by_explicit_loops():
    rng = np.random.default_rng(64)
    vals = rng.normal(size=(3, 8))
    idx = np.array([[0, 3, 1, 2, 0, 1, 2, 3]] * 3)
    X = rng.normal(size=(2, 16))
    pis = np.array([rng.permutation(8), rng.permutation(8)])
    Y = O.sparse24_mm(vals, idx, X, pis)
    src = {}                     # slot -> source channel
    for b in range(2):
        for i in range(8):
            src[8 * b + pis[b, i]] = 8 * b + i
    for t in range(2):
        for o in range(3):
            ref = sum(vals[o, k] * X[t, src[4 * (k // 2) + idx[o, k]]] for k in range(8))
            assert math.isclose(Y[t, o], ref, rel_tol=1e-12, abs_tol=1e-12)


# ---------------------------------------------------------------------------
# The reverse pass against autograd of an independent torch restatement
# ---------------------------------------------------------------------------

def _small(seed, B, cin_blocks=2, cout=12, T=10, lscale=0.5):
    rng = np.random.default_rng(seed)
    W = rng.standard_normal((cout, cin_blocks * B)) * 0.02
    X = rng.standard_normal((T, cin_blocks * B))
    L = rng.standard_normal((cin_blocks, B, B)) * lscale
    return W, X, L


def _agree(out, ref):
    assert ref["gap"] > 1e-9                       # the mask is unique: rounding cannot flip it
    assert np.array_equal(out["mask"], ref["mask"])
    assert abs(out["loss"] - ref["loss"]) <= 1e-12 * abs(ref["loss"])
    nrm = np.linalg.norm(ref["dL"])
    assert nrm > 0 and np.linalg.norm(out["dL"] - ref["dL"]) <= 1e-12 * nrm


@pytest.mark.parametrize("B,n,m,iters,tau", [(8, 2, 4, 1, 1.0), (8, 2, 4, 5, 0.5), (16, 4, 8, 3, 0.2),
                                             (16, 2, 4, 20, 0.1)])
def test_dL_equals_autograd_of_a_torch_restatement(B, n, m, iters, tau):
    W, X, L = _small(40 + B + iters, B)
    ref = AR.autograd_step(W, X, L, tau, iters, n, m)
    out = O.step(W, X, L, tau, iters, n, m)
    assert np.max(np.abs(out["P"] - ref["P"])) <= 1e-13
    _agree(out, ref)


def test_hardened_step_equals_autograd_with_a_straight_through_estimator():
    W, X, L = _small(51, 16, lscale=1.0)
    out = O.step_hard(W, X, L, 0.5, 5, 2, 4)
    ref = AR.autograd_step(W, X, L, 0.5, 5, 2, 4, hard_perm=out["perm"])
    assert np.max(np.abs(out["P_soft"] - ref["P"])) <= 1e-13
    _agree(out, ref)


@pytest.mark.parametrize("kind", ["wanda", "ria"])
def test_score_ranked_mask_step_equals_autograd(kind):
    W, X, L = _small(52, 8)
    S = O.importance(W, X, kind)
    out = O.step(W, X, L, 0.5, 5, 2, 4, score=S)
    ref = AR.autograd_step(W, X, L, 0.5, 5, 2, 4, score=S)
    _agree(out, ref)

"""An independent restatement of one step of the method for pinning the oracle
(test infrastructure): the forward equations of [PermLLM] "Method" written with
torch float64 ops, and the gradient to the logits taken by torch autograd
instead of the oracle's hand-written reverse pass.

Independent of the oracle where it matters: Sinkhorn runs in the linear domain
(Sinkhorn-Knopp on exp(L / tau): rows, then columns), the N:M mask is a top-k
per group, the loss is torch's cosine similarity, and every derivative comes
from autograd.  The mask is held constant (its ranking is detached), as the
method's straight-through treatment of the mask prescribes.
"""
import numpy as np
import torch
import torch.nn.functional as F


def autograd_step(W, X_tokens, L, tau, iters, n, m, hard_perm=None, score=None):
    """Loss, soft P, mask, dL/dlogits and the mask's decision gap.

    hard_perm [nb, B]: the forward uses the hard permutation matrices, the
    gradient passes straight through to the soft P (value P_hard, derivative
    that of P_soft).  score [C_out, C_in] (non-negative): the mask ranks
    S P_B instead of |W P_B|.  gap > 0 means no group of the ranking ties at
    its n-th entry, so the mask is unique.
    """
    Lt = torch.tensor(np.asarray(L, np.float64), requires_grad=True)
    K = torch.exp(Lt / tau)
    for _ in range(iters):
        K = K / K.sum(dim=2, keepdim=True)
        K = K / K.sum(dim=1, keepdim=True)
    P = K
    if hard_perm is not None:
        Ph = torch.zeros_like(K)
        nb, B = np.asarray(hard_perm).shape
        for b in range(nb):
            Ph[b, torch.arange(B), torch.as_tensor(np.asarray(hard_perm)[b])] = 1.0
        P = Ph + K - K.detach()
    PB = torch.block_diag(*P)
    Wt = torch.tensor(np.asarray(W, np.float64))
    Xt = torch.tensor(np.asarray(X_tokens, np.float64))            # [T, C_in]
    Wp = Wt @ PB
    rank = (torch.tensor(np.asarray(score, np.float64)) @ PB if score is not None else Wp).detach().abs()
    groups = rank.reshape(Wp.shape[0], -1, m)
    top = groups.topk(n, dim=2)
    M = torch.zeros_like(groups, dtype=torch.bool).scatter_(2, top.indices, True).reshape(Wp.shape)
    Ys = (Xt @ PB) @ torch.where(M, Wp, 0.0).T
    Yd = Xt @ Wt.T
    loss = (1.0 - F.cosine_similarity(Yd, Ys, dim=1)).mean()
    loss.backward()
    dropped = torch.where(M.reshape(groups.shape), -torch.inf, groups).amax(dim=2)
    gap = float((top.values[..., -1] - dropped).min())
    return dict(loss=float(loss.detach()), P=K.detach().numpy(), mask=M.numpy(), dL=Lt.grad.numpy(), gap=gap)

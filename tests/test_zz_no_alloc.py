"""The allocation-free loss entry point (lcp_loss_fwd_static) gives the same
loss as lcp_loss_fwd and as the float64 oracle, called through the C ABI, on
two calls in a row.

lcp_loss_fwd_static exists for callers that cannot allocate device memory: an
embedder whose device memory belongs to another allocator or is reserved up
front under a fixed budget, or a latency-critical pipeline in which
cudaMalloc's implicit synchronisation would stall other streams.  Its scratch
is a static device array shared by every call, so the second call here uses
different shapes to show that the first call's contents do not leak into its
result.  This file is collected last on purpose.
"""

import numpy as np
import pytest
import torch

from learnable_channel_permutation_b200 import binding as b
from oracle import lcp_oracle as O

pytestmark = pytest.mark.gpu

TOL_LOSS = 1e-5   # the float32 loss tolerance of the other GPU tests


def _inputs(T, cout, seed):
    rng = np.random.default_rng(seed)
    Yd = rng.standard_normal((T, cout)).astype(np.float32)
    Ys = (0.6 * Yd + 0.8 * rng.standard_normal((T, cout))).astype(np.float32)
    return Yd, Ys


def test_static_loss_matches_the_allocating_entry_point_and_the_oracle_twice(gpu_lib):
    for T, cout, seed in ((1000, 4096, 1), (37, 264, 2)):
        Yd_h, Ys_h = _inputs(T, cout, seed)
        Yd, Ys = torch.from_numpy(Yd_h).cuda(), torch.from_numpy(Ys_h).cuda()
        ref = torch.empty(1, device="cuda")
        stats = torch.empty(T, 4, device="cuda")
        b.loss_fwd(Yd, Ys, ref, stats)
        got = torch.full((1,), float("nan"), device="cuda")
        b.loss_fwd_static(Yd, Ys, got)
        torch.cuda.synchronize()
        r, g = float(ref[0]), float(got[0])
        assert abs(g - r) <= TOL_LOSS * abs(r), (T, cout, g, r)
        # the oracle takes Y as [C_out, T] (tokens are columns)
        o, _ = O.cosine_loss(Yd_h.T.astype(np.float64), Ys_h.T.astype(np.float64))
        assert abs(g - o) <= TOL_LOSS * abs(o), (T, cout, g, o)


def test_static_loss_rejects_more_tokens_than_its_scratch(gpu_lib):
    L = b.lib()
    st = L.lcp_loss_fwd_static(0x1000, 0x2000, 0x3000, 64, b.STATIC_MAX_TOKENS + 1, None)
    assert st == 2
    assert "LCP_STATIC_MAX_TOKENS" in L.lcp_last_error().decode()

"""LCP_FLAG_CACHED_DENSE: a step that reads Y_d = X W^T from layer.Yd gives the
same P, loss, dL and mask as the step that computes it, and the Y_d a step
writes matches the float64 oracle's dense output."""
import pytest
import torch

from learnable_channel_permutation_b200 import binding as b
from learnable_channel_permutation_b200 import synth

import gpu_helpers as H

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,flags", [("bf16", 0), ("bf16", b.FLAG_SIMT), ("f32", 0)])
def test_cached_dense_step_reproduces_the_full_step(gpu_lib, dtype, flags):
    wl = synth.custom(384, 512, 200, 64, 2, 4, 0.5, 5, dtype, seed=11, outliers=True)
    li = synth.make_inputs(wl)[0]
    W, X, L = H.to_dev(li, dtype)
    d = b.alloc_outputs(W, X, L)
    d["Yd"] = torch.empty(li.spec.tokens, li.spec.cout, dtype=torch.float32, device="cuda")
    full = b.Step([d], wl.block, wl.n, wl.m, wl.iters, wl.tau, flags=flags)
    full.run()
    torch.cuda.synchronize()
    ref = {k: d[k].clone() for k in ("P", "dL", "loss", "mask")}
    ref["loss"] = ref["loss"][:1]        # the layer's loss is the first float
    yd_ref = X.double().cpu().numpy() @ W.double().cpu().numpy().T   # the same rounded inputs, float64
    assert H.relerr(d["Yd"].cpu().numpy(), yd_ref) <= 1e-5
    cached = b.Step([d], wl.block, wl.n, wl.m, wl.iters, wl.tau, flags=flags | b.FLAG_CACHED_DENSE,
                    workspace=full.ws)
    # one GEMM launch computes both outputs on the tensor-core path; the CUDA-core
    # path drops its separate dense GEMM
    tc = dtype == "bf16" and not flags
    assert cached.launches == full.launches - (0 if tc else 1)
    for k in ("P", "dL", "loss", "mask"):
        d[k].fill_(0)
    cached.run()
    torch.cuda.synchronize()
    for k in ("P", "dL", "mask"):
        assert torch.equal(d[k], ref[k]), k
    assert torch.equal(d["loss"][:1], ref["loss"])
    assert b.device_error() == 0

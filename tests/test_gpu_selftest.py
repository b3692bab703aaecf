"""Failure detection without a GPU fault: the bounded wait that every
tensor-core kernel uses gives up after its time limit on a barrier phase that
nothing completes, records its site, and the context keeps working (a whole
step afterwards still matches the oracle)."""
import pytest

from learnable_channel_permutation_b200 import binding as b
from learnable_channel_permutation_b200 import synth

import gpu_helpers as H

pytestmark = pytest.mark.gpu


def test_bounded_wait_expires_reports_and_leaves_the_context_usable(gpu_lib):
    assert b.device_error() == 0
    assert b.selftest_bounded_wait() == 901
    assert b.device_error() == 0          # the step kernels' words were untouched
    wl = synth.custom(256, 512, 160, 64, 2, 4, 0.5, 5, "bf16", seed=8, outliers=True)
    inputs = synth.make_inputs(wl)
    out, _ = H.run_gpu(wl, inputs)
    H.check_layer(inputs[0], wl, out[0], H.TOL_LOSS_BF16, H.TOL_DL_BF16, cos_dl=H.COS_DL_BF16)
